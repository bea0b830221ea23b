// fa_combine_kernel.cuh -- merges the partial results of a key-split forward.
//
// With the keys of each query row split into S contiguous ranges, range s
// yields O_s (normalised over the keys of range s) and lse_s = log of its sum
// of exponentials.  The row's result is exact again after one more step of
// the online-softmax rescaling of page "FlashAttention (ES)", section "Calculo
// de Softmax en linea", taken across the ranges instead of across key tiles:
//     lse = m + log(sum_s exp(lse_s - m)),  m = max_s lse_s
//     O   = sum_s exp(lse_s - lse) O_s
// A range with no allowed key has lse_s = -inf and weight 0; a row with no
// allowed key at all gets O = 0, lse = -inf.
//
// One warp per row (grid-stride); lane l holds columns [l*D/32, (l+1)*D/32),
// so each partial row is one coalesced 4*D-byte read (D = 64, 128 or 256).  Memory-bound:
// S * (4D + 4) bytes read and 4D (or 2D) + 4 written per row.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

template <int D, bool O_BF16>
__global__ void __launch_bounds__(256) fa_combine_kernel(const float *__restrict__ o_part,
                                                          const float *__restrict__ lse_part, void *o, float *lse,
                                                          int n_splits, long long rows) {
    constexpr int W = D / 32;  // columns per lane (2, 4 or 8)
    static_assert(W == 2 || W % 4 == 0, "D / 32 must be 2 or a multiple of 4");
    const int lane = threadIdx.x & 31;
    const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
    const float NEG_INF = __int_as_float(0xff800000);
    for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += n_warps) {
        float m = NEG_INF;
        for (int s = 0; s < n_splits; ++s) m = fmaxf(m, __ldg(lse_part + s * rows + r));
        float acc[W];
#pragma unroll
        for (int i = 0; i < W; ++i) acc[i] = 0.f;
        float wsum = 0.f;
        if (m != NEG_INF) {
            for (int s = 0; s < n_splits; ++s) {
                const float w = expf(__ldg(lse_part + s * rows + r) - m);
                wsum += w;
                const float *src = o_part + ((long long)s * rows + r) * D + lane * W;
                if constexpr (W % 4 == 0) {
#pragma unroll
                    for (int i = 0; i < W; i += 4) {
                        const float4 v = __ldg(reinterpret_cast<const float4 *>(src + i));
                        acc[i + 0] += w * v.x;
                        acc[i + 1] += w * v.y;
                        acc[i + 2] += w * v.z;
                        acc[i + 3] += w * v.w;
                    }
                } else {
                    const float2 v = __ldg(reinterpret_cast<const float2 *>(src));
                    acc[0] += w * v.x;
                    acc[1] += w * v.y;
                }
            }
        }
        const float inv = (m != NEG_INF) ? 1.f / wsum : 0.f;
        if constexpr (O_BF16) {
            uint16_t *dst = reinterpret_cast<uint16_t *>(o) + r * D + lane * W;
            if constexpr (W % 4 == 0) {
#pragma unroll
                for (int i = 0; i < W; i += 4) {
                    uint2 v;
                    v.x = pack_bf16x2(acc[i + 0] * inv, acc[i + 1] * inv);
                    v.y = pack_bf16x2(acc[i + 2] * inv, acc[i + 3] * inv);
                    *reinterpret_cast<uint2 *>(dst + i) = v;
                }
            } else {
                *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
            }
        } else {
            float *dst = reinterpret_cast<float *>(o) + r * D + lane * W;
            if constexpr (W % 4 == 0) {
#pragma unroll
                for (int i = 0; i < W; i += 4)
                    *reinterpret_cast<float4 *>(dst + i) =
                        make_float4(acc[i + 0] * inv, acc[i + 1] * inv, acc[i + 2] * inv, acc[i + 3] * inv);
            } else {
                *reinterpret_cast<float2 *>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
            }
        }
        if (lane == 0) lse[r] = (m != NEG_INF) ? m + logf(wsum) : NEG_INF;
    }
}

}  // namespace fa

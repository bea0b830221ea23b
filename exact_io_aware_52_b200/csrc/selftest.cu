// selftest.cu -- single-CTA checks of the sm_100a building blocks the attention
// kernel is made of, each runnable on its own (include/fa_selftest.h):
//   * a TMA load with 128-byte swizzle, returning the raw shared-memory image;
//   * S = A B^T with tcgen05.mma, both operands K-major in shared memory;
//   * O = P V with tcgen05.mma, P packed into TMEM by tcgen05.st, V MN-major
//     in shared memory;
//   * the same two products with E4M3 operands (tcgen05.mma kind::f8f6f4),
//     P rounded to E4M3 and packed four per TMEM column by the kernel's packer;
//   * the bounded mbarrier wait running out on a barrier nobody arrives at.
// They use exactly the descriptor builders and MMA issue blocks of the kernel.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "fa_selftest.h"
#include "sm100_ptx.cuh"

namespace {

using namespace fa;

constexpr uint64_t kTimeoutNs = 1000000000ull;  // 1 s

struct SelfParams {
    CUtensorMap ta, tb;  // 3-D maps, box {64, 128, 1} (bf16) or {128, 128, 1} (E4M3), 128-byte swizzle
    const uint16_t *p;   // P for the P V check, [128][128] bf16
    const float *pf;     // P for the E4M3 P V check, [128][128] fp32 (rounded on the device)
    float *out;
    uint8_t *raw;
    int32_t *status;
    int K;               // contraction length (S = A B^T) or value width D (P V)
};

__device__ void set_status(int32_t *status, int v) { atomicCAS(reinterpret_cast<int *>(status), 0, v); }

// ---------------------------------------------------------------------------
__global__ void k_tma(const __grid_constant__ SelfParams sp) {
    __shared__ __align__(1024) uint8_t tile[128 * 128];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar, sizeof(tile));
        tma_load_3d(tile, &sp.ta, &bar, 0, 0, 0);
    }
    bool ok = mbar_wait(&bar, 0, &abort_flag, kTimeoutNs);
    if (!ok) set_status(sp.status, 5);
    __syncthreads();
    for (int i = threadIdx.x; i < (int)sizeof(tile); i += blockDim.x) sp.raw[i] = tile[i];
}

// ---------------------------------------------------------------------------
// S[128][128] = A[128][K] * B[128][K]^T, K in {64, 128}
__global__ void k_mma_ss(const __grid_constant__ SelfParams sp) {
    extern __shared__ uint8_t raw_smem[];
    uint8_t *smem = raw_smem + ((1024u - (smem_u32(raw_smem) & 1023u)) & 1023u);
    uint8_t *sA = smem;
    uint8_t *sB = smem + 32768;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 65536);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + 65536 + 64);
    int *abort_flag = reinterpret_cast<int *>(smem + 65536 + 68);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunks = sp.K / 64;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    bool ok = true;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bars[0], 2 * chunks * 16384);
        for (int c = 0; c < chunks; ++c) {
            tma_load_3d(sA + c * 16384, &sp.ta, &bars[0], c * 64, 0, 0);
            tma_load_3d(sB + c * 16384, &sp.tb, &bars[0], c * 64, 0, 0);
        }
        ok = mbar_wait(&bars[0], 0, abort_flag, kTimeoutNs);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, 128, false);
            const uint64_t da = sw128_desc(smem_u32(sA), 16, 1024), db = sw128_desc(smem_u32(sB), 16, 1024);
            if (sp.K == 128) mma_ss_k128(tmem, da, db, idesc, 0u);
            else mma_ss_k64(tmem, da, db, idesc, 0u);
        }
        tc_commit(&bars[1]);
    }
    __syncwarp();
    ok = mbar_wait(&bars[1], 0, abort_flag, kTimeoutNs);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        const int row = warp * 32 + lane;
        for (int ch = 0; ch < 4; ++ch) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, r);
            tmem_ld_wait();
            tmem_reg_fence(r);
            for (int c = 0; c < 32; ++c) sp.out[row * 128 + ch * 32 + c] = __uint_as_float(r[c]);
        }
    } else {
        set_status(sp.status, 5);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// O[128][D] = P[128][128] * V[128][D], P staged through TMEM, D in {64, 128}
__global__ void k_mma_ts(const __grid_constant__ SelfParams sp) {
    extern __shared__ uint8_t raw_smem[];
    uint8_t *smem = raw_smem + ((1024u - (smem_u32(raw_smem) & 1023u)) & 1023u);
    uint8_t *sV = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 32768);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + 32768 + 64);
    int *abort_flag = reinterpret_cast<int *>(smem + 32768 + 68);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = sp.K;
    const int chunks = D / 64;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t colO = 0, colP = 128;
    const int row = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // P row -> TMEM, two bf16 per 32-bit column (low half = even key)
    {
        uint32_t r0[32], r1[32];
        const uint32_t *prow = reinterpret_cast<const uint32_t *>(sp.p + row * 128);
        for (int c = 0; c < 32; ++c) {
            r0[c] = prow[c];
            r1[c] = prow[32 + c];
        }
        tmem_st32(tmem + lane_off + colP, r0);
        tmem_st32(tmem + lane_off + colP + 32, r1);
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    bool ok = true;
    if (threadIdx.x == 0) {
        tc_fence_after();
        mbar_arrive_expect_tx(&bars[0], chunks * 16384);
        for (int c = 0; c < chunks; ++c) tma_load_3d(sV + c * 16384, &sp.tb, &bars[0], c * 64, 0, 0);
        ok = mbar_wait(&bars[0], 0, abort_flag, kTimeoutNs);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, D, true);
            mma_ts_k128(tmem + colO, tmem + colP, sw128_desc(smem_u32(sV), 16384, 1024), idesc, 0u);
        }
        tc_commit(&bars[1]);
    }
    __syncwarp();
    ok = mbar_wait(&bars[1], 0, abort_flag, kTimeoutNs);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + colO + ch * 32, r);
            tmem_ld_wait();
            tmem_reg_fence(r);
            for (int c = 0; c < 32; ++c) sp.out[row * D + ch * 32 + c] = __uint_as_float(r[c]);
        }
    } else {
        set_status(sp.status, 5);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// S[128][128] = A[128][128] * B[128][128]^T, E4M3 operands K-major
__global__ void k_mma_e4m3_ss(const __grid_constant__ SelfParams sp) {
    extern __shared__ uint8_t raw_smem[];
    uint8_t *smem = raw_smem + ((1024u - (smem_u32(raw_smem) & 1023u)) & 1023u);
    uint8_t *sA = smem;
    uint8_t *sB = smem + 16384;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 32768);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + 32768 + 64);
    int *abort_flag = reinterpret_cast<int *>(smem + 32768 + 68);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    bool ok = true;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bars[0], 2 * 16384);
        tma_load_3d(sA, &sp.ta, &bars[0], 0, 0, 0);
        tma_load_3d(sB, &sp.tb, &bars[0], 0, 0, 0);
        ok = mbar_wait(&bars[0], 0, abort_flag, kTimeoutNs);
        if (ok) {
            tc_fence_after();
            mma_e4m3_ss_k128(tmem, sw128_desc(smem_u32(sA), 16, 1024), sw128_desc(smem_u32(sB), 16, 1024),
                             idesc_e4m3_f32(128, 128, false), 0u);
        }
        tc_commit(&bars[1]);
    }
    __syncwarp();
    ok = mbar_wait(&bars[1], 0, abort_flag, kTimeoutNs);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        const int row = warp * 32 + lane;
        for (int ch = 0; ch < 4; ++ch) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, r);
            tmem_ld_wait();
            tmem_reg_fence(r);
            for (int c = 0; c < 32; ++c) sp.out[row * 128 + ch * 32 + c] = __uint_as_float(r[c]);
        }
    } else {
        set_status(sp.status, 5);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// O[128][128] = E4M3(P)[128][128] * V[128][128]: P rounded to E4M3 and packed
// into TMEM by pack_e4m3x4, V (E4M3) MN-major in shared memory
__global__ void k_mma_e4m3_ts(const __grid_constant__ SelfParams sp) {
    extern __shared__ uint8_t raw_smem[];
    uint8_t *smem = raw_smem + ((1024u - (smem_u32(raw_smem) & 1023u)) & 1023u);
    uint8_t *sV = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 16384);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + 16384 + 64);
    int *abort_flag = reinterpret_cast<int *>(smem + 16384 + 68);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t colO = 0, colP = 128;
    const int row = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    {
        uint32_t r[32];
        const float *prow = sp.pf + row * 128;
        for (int c = 0; c < 32; ++c) r[c] = pack_e4m3x4(prow[4 * c], prow[4 * c + 1], prow[4 * c + 2], prow[4 * c + 3]);
        tmem_st32(tmem + lane_off + colP, r);
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    bool ok = true;
    if (threadIdx.x == 0) {
        tc_fence_after();
        mbar_arrive_expect_tx(&bars[0], 16384);
        tma_load_3d(sV, &sp.tb, &bars[0], 0, 0, 0);
        ok = mbar_wait(&bars[0], 0, abort_flag, kTimeoutNs);
        if (ok) {
            tc_fence_after();
            mma_e4m3_ts_k128(tmem + colO, tmem + colP, sw128_desc(smem_u32(sV), 16384, 1024),
                             idesc_e4m3_f32(128, 128, true), 0u);
        }
        tc_commit(&bars[1]);
    }
    __syncwarp();
    ok = mbar_wait(&bars[1], 0, abort_flag, kTimeoutNs);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        for (int ch = 0; ch < 4; ++ch) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + colO + ch * 32, r);
            tmem_ld_wait();
            tmem_reg_fence(r);
            for (int c = 0; c < 32; ++c) sp.out[row * 128 + ch * 32 + c] = __uint_as_float(r[c]);
        }
    } else {
        set_status(sp.status, 5);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// A wait on a barrier that nothing ever arrives at must give up after the
// limit and report it, leaving the context usable.
__global__ void k_wait_timeout(int32_t *status, uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, &abort_flag, timeout_ns);
    if (!ok) set_status(status, 5);
}

// y[i] = 2^x[i] through the FMA-pipe polynomial (pairs of lanes), n even.
__global__ void k_exp2_poly(const float *x, float *y, int n) {
    for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * gridDim.x * blockDim.x) {
        const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = r.x;
        y[i + 1] = r.y;
    }
}

// Exponential-unit rate: every thread runs `iters` passes of 128 exponentials
// of its own values (MIX = 0: independent ex2 only, summed into 8 chains;
// MIX = 1: the softmax's mix per pair of keys, one FFMA2, two ex2, one FADD2
// into 4 chains and one bf16 pack); lane 0 of each warp records the cycles.
template <int MIX>
__global__ void k_mufu_rate(float *sink, long long *cycles, int iters) {
    float s[128];
#pragma unroll
    for (int i = 0; i < 128; ++i) s[i] = (threadIdx.x * 0.001f + i) * 0.01f;
    float m = 0.5f, acc = 0.f;
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
        if (MIX == 0) {
            float b[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 128; ++c) b[c & 7] += ex2_approx(s[c] - m);
            acc += ((b[0] + b[1]) + (b[2] + b[3])) + ((b[4] + b[5]) + (b[6] + b[7]));
        } else {
            const float2 sl2 = make_float2(1.4426950f, 1.4426950f), nm = make_float2(-m, -m);
            float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            uint32_t h = 0;
#pragma unroll
            for (int c = 0; c < 128; c += 2) {
                const float2 xx = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2, nm);
                const float2 pp = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
                a[(c >> 1) & 3] = __fadd2_rn(a[(c >> 1) & 3], pp);
                h ^= pack_bf16x2(pp.x, pp.y);
            }
            acc += (a[0].x + a[1].x) + (a[2].x + a[3].x) + (a[0].y + a[1].y) + (a[2].y + a[3].y) +
                   __uint_as_float(h & 0x3fffffffu);
        }
        m += 1e-7f;
    }
    const long long t1 = clock64();
    sink[blockIdx.x * blockDim.x + threadIdx.x] = acc;
    if ((threadIdx.x & 31) == 0) cycles[blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)] = t1 - t0;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

int make_map(CUtensorMap *m, const void *base, int rows, int cols) {
    auto enc = encoder();
    if (!enc) return 4;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, 1};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? 0
               : 4;
}

// 3-D map over a [rows][128] byte tensor (E4M3), box {128, 128, 1}, 128-byte swizzle
int make_map8(CUtensorMap *m, const void *base, int rows) {
    auto enc = encoder();
    if (!enc) return 4;
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, 1};
    cuuint64_t strides[2] = {128, (cuuint64_t)rows * 128};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? 0
               : 4;
}

int finish(void *stream) {
    if (cudaPeekAtLastError() != cudaSuccess) return 4;
    return cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? 0 : 4;
}

}  // namespace

extern "C" {

int fa_selftest_tma_sw128(const void *src, void *dst, int32_t *status, void *stream) {
    SelfParams sp;
    std::memset(&sp, 0, sizeof sp);
    if (make_map(&sp.ta, src, 128, 64)) return 4;
    sp.raw = static_cast<uint8_t *>(dst);
    sp.status = status;
    k_tma<<<1, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(sp);
    return finish(stream);
}

int fa_selftest_mma_ss(const void *a, const void *b, float *s, int K, int32_t *status, void *stream) {
    if (K != 64 && K != 128) return 1;
    SelfParams sp;
    std::memset(&sp, 0, sizeof sp);
    if (make_map(&sp.ta, a, 128, K) || make_map(&sp.tb, b, 128, K)) return 4;
    sp.out = s;
    sp.status = status;
    sp.K = K;
    const int smem = 65536 + 128 + 1024;
    if (cudaFuncSetAttribute(k_mma_ss, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 4;
    k_mma_ss<<<1, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(sp);
    return finish(stream);
}

int fa_selftest_mma_ts(const void *p, const void *v, float *o, int D, int32_t *status, void *stream) {
    if (D != 64 && D != 128) return 1;
    SelfParams sp;
    std::memset(&sp, 0, sizeof sp);
    if (make_map(&sp.tb, v, 128, D)) return 4;
    sp.p = static_cast<const uint16_t *>(p);
    sp.out = o;
    sp.status = status;
    sp.K = D;
    const int smem = 32768 + 128 + 1024;
    if (cudaFuncSetAttribute(k_mma_ts, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 4;
    k_mma_ts<<<1, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(sp);
    return finish(stream);
}

int fa_selftest_mma_e4m3_ss(const void *a, const void *b, float *s, int32_t *status, void *stream) {
    SelfParams sp;
    std::memset(&sp, 0, sizeof sp);
    if (make_map8(&sp.ta, a, 128) || make_map8(&sp.tb, b, 128)) return 4;
    sp.out = s;
    sp.status = status;
    const int smem = 32768 + 128 + 1024;
    if (cudaFuncSetAttribute(k_mma_e4m3_ss, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 4;
    k_mma_e4m3_ss<<<1, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(sp);
    return finish(stream);
}

int fa_selftest_mma_e4m3_ts(const float *p, const void *v, float *o, int32_t *status, void *stream) {
    SelfParams sp;
    std::memset(&sp, 0, sizeof sp);
    if (make_map8(&sp.tb, v, 128)) return 4;
    sp.pf = p;
    sp.out = o;
    sp.status = status;
    const int smem = 16384 + 128 + 1024;
    if (cudaFuncSetAttribute(k_mma_e4m3_ts, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 4;
    k_mma_e4m3_ts<<<1, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(sp);
    return finish(stream);
}

int fa_selftest_exp2_poly(const float *x, float *y, int n, void *stream) {
    if (n < 0 || (n & 1)) return 1;
    if (n == 0) return 0;
    k_exp2_poly<<<64, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    return finish(stream);
}

int fa_selftest_mufu_rate(int warps_per_subpartition, int mix, int iters, double *cycles_per_pass, void *stream) {
    if (warps_per_subpartition < 1 || warps_per_subpartition > 8 || (mix != 0 && mix != 1) || iters < 1 ||
        iters > 100000 || !cycles_per_pass)
        return 1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return 4;
    const int threads = 128 * warps_per_subpartition, warps = sms * (threads / 32);
    float *sink = nullptr;
    long long *cyc = nullptr;
    if (cudaMalloc(&sink, (size_t)sms * threads * sizeof(float)) != cudaSuccess) return 4;
    if (cudaMalloc(&cyc, (size_t)warps * sizeof(long long)) != cudaSuccess) {
        cudaFree(sink);
        return 4;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int rep = 0; rep < 2; ++rep) {  // the first launch warms up
        if (mix) k_mufu_rate<1><<<sms, threads, 0, st>>>(sink, cyc, iters);
        else k_mufu_rate<0><<<sms, threads, 0, st>>>(sink, cyc, iters);
    }
    int rc = finish(stream);
    if (rc == 0) {
        long long *h = new long long[warps];
        if (cudaMemcpy(h, cyc, (size_t)warps * sizeof(long long), cudaMemcpyDeviceToHost) != cudaSuccess) rc = 4;
        double sum = 0.0;
        for (int i = 0; i < warps; ++i) sum += (double)h[i];
        *cycles_per_pass = sum / warps / iters;
        delete[] h;
    }
    cudaFree(sink);
    cudaFree(cyc);
    return rc;
}

int fa_selftest_wait_timeout(int32_t *status, uint32_t timeout_ms, void *stream) {
    k_wait_timeout<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, (uint64_t)timeout_ms * 1000000ull);
    return finish(stream);
}

}  // extern "C"

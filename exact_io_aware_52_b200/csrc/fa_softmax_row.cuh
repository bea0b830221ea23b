// fa_softmax_row.cuh -- the per-row steps of the online softmax shared by the
// forward kernels (fa_fwd_kernel.cuh for d <= 128, fa_fwd_d256_kernel.cuh for
// d = 256): one thread owns one query row of a 128-row tile, whose scores,
// probabilities and output accumulator sit in its TMEM lane.
//
// The steps follow page "FlashAttention (ES)", section "Calculo de Softmax en
// linea": a reference maximum m and running sums of exponentials relative to
// it are kept per row; a new key tile's terms are taken relative to m, and
// when m must grow the accumulated output and sums are multiplied by
// 2^(m_old - m_new) (base 2: scores are scaled by scale * log2(e)).  The
// masking step is that of section "Fusion de operaciones en un unico kernel
// de CUDA".
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr int BM = 128;  // query rows per tile (tcgen05 M)
constexpr int BN = 128;  // keys per tile

// Running state of one row: reference maximum (log2 units), the sum of the
// unrounded exponentials (gives lse) and the sum of the bf16-rounded ones
// (the weights the tensor core multiplies V by: O's normaliser).
struct RowState {
    float m_ref = 0.f;
    float l = 0.f;
    float lr = 0.f;
};

// The row's 128 scores of one S tile: four 32-column TMEM loads, one wait.
__device__ __forceinline__ void load_score_row(uint32_t t_s, float (&s)[BN]) {
    tmem_ld32f(t_s + 0, s);
    tmem_ld32f(t_s + 32, s + 32);
    tmem_ld32f(t_s + 64, s + 64);
    tmem_ld32f(t_s + 96, s + 96);
    tmem_ld_wait();
    tmem_reg_fence_f<BN>(s);
}

// max of 64 scores: four chains of three-input maxima
__device__ __forceinline__ float max64(const float *v) {
    float a0 = fmaxf(v[0], v[1]), a1 = fmaxf(v[2], v[3]), a2 = fmaxf(v[4], v[5]), a3 = fmaxf(v[6], v[7]);
#pragma unroll
    for (int c = 8; c < 64; c += 8) {
        a0 = fmax3(a0, v[c], v[c + 1]);
        a1 = fmax3(a1, v[c + 2], v[c + 3]);
        a2 = fmax3(a2, v[c + 4], v[c + 5]);
        a3 = fmax3(a3, v[c + 6], v[c + 7]);
    }
    return fmaxf(fmax3(a0, a1, a2), a3);
}

// Masking step for keys [64H, 64H+64) of a tile starting at key kv0: keys at
// or beyond the row's limit get -inf.
template <int H>
__device__ __forceinline__ void mask_scores(float *s, int kv0, int lim) {
#pragma unroll
    for (int c = 64 * H; c < 64 * H + 64; ++c)
        if (kv0 + c >= lim) s[c] = __int_as_float(0xff800000);
}

// Masking step (keys at or beyond the row's limit `lim` get -inf) and the
// row maximum in log2 units.
__device__ __forceinline__ float masked_row_max(float (&s)[BN], int kv0, int lim, float scale_log2) {
    if (kv0 + BN > lim) {
        mask_scores<0>(s, kv0, lim);
        mask_scores<1>(s, kv0, lim);
    }
    return fmaxf(max64(s), max64(s + 64)) * scale_log2;
}

// Reference update for key tile j of the row (j = 0 starts it): the first
// tile sets m_ref (0 for a row whose tile is fully masked); a later one moves
// it only when the tile's maximum exceeds it by more than tau, scaling the
// sums by alpha = 2^(m_old - m_new).  Returns true when O must be scaled by
// alpha as well.
__device__ __forceinline__ bool update_reference(RowState &st, int j, float m_new, float tau, float &alpha) {
    alpha = 1.f;
    if (j == 0) {
        st.m_ref = (m_new == __int_as_float(0xff800000)) ? 0.f : m_new;
        st.l = 0.f;
        st.lr = 0.f;
        return false;
    }
    if (m_new > st.m_ref + tau) {
        alpha = ex2_approx(st.m_ref - m_new);
        st.l *= alpha;
        st.lr *= alpha;
        st.m_ref = m_new;
        return true;
    }
    return false;
}

// O row *= alpha in TMEM (D fp32 columns from t_o); nothing may be adding
// to O while this runs.
template <int D>
__device__ __forceinline__ void rescale_o_row(uint32_t t_o, float alpha) {
#pragma unroll
    for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(t_o + ch * 32, r);
        tmem_ld_wait();
        tmem_reg_fence(r);
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
        tmem_st32(t_o + ch * 32, r);
    }
}

// Probabilities of keys [64H, 64H+64) of one score row against reference -neg_m
// (log2 units): p = 2^(s * scale_log2 - m), summed unrounded into `ls` and
// packed as bf16 pairs (round to nearest even) into pk (column c holds keys
// 64H + 2c and 64H + 2c + 1).
template <int H>
__device__ __forceinline__ void exp_half_p(const float *s, float scale_log2, float neg_m, uint32_t (&pk)[32],
                                           float2 &ls) {
    const float2 sl2 = make_float2(scale_log2, scale_log2);
    const float2 nm = make_float2(neg_m, neg_m);
    float2 a[4] = {ls, make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
        const float2 xx = __ffma2_rn(make_float2(s[64 * H + c], s[64 * H + c + 1]), sl2, nm);
        const float2 pp = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
        a[(c >> 1) & 3] = __fadd2_rn(a[(c >> 1) & 3], pp);
        pk[c >> 1] = pack_bf16x2(pp.x, pp.y);
    }
    ls = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
}

// Sum of a tile's 128 bf16 probabilities (two per word of pk0 and pk1).
__device__ __forceinline__ float rounded_sum(const uint32_t (&pk0)[32], const uint32_t (&pk1)[32]) {
    float b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        b[i & 3] = add_bf16x2_to(b[i & 3], pk0[i]);
        b[(i + 2) & 3] = add_bf16x2_to(b[(i + 2) & 3], pk1[i]);
    }
    return (b[0] + b[1]) + (b[2] + b[3]);
}

// E4M3 probabilities of one 128-key score row: p = 2^(s * scale_log2 - m)
// summed unrounded into `ls` and rounded to E4M3, four keys per 32-bit
// column (key 4c + i in byte i of column c).
// Of every 4 groups of four keys, the second pair of the first kF8PolyGroups
// groups takes its exponentials from the FMA-pipe polynomial instead of MUFU.
constexpr int kF8PolyGroups = 2;
__device__ __forceinline__ void exp_e4m3(const float *s, float scale_log2, float neg_m, uint32_t (&pk)[32],
                                         float2 &ls) {
    const float2 sl2 = make_float2(scale_log2, scale_log2);
    const float2 nm = make_float2(neg_m, neg_m);
    float2 a[4] = {ls, make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 128; c += 4) {
        const float2 x0 = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2, nm);
        const float2 x1 = __ffma2_rn(make_float2(s[c + 2], s[c + 3]), sl2, nm);
        const float2 p0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
        const float2 p1 = ((c >> 2) & 3) < kF8PolyGroups ? exp2_poly2(x1)
                                                          : make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
        a[(c >> 2) & 3] = __fadd2_rn(a[(c >> 2) & 3], __fadd2_rn(p0, p1));
        pk[c >> 2] = pack_e4m3x4(p0.x, p0.y, p1.x, p1.y);
    }
    ls = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
}

template <int D, bool O_BF16>
__device__ __forceinline__ void store_row_chunk(void *o, size_t row_id, int ch, const uint32_t (&r)[32], float inv_l) {
    if constexpr (O_BF16) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(o) + row_id * D + ch * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv_l, __uint_as_float(r[8 * i + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv_l, __uint_as_float(r[8 * i + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv_l, __uint_as_float(r[8 * i + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv_l, __uint_as_float(r[8 * i + 7]) * inv_l);
            dst[i] = v;
        }
    } else {
        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(o) + row_id * D + ch * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(r[4 * i + 0]) * inv_l, __uint_as_float(r[4 * i + 1]) * inv_l,
                                 __uint_as_float(r[4 * i + 2]) * inv_l, __uint_as_float(r[4 * i + 3]) * inv_l);
    }
}

// Fills one output row with a constant (0 for rows without allowed keys, NaN
// for rows of a unit abandoned after a time-out) and sets its lse.
template <int D, bool O_BF16>
__device__ __forceinline__ void fill_row(void *o, float *lse, size_t row_id, bool nan, float lv) {
    if constexpr (O_BF16) {
        const uint16_t b = nan ? 0x7fc0 : 0;
        uint16_t *dst = reinterpret_cast<uint16_t *>(o) + row_id * D;
        for (int i = 0; i < D; ++i) dst[i] = b;
    } else {
        const float f = nan ? __int_as_float(0x7fc00000) : 0.f;
        float *dst = reinterpret_cast<float *>(o) + row_id * D;
        for (int i = 0; i < D; ++i) dst[i] = f;
    }
    lse[row_id] = lv;
}

// Epilogue of one row: O (D fp32 columns in TMEM from t_o) times `scale`
// over the normaliser `norm` to the output row, and lse = ln 2 * lse_log2.
// A row whose normaliser is not positive (no allowed key in its range) gets
// O = 0, lse = -inf.
template <int D, bool O_BF16>
__device__ __forceinline__ void write_row(uint32_t t_o, void *o, float *lse, size_t row_id, bool row_valid, float norm,
                                          float scale, float lse_log2) {
    const float LN2 = 0.69314718055994530942f;
    const bool empty = !(norm > 0.f);
    const float inv_l = empty ? 0.f : scale / norm;
#pragma unroll
    for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(t_o + ch * 32, r);
        tmem_ld_wait();
        tmem_reg_fence(r);
        if (row_valid) store_row_chunk<D, O_BF16>(o, row_id, ch, r, inv_l);
    }
    if (row_valid) lse[row_id] = empty ? __int_as_float(0xff800000) : lse_log2 * LN2;
}

// Epilogue of the 32 rows of one warp through a TMA store (fp32 O): each
// thread scales its row's D columns and writes them into the warp's stage, D / 32
// boxes of [32 rows][32 columns] in the 128-byte swizzle of the O tensor map
// (conflict-free: each 16-byte chunk of a row lands in its own bank group);
// lane 0 then stores the boxes with one TMA store each and returns at once.
// `stage` is 1024-byte aligned; `pending` (lane 0) records that an earlier
// store may still be reading it.  Rows past the head's N are clipped by the
// tensor map; lse goes out per thread.
template <int D>
__device__ __forceinline__ void write_rows_tma(uint32_t t_o, uint8_t *stage, int lane, const CUtensorMap *tm_o,
                                               int row0, int plane, float *lse, size_t first_row_id, int n_valid,
                                               float norm, float lse_log2, bool &pending) {
    const float LN2 = 0.69314718055994530942f;
    const bool empty = !(norm > 0.f);
    const float inv_l = empty ? 0.f : 1.f / norm;
    if (lane == 0 && pending) bulk_wait_group_read0();  // the previous unit's boxes have left the stage
    __syncwarp();
#pragma unroll
    for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(t_o + ch * 32, r);
        tmem_ld_wait();
        tmem_reg_fence(r);
        uint8_t *box = stage + ch * 4096 + lane * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4 *>(box + ((u ^ (lane & 7)) << 4)) =
                make_float4(__uint_as_float(r[4 * u + 0]) * inv_l, __uint_as_float(r[4 * u + 1]) * inv_l,
                            __uint_as_float(r[4 * u + 2]) * inv_l, __uint_as_float(r[4 * u + 3]) * inv_l);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the TMA engine
    __syncwarp();
    if (lane == 0) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) tma_store_3d(tm_o, stage + ch * 4096, ch * 32, row0, plane);
        bulk_commit_group();
        pending = true;
    }
    if (lane < n_valid) lse[first_row_id + lane] = empty ? __int_as_float(0xff800000) : lse_log2 * LN2;
}

}  // namespace fa

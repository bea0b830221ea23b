// fa_bwd_kernel.cuh -- gradients of exact attention on sm_100a.
//
// The pages report the method's training speed-ups (page "FlashAttention
// (ES)", section "Resultados empiricos") without a backward algorithm;
// this is the derivative of the forward definition ("El problema de la
// atencion estandar") computed IO-aware the way the forward is: tiles in
// shared memory and TMEM, P recomputed from Q, K and the forward's lse rather
// than stored.  With sigma the softmax scale, P = exp(sigma Q K^T - lse),
//     dV = P^T dO,  dP = dO V^T,  dS = sigma P o (dP - D),  D_i = dO_i . O_i,
//     dQ = dS K,  dK = dS^T Q.
//
// fa_bwd_prep_kernel computes D and zeroes dQ.  fa_bwd_sm100_kernel: one work
// unit = one 128-key tile of one (b, key/value head); the unit loops over the
// query heads that use the key/value head and over the 128-row query tiles
// that may attend to its keys, keeping dK and dV in TMEM; each query tile's
// dQ contribution is added to the fp32 dQ in global memory by a TMA
// reduce-add from shared memory.  Per query tile t (products on tcgen05,
// bf16 operands, fp32 in TMEM):
//     S^T  = K Q_t^T      -> R_S      (keys x queries)
//     dP^T = V dO_t^T     -> R_P
//     P^T  = exp2(S^T sigma log2e - lse log2e)  (compute warps; bf16 over R_S)
//     dV  += P^T dO_t     (A = P^T from TMEM, B = dO_t MN-major)
//     dS^T = sigma P^T o (dP^T - D)  (compute warps; bf16 over R_P and, as
//                                     the MN-major A of dQ_t, in shared memory)
//     dK  += dS^T Q_t     (A = dS^T from TMEM, B = Q_t MN-major)
//     dQ_t = dS K         -> R_P (A = dS MN-major, B = K MN-major)
// Issue order: S_{t+1} right after dV_t (P_t has been read), so the scores of
// the next tile are ready when the compute warps finish dS_t and the dQ_t
// read-out; dP_{t+1} once dQ_t has left R_P.  dQ_t goes from TMEM through
// the query tile's own (no longer needed) Q and dO buffers, in the 128-byte
// swizzle of the dQ tensor map, to the reduce-add.
// TMEM: R_S [0,128), R_P [128,256), dV [256, 256+D), dK [256+D, 256+2D).
// Warps 0-3 compute (thread = TMEM lane: a key row of S^T, dP^T, dV, dK and a
// query row of dQ_t), warp 4 issues the MMAs, warp 5 the TMA loads, warp 6 the
// dQ reduce-adds.  Every wait is bounded as in the forward kernel.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {
namespace bwd {

constexpr int kThreads = 224;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr int kReduceWarp = 6;  // one thread issues the dQ reduce-adds
constexpr uint32_t kColS = 0, kColP = 128, kColDV = 256;

struct BwdParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;  // Q, dO over [B*H][N][D]; K, V over [B*H_kv][Nk][D]
    CUtensorMap tm_dq;                    // dQ fp32 over [B*H][N][D], box {32, 128, 1}, 128-byte swizzle
    const float *lse;                     // [B, H, N] from the forward
    const float *delta;                   // [B, H, N]: D_i = dO_i . O_i
    float *dq;                            // [B, H, N, D] fp32, zeroed, accumulated by reduce-add
    float *dk, *dv;                       // [B, H_kv, Nk, D] fp32
    const int32_t *k_len;
    int32_t *status;
    int B, H, N, Nk, H_kv, group;
    int n_kv_tiles;                       // ceil(Nk / 128)
    int n_units;                          // B * H_kv * n_kv_tiles
    int band_tiles;                       // key tiles per band of the unit order (see decode_bunit)
    uint32_t *sched;                      // this launch's scheduler slot (as FwdParams::sched)
    int causal;
    float scale;                          // sigma
    float scale_log2;                     // sigma * log2(e)
    uint64_t timeout_ns;
};

template <int D>
struct BCfg {
    static constexpr int kChunks = D / 64;
    static constexpr int kTileBytes = BM * D * 2;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTileBytes;
    static constexpr int kOffQ = kOffV + kTileBytes;      // [2]
    static constexpr int kOffDO = kOffQ + 2 * kTileBytes; // [2]
    static constexpr int kOffDS = kOffDO + 2 * kTileBytes;  // 128 keys x 128 queries bf16, MN-major A of dQ
    static constexpr int kOffCol = kOffDS + BM * BN * 2;     // per-query constants of the tile: 2 x 128 fp32
    static constexpr int kOffBar = kOffCol + 2 * BN * 4;
    static constexpr int kBarKV = 0, kBarKVEmpty = 1;
    static constexpr int kBarSlot = 2, kBarSlotEmpty = 4;  // [2] each; empty: after the dQ reduce read the slot
    static constexpr int kBarS = 6, kBarDP = 7, kBarPReady = 8, kBarDSReady = 9, kBarDQ = 10, kBarRPFree = 11;
    static constexpr int kBarDKV = 12, kBarDKVFree = 13, kBarStage = 14, kBarColReady = 15, kBarColFree = 16;
    static constexpr int kBarDrain = 17;
    static constexpr int kBarUnitFull = 18;                    // [kUnitQueue]
    static constexpr int kBarUnitFree = 18 + kUnitQueue;       // [kUnitQueue]: compute, MMA, reduce threads
    static constexpr int kNumBars = 18 + 2 * kUnitQueue;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 4;
    static constexpr int kOffClaimed = kOffAbort + 4;          // scheduler slot claimed (int)
    static constexpr int kOffUnitIds = kOffClaimed + 4;        // [kUnitQueue][4] ints
    // + slack to align the base to 1024 bytes; at least 117 KB so that one CTA
    // (which allocates all of TMEM) runs per SM
    static constexpr int kSmemBytes =
        (kOffUnitIds + 16 * kUnitQueue + 1024) > 119808 ? (kOffUnitIds + 16 * kUnitQueue + 1024) : 119808;
    static_assert(kTileBytes % 1024 == 0, "1024-byte alignment of swizzled tiles");
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
    static_assert(2 * kSmemBytes > 233472, "one CTA per SM: TMEM is allocated whole");
};

struct BUnit {
    int b, hkv, kvt;   // batch, key/value head, key tile
    int kv0;           // first key
    int klim;          // keys [0, klim) exist and are not padded
    int qt0, nq;       // query tiles [qt0, qt0 + nq) per query head
    int n_iter;        // group * nq (0: the key tile gets no gradient)
};

// Unit numbering: the key tiles of every (b, key/value head) are cut into
// bands of band_tiles consecutive tiles (the first tiles see the most causal
// query tiles); units go band by band, head-major inside a band.  Units are
// handed out dynamically in this order (the forward's unit queue).
__device__ __forceinline__ BUnit decode_bunit(const BwdParams &p, int t) {
    BUnit u;
    const int G = p.B * p.H_kv;
    const int band = t / (p.band_tiles * G);
    const int in_band = t - band * p.band_tiles * G;
    const int bsz = min(p.band_tiles, p.n_kv_tiles - band * p.band_tiles);
    const int g = in_band / bsz;
    u.kvt = band * p.band_tiles + (in_band - g * bsz);
    u.b = g / p.H_kv;
    u.hkv = g - u.b * p.H_kv;
    u.kv0 = u.kvt * BN;
    u.klim = p.Nk;
    if (p.k_len) u.klim = min(max(__ldg(p.k_len + u.b), 0), p.Nk);
    const int n_qt = (p.N + BM - 1) / BM;
    u.qt0 = 0;
    if (p.causal) {  // queries i with i + Nk - N >= kv0 may attend to key kv0
        const int first_q = u.kv0 - (p.Nk - p.N);
        u.qt0 = first_q > 0 ? first_q / BM : 0;
    }
    u.nq = (u.kv0 < u.klim) ? max(0, n_qt - u.qt0) : 0;
    u.n_iter = u.nq * p.group;
    return u;
}

// query head and query tile of iteration `it` of a unit
__device__ __forceinline__ void iter_coord(const BwdParams &p, const BUnit &u, int it, int &bh, int &qt) {
    const int hl = it / u.nq;
    qt = u.qt0 + (it - hl * u.nq);
    bh = u.b * p.H + u.hkv * p.group + hl;
}

__device__ __forceinline__ void record_timeout_b(const BwdParams &p) {
    if (p.status) atomicCAS(reinterpret_cast<int *>(p.status), 0, kStatusTimeout);
}

// 16 bytes of a bf16 row into the 128-byte-swizzled MN-major image: row r of
// a 128-row block, 16-byte unit u of the row's 128 bytes.
__device__ __forceinline__ void st_sw128(uint8_t *block, int r, int u, uint4 v) {
    *reinterpret_cast<uint4 *>(block + r * 128 + ((u ^ (r & 7)) << 4)) = v;
}

// ------------------------------------------------------------------ compute warps
template <int D>
__device__ __forceinline__ bool compute_role(const BwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                             const UnitQueue &uq, uint32_t tmem, uint8_t *smem, int warp,
                                             int lane) {
    using C = BCfg<D>;
    const int r = warp * 32 + lane;  // TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float LOG2E = 1.4426950408889634f;
    const float NEG_INF = __int_as_float(0xff800000);
    const float POS_INF = __int_as_float(0x7f800000);
    uint8_t *s_ds = smem + C::kOffDS;
    float *s_l2 = reinterpret_cast<float *>(smem + C::kOffCol);  // [128] lse log2(e)
    float *s_sd = s_l2 + BN;                                      // [128] sigma D
    const uint64_t to = p.timeout_ns;
    uint32_t gt = 0;  // iterations (global): phase of the per-iteration barriers
    uint32_t gu = 0;  // units with work: phase of dkv / dkv_free
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = unit_pop(uq, k, abort_flag, to, ok);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || t < 0) break;
        const BUnit u = decode_bunit(p, t);
        const int kj = u.kv0 + r;  // this thread's key (rows of S^T, dP^T, dK, dV)
        const size_t kv_row = ((size_t)u.b * p.H_kv + u.hkv) * p.Nk + kj;
        if (u.n_iter == 0) {  // no query attends to these keys: zero gradients
            if (kj < p.Nk) {
                float4 *a = reinterpret_cast<float4 *>(p.dk + kv_row * D);
                float4 *b = reinterpret_cast<float4 *>(p.dv + kv_row * D);
                for (int c = 0; c < D / 4; ++c) a[c] = b[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            continue;
        }
        const bool key_ok = kj < u.klim;
        for (int it = 0; it < u.n_iter && ok; ++it, ++gt) {
            int bh, qt;
            iter_coord(p, u, it, bh, qt);
            const int q0 = qt * BM;
            // the tile's per-query constants into shared memory, one query per
            // thread: lse log2(e) (+inf for queries past N or without a key, so
            // that their P is 0) and sigma D; every thread then reads all 128
            // with broadcast loads
            if (gt > 0) {  // everyone has finished the previous tile's dS
                ok = mbar_wait(&bars[C::kBarColFree], (gt - 1) & 1, abort_flag, to);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            {
                const int qi = q0 + r;
                const float l = qi < p.N ? __ldg(p.lse + (size_t)bh * p.N + qi) : NEG_INF;
                s_l2[r] = l == NEG_INF ? POS_INF : l * LOG2E;
                s_sd[r] = qi < p.N ? p.scale * __ldg(p.delta + (size_t)bh * p.N + qi) : 0.f;
            }
            mbar_arrive(&bars[C::kBarColReady]);
            ok = mbar_wait(&bars[C::kBarColReady], gt & 1, abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            // queries [qlo, N) may attend to key kj (causal: qi >= kj - (Nk - N))
            int qlo = 0;
            if (p.causal) qlo = kj - (p.Nk - p.N);
            const int c_lo = key_ok ? max(0, qlo - q0) : BN;  // first allowed column

            // ---- P^T row
            ok = mbar_wait(&bars[C::kBarS], gt & 1, abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t pk[64];  // P^T row as bf16 pairs (query 2c in the low half)
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float sv[32];
                tmem_ld32f(tmem + lane_off + kColS + ch * 32, sv);
                tmem_ld_wait();
                tmem_reg_fence_f<32>(sv);
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const int col = ch * 32 + c;
                    const float4 l = *reinterpret_cast<const float4 *>(s_l2 + col);
                    float p0 = ex2_approx(fmaf(sv[c], p.scale_log2, -l.x));
                    float p1 = ex2_approx(fmaf(sv[c + 1], p.scale_log2, -l.y));
                    float p2 = ex2_approx(fmaf(sv[c + 2], p.scale_log2, -l.z));
                    float p3 = ex2_approx(fmaf(sv[c + 3], p.scale_log2, -l.w));
                    if (col < c_lo) p0 = 0.f;
                    if (col + 1 < c_lo) p1 = 0.f;
                    if (col + 2 < c_lo) p2 = 0.f;
                    if (col + 3 < c_lo) p3 = 0.f;
                    pk[col >> 1] = pack_bf16x2(p0, p1);
                    pk[(col >> 1) + 1] = pack_bf16x2(p2, p3);
                }
            }
            tmem_st32(tmem + lane_off + kColS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_off + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[C::kBarPReady]);

            // ---- dS^T row = sigma P^T (dP^T - D)
            ok = mbar_wait(&bars[C::kBarDP], gt & 1, abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t ds[16];  // dS^T for queries [32 ch, 32 ch + 32), bf16 pairs
                float dp[32];
                tmem_ld32f(tmem + lane_off + kColP + ch * 32, dp);
                tmem_ld_wait();
                tmem_reg_fence_f<32>(dp);
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const int col = ch * 32 + c;
                    const float4 sd = *reinterpret_cast<const float4 *>(s_sd + col);
                    const uint32_t pa = pk[col >> 1], pb = pk[(col >> 1) + 1];
                    ds[c >> 1] = pack_bf16x2(bf16x2_lo(pa) * fmaf(dp[c], p.scale, -sd.x),
                                             bf16x2_hi(pa) * fmaf(dp[c + 1], p.scale, -sd.y));
                    ds[(c >> 1) + 1] = pack_bf16x2(bf16x2_lo(pb) * fmaf(dp[c + 2], p.scale, -sd.z),
                                                   bf16x2_hi(pb) * fmaf(dp[c + 3], p.scale, -sd.w));
                }
                // over R_P columns [16 ch, 16 ch + 16), whose fp32 dP has been read
                tmem_st16(tmem + lane_off + kColP + ch * 16, ds);
                // dS as the MN-major A operand of dQ = dS K: key row r, queries
                // [32 ch, 32 ch + 32) = 4 16-byte units of 64-query block ch / 2
                uint8_t *blk = s_ds + (ch >> 1) * (BM * 128);
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4)
                    st_sw128(blk, r, (ch & 1) * 4 + u4, make_uint4(ds[4 * u4], ds[4 * u4 + 1], ds[4 * u4 + 2],
                                                                   ds[4 * u4 + 3]));
            }
            tmem_st_wait();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // dS visible to the tensor core
            tc_fence_before();
            mbar_arrive(&bars[C::kBarDSReady]);
            mbar_arrive(&bars[C::kBarColFree]);  // done with this tile's lse and D

            // ---- dQ_t rows (TMEM lane = query q0 + r) into the tile's Q and dO
            // buffers in the dQ map's swizzled layout, then reduce-added to dQ
            ok = mbar_wait(&bars[C::kBarDQ], gt & 1, abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t slot = gt & 1;
            uint8_t *stage[2] = {smem + C::kOffQ + slot * C::kTileBytes, smem + C::kOffDO + slot * C::kTileBytes};
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + kColP + ch * 32, v);
                tmem_ld_wait();
                tmem_reg_fence(v);
                uint8_t *blk = stage[ch / C::kChunks] + (ch % C::kChunks) * (BM * 128);
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8)
                    st_sw128(blk, r, u8, make_uint4(v[4 * u8], v[4 * u8 + 1], v[4 * u8 + 2], v[4 * u8 + 3]));
            }
            tc_fence_before();
            mbar_arrive(&bars[C::kBarRPFree]);  // R_P may take dP of the next tile
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&bars[C::kBarStage]);  // the reduce warp adds the tile to dQ
        }
        if (!ok) break;
        // ---- dK, dV rows of the key tile
        ok = mbar_wait(&bars[C::kBarDKV], gu & 1, abort_flag, to);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            float *out = (which == 0 ? p.dv : p.dk) + kv_row * D;
            const uint32_t col = kColDV + which * D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + col + ch * 32, v);
                tmem_ld_wait();
                tmem_reg_fence(v);
                if (kj < p.Nk) {
                    float4 *o4 = reinterpret_cast<float4 *>(out + ch * 32);
#pragma unroll
                    for (int c = 0; c < 32; c += 4)
                        o4[c / 4] = make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                                __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
                }
            }
        }
        tc_fence_before();
        mbar_arrive(&bars[C::kBarDKVFree]);
        ++gu;
    }
    return ok;
}

// ------------------------------------------------------------------ dQ reduce
// One thread: for every query tile, once the compute warps have staged dQ_t
// in the tile's Q and dO buffers, reduce-add it to dQ through the fp32 map and
// release the buffers to the loader after the copy engine has read them.
template <int D>
__device__ __forceinline__ bool reduce_role(const BwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                            const UnitQueue &uq, uint8_t *smem) {
    using C = BCfg<D>;
    uint32_t gt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = unit_pop(uq, k, abort_flag, p.timeout_ns, ok);
        if (!ok || t < 0) break;
        const BUnit u = decode_bunit(p, t);
        for (int it = 0; it < u.n_iter; ++it, ++gt) {
            if (!mbar_wait(&bars[C::kBarStage], gt & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
            int bh, qt;
            iter_coord(p, u, it, bh, qt);
            const uint32_t slot = gt & 1;
            uint8_t *stage[2] = {smem + C::kOffQ + slot * C::kTileBytes, smem + C::kOffDO + slot * C::kTileBytes};
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch)
                tma_reduce_add_3d(&p.tm_dq, stage[ch / C::kChunks] + (ch % C::kChunks) * (BM * 128), ch * 32,
                                  qt * BM, bh);
            bulk_commit_group();
            bulk_wait_group_read0();
            mbar_arrive(&bars[C::kBarSlotEmpty + slot]);
        }
    }
    bulk_wait_group0();  // every reduce-add has completed before the CTA exits
    return ok;
}

// ------------------------------------------------------------------ MMA issuer
template <int D>
__device__ __forceinline__ bool mma_role(const BwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                         const UnitQueue &uq, uint32_t tmem, uint32_t smem_base) {
    using C = BCfg<D>;
    const uint64_t to = p.timeout_ns;
    // K-major views (contraction over d) and MN-major views (contraction over rows)
    const uint64_t k_km = sw128_desc(smem_base + C::kOffK, 16, 1024);
    const uint64_t v_km = sw128_desc(smem_base + C::kOffV, 16, 1024);
    const uint64_t k_mn = sw128_desc(smem_base + C::kOffK, BM * 128, 1024);
    const uint64_t q_km = sw128_desc(smem_base + C::kOffQ, 16, 1024);
    const uint64_t q_mn = sw128_desc(smem_base + C::kOffQ, BM * 128, 1024);
    const uint64_t do_km = sw128_desc(smem_base + C::kOffDO, 16, 1024);
    const uint64_t do_mn = sw128_desc(smem_base + C::kOffDO, BM * 128, 1024);
    const uint64_t ds_mn = sw128_desc(smem_base + C::kOffDS, BM * 128, 1024);
    const uint32_t id_sp = idesc_bf16_f32(BM, BN, false);            // S^T, dP^T: N = 128 queries
    const uint32_t id_kv = idesc_bf16_f32(BM, D, true);              // dV, dK: B MN-major, N = D
    const uint32_t id_dq = idesc_bf16_f32_ab(BM, D, true, true);     // dQ: A and B MN-major
    const uint32_t slot_step = C::kTileBytes >> 4;
    uint32_t gt = 0, gu = 0, gkv = 0;
    auto qk = [&](uint32_t d_col, uint64_t a, uint64_t b) {
        if constexpr (D == 128) mma_ss_k128(tmem + d_col, a, b, id_sp, 0u);
        else mma_ss_k64(tmem + d_col, a, b, id_sp, 0u);
    };
    auto wait = [&](int bar, uint32_t parity) -> bool {
        if (!mbar_wait(&bars[bar], parity, abort_flag, to)) return false;
        tc_fence_after();
        return true;
    };
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = unit_pop(uq, k, abort_flag, to, ok);
        if (!ok || t < 0) break;
        const BUnit u = decode_bunit(p, t);
        if (u.n_iter == 0) continue;
        if (!wait(C::kBarKV, gkv & 1)) { ok = false; break; }
        ++gkv;
        // scores and dP^T of the unit's first tile
        {
            const uint32_t slot = gt & 1;
            if (!wait(C::kBarSlot + slot, (gt >> 1) & 1)) { ok = false; break; }
            qk(kColS, k_km, q_km + slot * slot_step);
            tc_commit(&bars[C::kBarS]);
            if (gt > 0 && !wait(C::kBarRPFree, (gt - 1) & 1)) { ok = false; break; }
            qk(kColP, v_km, do_km + slot * slot_step);
            tc_commit(&bars[C::kBarDP]);
        }
        for (int it = 0; it < u.n_iter; ++it, ++gt) {
            const uint32_t slot = gt & 1, ns = (gt + 1) & 1;
            const bool more = it + 1 < u.n_iter;
            // dV += P^T dO_t
            if (!wait(C::kBarPReady, gt & 1)) { ok = false; break; }
            if (it == 0 && gu > 0 && !wait(C::kBarDKVFree, (gu - 1) & 1)) { ok = false; break; }
            mma_ts_k128(tmem + kColDV, tmem + kColS, do_mn + slot * slot_step, id_kv, it == 0 ? 0u : 1u);
            // scores of the next tile into R_S (P_t is read by the product above, in order)
            if (more) {
                if (!wait(C::kBarSlot + ns, ((gt + 1) >> 1) & 1)) { ok = false; break; }
                qk(kColS, k_km, q_km + ns * slot_step);
                tc_commit(&bars[C::kBarS]);
            }
            // dK += dS^T Q_t ; dQ_t = dS K into R_P (after dK has read dS^T there)
            if (!wait(C::kBarDSReady, gt & 1)) { ok = false; break; }
            mma_ts_k128(tmem + kColDV + D, tmem + kColP, q_mn + slot * slot_step, id_kv, it == 0 ? 0u : 1u);
            mma_ss_mn_k128(tmem + kColP, ds_mn, k_mn, id_dq, 0u);
            tc_commit(&bars[C::kBarDQ]);
            if (more) {  // dP^T of the next tile once dQ_t has been read out of R_P
                if (!wait(C::kBarRPFree, gt & 1)) { ok = false; break; }
                qk(kColP, v_km, do_km + ns * slot_step);
                tc_commit(&bars[C::kBarDP]);
            } else {
                tc_commit(&bars[C::kBarDKV]);
                tc_commit(&bars[C::kBarKVEmpty]);
            }
        }
        if (!ok) break;
        ++gu;
    }
    return ok;
}

// ------------------------------------------------------------------ TMA producer
template <int D>
__device__ __forceinline__ void load_role(const BwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                          const UnitQueue &uq, uint8_t *smem) {
    using C = BCfg<D>;
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
    prefetch_tensormap(&p.tm_do);
    prefetch_tensormap(&p.tm_dq);
    const uint64_t to = p.timeout_ns;
    uint32_t gt = 0, gkv = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = unit_take(uq, p.sched, p.n_units, true, k, abort_flag, to, ok);
        if (!ok) break;
        unit_publish(uq, k, t, 0, 0);
        if (t < 0) break;
        const BUnit u = decode_bunit(p, t);
        if (u.n_iter == 0) continue;
        if (gkv > 0 && !mbar_wait(&bars[C::kBarKVEmpty], (gkv - 1) & 1, abort_flag, to)) { ok = false; break; }
        const int kv_head = u.b * p.H_kv + u.hkv;
        mbar_arrive_expect_tx(&bars[C::kBarKV], 2 * C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
            tma_load_3d(smem + C::kOffK + c * BM * 128, &p.tm_k, &bars[C::kBarKV], c * 64, u.kv0, kv_head);
            tma_load_3d(smem + C::kOffV + c * BM * 128, &p.tm_v, &bars[C::kBarKV], c * 64, u.kv0, kv_head);
        }
        ++gkv;
        for (int it = 0; it < u.n_iter; ++it, ++gt) {
            const uint32_t slot = gt & 1, round = gt >> 1;
            if (round > 0 && !mbar_wait(&bars[C::kBarSlotEmpty + slot], (round - 1) & 1, abort_flag, to)) {
                ok = false;
                break;
            }
            int bh, qt;
            iter_coord(p, u, it, bh, qt);
            mbar_arrive_expect_tx(&bars[C::kBarSlot + slot], 2 * C::kTileBytes);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
                tma_load_3d(smem + C::kOffQ + slot * C::kTileBytes + c * BM * 128, &p.tm_q, &bars[C::kBarSlot + slot],
                            c * 64, qt * BM, bh);
                tma_load_3d(smem + C::kOffDO + slot * C::kTileBytes + c * BM * 128, &p.tm_do,
                            &bars[C::kBarSlot + slot], c * 64, qt * BM, bh);
            }
        }
    }
    if (!ok) record_timeout_b(p);
    // drain: every copy this thread issued has landed before the CTA may exit
    if (gkv > 0) mbar_wait_drain(&bars[C::kBarKV], (gkv - 1) & 1);
    const uint32_t n = gt < 2u ? gt : 2u;
    for (uint32_t i = 0; i < n; ++i) {
        const uint32_t g = gt - 1 - i;
        mbar_wait_drain(&bars[C::kBarSlot + (g & 1)], (g >> 1) & 1);
    }
}

}  // namespace bwd

// D_i = dO_i . O_i (O fp32 or bf16) and dQ_i = 0; one warp per row.
template <int D, bool O_BF16>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const void *o, const uint16_t *dout, float *delta,
                                                           float *dq, long long rows) {
    const int lane = threadIdx.x & 31;
    const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += n_warps) {
        float acc = 0.f;
        for (int c = lane; c < D; c += 32) {
            const float ov = O_BF16 ? bf16x2_lo(reinterpret_cast<const uint16_t *>(o)[r * D + c])
                                    : reinterpret_cast<const float *>(o)[r * D + c];
            acc += ov * bf16x2_lo(dout[r * D + c]);
            dq[r * D + c] = 0.f;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) delta[r] = acc;
    }
}

template <int D>
__global__ void __launch_bounds__(bwd::kThreads, 1) fa_bwd_sm100_kernel(const __grid_constant__ bwd::BwdParams p) {
    using C = bwd::BCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    volatile int *claimed = reinterpret_cast<volatile int *>(smem + C::kOffClaimed);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const UnitQueue uq{reinterpret_cast<volatile int *>(smem + C::kOffUnitIds), &bars[C::kBarUnitFull],
                       &bars[C::kBarUnitFree]};
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            const bool per_row = i == C::kBarPReady || i == C::kBarDSReady || i == C::kBarRPFree ||
                                 i == C::kBarDKVFree || i == C::kBarStage || i == C::kBarColReady ||
                                 i == C::kBarColFree;
            // a queued unit id is read by the 128 compute threads, the MMA thread and the reduce thread
            const bool unit_free = i >= C::kBarUnitFree && i < C::kBarUnitFree + kUnitQueue;
            mbar_init(&bars[i], unit_free ? 130u : (per_row ? 128u : 1u));
        }
        *abort_flag = 0;
        *claimed = sched_claim(p.sched, p.timeout_ns) ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == bwd::kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (!*claimed) {  // the scheduler slot stayed in use by another launch: no work, report it
        if (threadIdx.x == 0) record_status(p.status, kStatusSchedBusy);
        if (warp == bwd::kMmaWarp) tmem_dealloc(tmem, kTmemCols);
        return;
    }
    if (warp < 4) {
        if (!bwd::compute_role<D>(p, bars, abort_flag, uq, tmem, smem, warp, lane)) bwd::record_timeout_b(p);
    } else if (warp == bwd::kMmaWarp) {
        if (lane == 0) {
            if (!bwd::mma_role<D>(p, bars, abort_flag, uq, tmem, smem_u32(smem))) bwd::record_timeout_b(p);
            tc_commit(&bars[C::kBarDrain]);
            mbar_wait_drain(&bars[C::kBarDrain], 0);
        }
    } else if (warp == bwd::kLoadWarp) {
        if (lane == 0) bwd::load_role<D>(p, bars, abort_flag, uq, smem);
    } else if (warp == bwd::kReduceWarp) {
        if (lane == 0 && !bwd::reduce_role<D>(p, bars, abort_flag, uq, smem)) bwd::record_timeout_b(p);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == bwd::kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0) sched_release(p.sched);
}

}  // namespace fa

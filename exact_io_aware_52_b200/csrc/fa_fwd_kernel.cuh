// fa_fwd_kernel.cuh -- fused exact attention forward for sm_100a.
//
// One launch computes O = softmax(Q K^T * scale + mask) V and the per-row
// logsumexp (page "FlashAttention (ES)", section "El problema de la atencion
// estandar"), following the three techniques of section "Innovaciones clave de
// FlashAttention":
//   * tiling ("Tiling y procesamiento por bloques"): a work unit is one
//     128-row query tile of one (b, h); its 128-key K and V tiles stream from
//     HBM into shared memory through TMA and a multi-stage mbarrier ring, and
//     the score tile S = Q K_j^T never leaves the SM;
//   * online softmax ("Calculo de Softmax en linea"): each row keeps a
//     reference maximum m and a running sum l of exp2 terms; a new tile's
//     terms are taken relative to m, and when m must grow the accumulated
//     output and l are multiplied by 2^(m_old - m_new);
//   * one fused kernel ("Fusion de operaciones en un unico kernel de CUDA"):
//     Q K^T, masking, softmax and the product with V run in this one kernel,
//     which writes only O and lse.
//
// Blackwell mapping (one CTA per SM, persistent over work units):
//   warps 0-3  softmax: thread t owns query row t of the tile; reads its S row
//              from tensor memory (TMEM), masks, updates m and l, writes the
//              bf16 probabilities P back to TMEM, rescales O in TMEM when
//              needed, and runs the epilogue (O / l, lse) for its row;
//   warp 4     MMA issuer (one thread): S_j = Q K_j^T (A and B from shared
//              memory) and O += P_j V_j (A = P from TMEM, B = V_j from shared
//              memory) with tcgen05.mma, fp32 accumulation in TMEM;
//   warp 5     TMA producer (one thread): Q once per work unit, K_j and V_j
//              through the stage ring.
// TMEM (512 columns): S double buffer [0,256), O [256, 256+D), P double
// buffer [384, 512) (128 bf16 keys pack into 64 columns).
// The MMA issue order is Q K_g^T, then P_{g-1} V_{g-1}, over a global sequence
// g of key tiles that runs across work units, so the tensor core computes the
// next score tile while the softmax warps work on the current one.
//
// Every wait is bounded in wall time.  On time-out the CTA raises a shared
// abort flag, records FA_ERR_DEVICE_TIMEOUT in the optional status word,
// drains its in-flight copies and MMAs (again bounded), frees TMEM and exits.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr int BM = 128;  // query rows per tile (tcgen05 M)
constexpr int BN = 128;  // keys per tile
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
__device__ __forceinline__ uint32_t col_s(uint32_t buf) { return buf * 128u; }        // S double buffer
__device__ __forceinline__ uint32_t col_p(uint32_t buf) { return 384u + buf * 64u; }  // P double buffer
constexpr int kStatusTimeout = 5;  // FA_ERR_DEVICE_TIMEOUT

struct FwdParams {
    CUtensorMap tm_q, tm_k, tm_v;  // 3-D maps over [B*H][N][D] bf16; box {64, 128, 1}; 128-byte swizzle
    void *o;                       // [B, H, N, D] fp32 or bf16
    float *lse;                    // [B, H, N]
    const int32_t *k_len;          // [B] or nullptr
    int32_t *status;               // device status word or nullptr
    int B, H, N;
    int n_qtiles;                  // ceil(N / BM)
    int n_tiles;                   // B * H * n_qtiles
    int causal;
    float scale_log2;              // scale * log2(e)
    float tau;                     // rescale threshold in log2 units (<= 0: rescale on any growth)
    uint64_t timeout_ns;
};

template <int D>
struct Cfg {
    static constexpr int kChunks = D / 64;          // 64-element (128-byte) column blocks per row
    static constexpr int kChunkBytes = BM * 128;    // one column block of a 128-row tile
    static constexpr int kTileBytes = BM * D * 2;   // one 128 x D bf16 tile
    static constexpr int kStages = (D == 128) ? 3 : 4;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    // barrier slots
    static constexpr int kBarQFull = 0;
    static constexpr int kBarQEmpty = 1;
    static constexpr int kBarKFull = 2;
    static constexpr int kBarVFull = kBarKFull + kStages;
    static constexpr int kBarKVEmpty = kBarVFull + kStages;
    static constexpr int kBarSFull = kBarKVEmpty + kStages;  // 2
    static constexpr int kBarPFull = kBarSFull + 2;          // 2
    static constexpr int kBarODone = kBarPFull + 2;
    static constexpr int kBarOFinal = kBarODone + 1;
    static constexpr int kBarOFree = kBarOFinal + 1;
    static constexpr int kBarDrain = kBarOFree + 1;
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 4;
    static constexpr int kSmemUsed = kOffAbort + 4;
    static constexpr int kSmemBytes = kSmemUsed + 1024;  // + slack to align the base to 1024 bytes
    static_assert(kChunkBytes % 1024 == 0 && kTileBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
};

struct TileCoord {
    int bh, b, qt, n_kv;
};

// Work unit k of this CTA: bands of gridDim.x consecutive units, walked in
// alternating direction so that per-CTA work evens out when the units'
// costs fall band by band (causal masking puts the longest units first).
__device__ __forceinline__ int unit_index(int k) {
    const int G = gridDim.x, c = blockIdx.x;
    return k * G + ((k & 1) ? (G - 1 - c) : c);
}

__device__ __forceinline__ TileCoord decode_tile(const FwdParams &p, int t) {
    TileCoord tc;
    const int BH = p.B * p.H;
    tc.qt = p.n_qtiles - 1 - t / BH;  // longest (causal) query tiles first
    tc.bh = t % BH;
    tc.b = tc.bh / p.H;
    int kv_end = p.N;
    if (p.k_len) kv_end = min(max(__ldg(p.k_len + tc.b), 0), p.N);
    if (p.causal) kv_end = min(kv_end, (tc.qt + 1) * BM);
    tc.n_kv = (kv_end + BN - 1) / BN;
    return tc;
}

__device__ __forceinline__ void record_timeout(const FwdParams &p) {
    if (p.status) atomicCAS(reinterpret_cast<int *>(p.status), 0, kStatusTimeout);
}

// Bounded wait that ignores the abort flag: used to drain in-flight work.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    int dummy = 0;
    return mbar_wait(bar, parity, &dummy, timeout_ns);
}

template <int D, bool O_BF16>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_sm100_kernel(const __grid_constant__ FwdParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    // 128-byte-swizzled TMA destinations and UMMA operands need 1024-byte alignment
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == C::kBarPFull || i == C::kBarPFull + 1 || i == C::kBarOFree) cnt = kSoftmaxWarps * 32;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kSoftmaxWarps) {
        // ------------------------------------------------------------ softmax
        const int row_in_tile = warp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float LN2 = 0.69314718055994530942f;
        const float NEG_INF = __int_as_float(0xff800000);
        uint32_t g = 0;   // global key-tile counter (same sequence as the MMA issuer)
        uint32_t tl = 0;  // non-empty work units seen
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int t = unit_index(k);
            if (t >= p.n_tiles) break;
            const TileCoord tc = decode_tile(p, t);
            const int row = tc.qt * BM + row_in_tile;
            const bool row_valid = row < p.N;
            const size_t row_id = (size_t)tc.bh * p.N + row;
            int lim = p.N;
            if (p.k_len) lim = min(max(__ldg(p.k_len + tc.b), 0), p.N);
            if (p.causal) lim = min(lim, row + 1);

            if (tc.n_kv == 0) {  // no allowed key in this unit: O = 0, lse = -inf
                if (row_valid) {
                    if constexpr (O_BF16) {
                        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.o) + row_id * D);
                        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.o) + row_id * D);
                        for (int i = 0; i < D / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    p.lse[row_id] = NEG_INF;
                }
                continue;
            }

            float m_ref = 0.f;  // reference maximum, log2 units
            float l = 0.f;      // running sum of 2^(x - m_ref), unrounded: gives lse
            float lr = 0.f;     // running sum of bf16(2^(x - m_ref)), the weights the tensor core
                                // multiplies V by: dividing O by it makes O an exact convex
                                // combination of V rows (a lone dominant weight is not rounded away)
            for (int j = 0; j < tc.n_kv; ++j, ++g) {
                const uint32_t buf = g & 1;
                ok = mbar_wait(&bars[C::kBarSFull + buf], (g >> 1) & 1, abort_flag, p.timeout_ns);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();

                float s[BN];
                {
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    const uint32_t a = tmem + lane_off + col_s(buf);
                    tmem_ld32(a + 0, r0);
                    tmem_ld32(a + 32, r1);
                    tmem_ld32(a + 64, r2);
                    tmem_ld32(a + 96, r3);
                    tmem_ld_wait();
                    tmem_reg_fence(r0);
                    tmem_reg_fence(r1);
                    tmem_reg_fence(r2);
                    tmem_reg_fence(r3);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        s[c] = __uint_as_float(r0[c]);
                        s[32 + c] = __uint_as_float(r1[c]);
                        s[64 + c] = __uint_as_float(r2[c]);
                        s[96 + c] = __uint_as_float(r3[c]);
                    }
                }
                const int kv0 = j * BN;
                if (kv0 + BN > lim) {  // masking step: keys at or beyond the row's limit
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        if (kv0 + c >= lim) s[c] = NEG_INF;
                }
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = s[i];
#pragma unroll
                for (int c = 8; c < BN; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
                const float rowmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                           fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                const float m_new = rowmax * p.scale_log2;
                float alpha = 1.f;
                bool resc = false;
                if (j == 0) {
                    m_ref = (m_new == NEG_INF) ? 0.f : m_new;
                    l = 0.f;
                    lr = 0.f;
                } else if (m_new > m_ref + p.tau) {
                    alpha = ex2_approx(m_ref - m_new);
                    l *= alpha;
                    lr *= alpha;
                    m_ref = m_new;
                    resc = true;
                }
                const float neg_m = -m_ref;
                float ls[8], lrs[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) ls[i] = lrs[i] = 0.f;
                uint32_t pk0[32], pk1[32];  // keys [0,64) and [64,128), two bf16 per column
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float p0 = ex2_approx(fmaf(s[c], p.scale_log2, neg_m));
                    const float p1 = ex2_approx(fmaf(s[c + 1], p.scale_log2, neg_m));
                    ls[(c >> 1) & 7] += p0 + p1;
                    pk0[c >> 1] = pack_bf16x2(p0, p1);
                    lrs[(c >> 1) & 7] += bf16x2_lo(pk0[c >> 1]) + bf16x2_hi(pk0[c >> 1]);
                }
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float p0 = ex2_approx(fmaf(s[64 + c], p.scale_log2, neg_m));
                    const float p1 = ex2_approx(fmaf(s[64 + c + 1], p.scale_log2, neg_m));
                    ls[(c >> 1) & 7] += p0 + p1;
                    pk1[c >> 1] = pack_bf16x2(p0, p1);
                    lrs[(c >> 1) & 7] += bf16x2_lo(pk1[c >> 1]) + bf16x2_hi(pk1[c >> 1]);
                }
                l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
                lr += ((lrs[0] + lrs[1]) + (lrs[2] + lrs[3])) + ((lrs[4] + lrs[5]) + (lrs[6] + lrs[7]));
                {
                    const uint32_t a = tmem + lane_off + col_p(buf);
                    tmem_st32(a + 0, pk0);
                    tmem_st32(a + 32, pk1);
                }
                if (__any_sync(0xffffffffu, resc)) {
                    // O holds P_0..P_{g-1} V; wait for the last of those products,
                    // then scale this warp's 32 rows in place.
                    ok = mbar_wait(&bars[C::kBarODone], (g - 1) & 1, abort_flag, p.timeout_ns);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t r[32];
                        const uint32_t a = tmem + lane_off + kColO + ch * 32;
                        tmem_ld32(a, r);
                        tmem_ld_wait();
                        tmem_reg_fence(r);
#pragma unroll
                        for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
                        tmem_st32(a, r);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars[C::kBarPFull + buf]);
            }
            if (ok) {
                ok = mbar_wait(&bars[C::kBarOFinal], tl & 1, abort_flag, p.timeout_ns);
                ok = __all_sync(0xffffffffu, ok);
            }
            if (!ok) {
                // abandon this unit: mark its rows
                if (row_valid) {
                    const float nan = __int_as_float(0x7fc00000);
                    if constexpr (O_BF16) {
                        uint16_t *dst = reinterpret_cast<uint16_t *>(p.o) + row_id * D;
                        for (int i = 0; i < D; ++i) dst[i] = 0x7fc0;
                    } else {
                        float *dst = reinterpret_cast<float *>(p.o) + row_id * D;
                        for (int i = 0; i < D; ++i) dst[i] = nan;
                    }
                    p.lse[row_id] = nan;
                }
                break;
            }
            tc_fence_after();
            const float inv_l = 1.f / lr;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + kColO + ch * 32, r);
                tmem_ld_wait();
                tmem_reg_fence(r);
                if (row_valid) {
                    if constexpr (O_BF16) {
                        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.o) + row_id * D + ch * 32);
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
                        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.o) + row_id * D + ch * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(r[4 * i + 0]) * inv_l, __uint_as_float(r[4 * i + 1]) * inv_l,
                                                 __uint_as_float(r[4 * i + 2]) * inv_l, __uint_as_float(r[4 * i + 3]) * inv_l);
                    }
                }
            }
            if (row_valid) p.lse[row_id] = (m_ref + log2f(l)) * LN2;
            tc_fence_before();
            mbar_arrive(&bars[C::kBarOFree]);
            ++tl;
        }
        if (!ok) record_timeout(p);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
            const uint32_t idesc_pv = idesc_bf16_f32(BM, D, true);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t k_addr = smem_u32(sK);
            const uint32_t v_addr = smem_u32(sV);
            uint32_t g = 0, tl = 0;
            bool ok = true;
            // the one P V product whose issue is deferred behind the next Q K^T
            bool pend = false;
            uint32_t pend_g = 0, pend_tl = 0;
            bool pend_first = false, pend_last = false;

            auto issue_pv = [&](uint32_t pg, uint32_t ptl, bool first, bool last) -> bool {
                const uint32_t stage = pg % C::kStages, round = pg / C::kStages, buf = pg & 1;
                if (!mbar_wait(&bars[C::kBarVFull + stage], round & 1, abort_flag, p.timeout_ns)) return false;
                if (!mbar_wait(&bars[C::kBarPFull + buf], (pg >> 1) & 1, abort_flag, p.timeout_ns)) return false;
                if (first && ptl > 0) {  // previous unit's epilogue must have read O
                    if (!mbar_wait(&bars[C::kBarOFree], (ptl - 1) & 1, abort_flag, p.timeout_ns)) return false;
                }
                tc_fence_after();
                const uint32_t vs = v_addr + stage * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bdesc = sw128_desc(vs + kk * 16 * 128, C::kChunkBytes, 1024);
                    mma_ts(tmem + kColO, tmem + col_p(buf) + kk * 8, bdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
                }
                tc_commit(&bars[C::kBarKVEmpty + stage]);
                tc_commit(&bars[C::kBarODone]);
                if (last) tc_commit(&bars[C::kBarOFinal]);
                return true;
            };

            for (int k = 0; ok; ++k) {
                const int t = unit_index(k);
                if (t >= p.n_tiles) break;
                const TileCoord tc = decode_tile(p, t);
                if (tc.n_kv == 0) continue;
                if (!mbar_wait(&bars[C::kBarQFull], tl & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                for (int j = 0; j < tc.n_kv; ++j, ++g) {
                    const uint32_t stage = g % C::kStages, round = g / C::kStages, buf = g & 1;
                    if (!mbar_wait(&bars[C::kBarKFull + stage], round & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t ks = k_addr + stage * C::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                        mma_ss(tmem + col_s(buf), sw128_desc(q_addr + off, 16, 1024), sw128_desc(ks + off, 16, 1024),
                               idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&bars[C::kBarSFull + buf]);
                    if (j == tc.n_kv - 1) tc_commit(&bars[C::kBarQEmpty]);
                    if (pend && !issue_pv(pend_g, pend_tl, pend_first, pend_last)) { ok = false; break; }
                    pend = true;
                    pend_g = g;
                    pend_tl = tl;
                    pend_first = (j == 0);
                    pend_last = (j == tc.n_kv - 1);
                }
                ++tl;
            }
            if (ok && pend) ok = issue_pv(pend_g, pend_tl, pend_first, pend_last);
            if (!ok) record_timeout(p);
            // drain: no MMA may still be running when TMEM is released
            tc_commit(&bars[C::kBarDrain]);
            mbar_wait_drain(&bars[C::kBarDrain], 0, p.timeout_ns);
        }
    } else if (warp == kLoadWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&p.tm_q);
            prefetch_tensormap(&p.tm_k);
            prefetch_tensormap(&p.tm_v);
            uint32_t g = 0, tl = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int t = unit_index(k);
                if (t >= p.n_tiles) break;
                const TileCoord tc = decode_tile(p, t);
                if (tc.n_kv == 0) continue;
                if (tl > 0 && !mbar_wait(&bars[C::kBarQEmpty], (tl - 1) & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
                mbar_arrive_expect_tx(&bars[C::kBarQFull], C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(sQ + c * C::kChunkBytes, &p.tm_q, &bars[C::kBarQFull], c * 64, tc.qt * BM, tc.bh);
                ++tl;
                for (int j = 0; j < tc.n_kv; ++j, ++g) {
                    const uint32_t stage = g % C::kStages, round = g / C::kStages;
                    if (round > 0 && !mbar_wait(&bars[C::kBarKVEmpty + stage], (round - 1) & 1, abort_flag, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *ks = sK + stage * C::kTileBytes;
                    uint8_t *vs = sV + stage * C::kTileBytes;
                    mbar_arrive_expect_tx(&bars[C::kBarKFull + stage], C::kTileBytes);
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(ks + c * C::kChunkBytes, &p.tm_k, &bars[C::kBarKFull + stage], c * 64, j * BN, tc.bh);
                    mbar_arrive_expect_tx(&bars[C::kBarVFull + stage], C::kTileBytes);
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(vs + c * C::kChunkBytes, &p.tm_v, &bars[C::kBarVFull + stage], c * 64, j * BN, tc.bh);
                }
            }
            if (!ok) record_timeout(p);
            // drain: every copy this thread issued has landed before the CTA may exit
            if (tl > 0) mbar_wait_drain(&bars[C::kBarQFull], (tl - 1) & 1, p.timeout_ns);
            const uint32_t n_last = g < (uint32_t)C::kStages ? g : (uint32_t)C::kStages;
            for (uint32_t i = 0; i < n_last; ++i) {
                const uint32_t gg = g - 1 - i;
                const uint32_t stage = gg % C::kStages, round = gg / C::kStages;
                mbar_wait_drain(&bars[C::kBarKFull + stage], round & 1, p.timeout_ns);
                mbar_wait_drain(&bars[C::kBarVFull + stage], round & 1, p.timeout_ns);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace fa

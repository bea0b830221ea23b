// fa_fwd_d256_kernel.cuh -- the fused exact attention forward for head
// dimension 256 on sm_100a.
//
// The same computation as fa_fwd_sm100_kernel (page "FlashAttention (ES)",
// sections "Tiling y procesamiento por bloques", "Calculo de Softmax en
// linea" and "Fusion de operaciones en un unico kernel de CUDA"; the
// FlashAttention-2 notes of the same page list head dimensions up to 256),
// laid out for d = 256.  One 128-row query tile's fp32 output already fills
// half of the 512 TMEM columns, so a work unit is one 128-row query tile of
// one (b, h) (and one key split), and the other half of TMEM holds two score
// buffers:
//     S_0 [0,128), S_1 [128,256), O [256,512)
// so that the scores of key tile j+1 are computed while the softmax works on
// tile j.  P_j (bf16) is written over the first 64 columns of its S buffer.
//
// Every operand is handled as 128 x 128 bf16 half tiles (32 KB; two 64-column
// blocks in the 128-byte-swizzle layout): Q = [Q_lo | Q_hi] along d stays in
// shared memory for the unit; K_j and V_j stream as [lo | hi] halves through
// one ring of five half-tile slots, loaded in the order the tensor core uses
// them.  Products (each one tcgen05.mma group of N = 128):
//     S_b  = Q_lo K_lo^T + Q_hi K_hi^T               (b = tile index mod 2)
//     O_lo += P V_lo,  O_hi += P V_hi
// Issue order in a unit with n key tiles:
//     QK_0, QK_1, PV_0, QK_2, PV_1, QK_3, ..., PV_{n-1}
// tcgen05.mma operations of one thread execute in issue order, so QK_{j+2}
// overwrites P_j only after PV_j has read it, and the commit that signals
// "S_j ready" covers PV_{j-2}.  PV_{j-1} may still run while the softmax of
// tile j does, so when the reference maximum moves the softmax first waits for
// PV_{j-1} (one o_done barrier per parity of the product index keeps that
// wait exact) before it rescales O.
//
// Warps: 0-3 softmax (thread t owns row t of the tile), 4 MMA issuer (one
// thread), 5 TMA producer (one thread).  192 threads, up to 255 registers each.
//
// The layout is written for any d that is a multiple of 128 up to 256 (Cfg1<D>:
// D / 128 half tiles per operand, a ring as deep as shared memory allows).
// Only d = 256 is instantiated: at d = 128 this design (six ring slots, one
// query tile) measured about 11% slower on a B200 than the two-query-tile
// ping-pong kernel of fa_fwd_kernel.cuh, with bit-identical outputs.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {
namespace d256 {

constexpr int kUnitRows = BM;                 // one query tile per work unit
constexpr int kHalfBytes = BM * 128 * 2;      // a 128 x 128 bf16 half tile
constexpr int kBlockBytes = BM * 128;         // one 64-column (128-byte) block of it
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr int kThreads = 192;
constexpr uint32_t kColO = 256;

// Layout for head dimension D (128 or 256): Q is D / 128 half tiles, every
// K_j and V_j D / 128 half tiles through the ring, whose depth is what the
// rest of shared memory holds.
template <int D>
struct Cfg1 {
    static_assert(D == 128 || D == 256, "one-tile kernel: d = 128 or 256");
    static constexpr int kHalves = D / 128;
    static constexpr int kOffQ = 0;
    static constexpr int kOffRing = kOffQ + kHalves * kHalfBytes;
    static constexpr int kSlots = (232448 - 1024 - 512 - kOffRing) / kHalfBytes;  // 5 for d = 256, 6 for 128
    static constexpr int kOffBar = kOffRing + kSlots * kHalfBytes;
    static constexpr int kBarQFull = 0;
    static constexpr int kBarQEmpty = 1;
    static constexpr int kBarFull = 2;                     // [kSlots]
    static constexpr int kBarEmpty = kBarFull + kSlots;    // [kSlots]
    static constexpr int kBarSFull = kBarEmpty + kSlots;   // [2] per score buffer
    static constexpr int kBarPFull = kBarSFull + 2;        // [2] per score buffer (128 arrivals)
    static constexpr int kBarODone = kBarPFull + 2;        // [2] per parity of the P V product index
    static constexpr int kBarOFree = kBarODone + 2;        // 128 arrivals
    static constexpr int kBarUnitFull = kBarOFree + 1;               // [kUnitQueue]
    static constexpr int kBarUnitFree = kBarUnitFull + kUnitQueue;   // [kUnitQueue], softmax threads + MMA thread
    static constexpr int kBarDrain = kBarUnitFree + kUnitQueue;
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 4;
    static constexpr int kOffClaimed = kOffAbort + 4;  // scheduler slot claimed (int)
    static constexpr int kOffUnitIds = kOffClaimed + 4;
    static constexpr int kSmemUsed = kOffUnitIds + 16 * kUnitQueue;
    static constexpr int kSmemBytes = kSmemUsed + 1024;  // + slack to align the base to 1024 bytes
    static_assert(kHalfBytes % 1024 == 0 && kBlockBytes % 1024 == 0, "1024-byte alignment of swizzled tiles");
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
    static_assert(2 * kSmemBytes > 233472, "one CTA per SM: TMEM is allocated whole");
};

// Unit t -> (b, h, query tile, split) and the key tiles [lo, lo + n) that some
// row of the tile may attend to: as decode_unit (same banded order) with one
// query tile per unit (p.n_blocks = ceil(N / 128)).
__device__ __forceinline__ UnitCoord decode_unit1(const FwdParams &p, int t) {
    UnitCoord u;
    u.split = t % p.n_splits;
    band_decode(p, t / p.n_splits, u.bh, u.blk);
    u.b = u.bh / p.H;
    u.bh_kv = u.b * p.H_kv + (u.bh - u.b * p.H) / p.group;
    u.lo = u.split * p.split_tiles;
    int e = p.Nk;
    if (p.k_len) e = min(max(__ldg(p.k_len + u.b), 0), p.Nk);
    const int first = u.blk * kUnitRows;
    if (p.causal) e = max(0, min(e, first + BM + (p.Nk - p.N)));
    const int tiles = (first < p.N) ? (e + BN - 1) / BN : 0;
    u.n[0] = max(0, min(tiles, u.lo + p.split_tiles) - u.lo);
    u.n[1] = 0;
    u.nmax = u.n[0];
    return u;
}

// Waits, in order, for the completion of every P V product up to index
// `upto` (global count over the CTA's units) not yet waited for.  Product i
// completes phase i / 2 of o_done[i % 2]; at most one phase per barrier is
// ever outstanding (see the issue order above), so the parity is exact.
template <int D>
__device__ __forceinline__ bool wait_pv_upto(uint64_t *bars, uint32_t &waited, long long upto,
                                             volatile int *abort_flag, uint64_t to) {
    using C = Cfg1<D>;
    while ((long long)waited <= upto) {
        if (!mbar_wait(&bars[C::kBarODone + (waited & 1)], (waited >> 1) & 1, abort_flag, to)) return false;
        ++waited;
    }
    return true;
}

// ------------------------------------------------------------------ softmax
template <int D, bool O_BF16>
__device__ __forceinline__ bool softmax_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                             const UnitQueue &uq, uint32_t tmem, int warp, int lane) {
    using C = Cfg1<D>;
    const int row_in_tile = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float NEG_INF = __int_as_float(0xff800000);
    const uint32_t t_o = tmem + lane_off + kColO;
    const uint64_t to = p.timeout_ns;
    uint32_t gs = 0;      // score tiles consumed (global): buffer gs % 2
    uint32_t waited = 0;  // P V products whose completion was waited for
    uint32_t tl = 0;      // units with work (o_free phase)
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = p.dynamic ? unit_pop(uq, k, abort_flag, to, ok) : unit_static(p, k);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || t < 0) break;
        const UnitCoord u = decode_unit1(p, t);
        const int row = u.blk * kUnitRows + row_in_tile;
        const bool row_valid = row < p.N;
        const size_t row_id = ((size_t)u.split * p.B * p.H + u.bh) * p.N + row;
        const int n = u.n[0];
        if (n == 0) {  // no allowed key for these rows: O = 0, lse = -inf
            if (row_valid) fill_row<D, O_BF16>(p.o, p.lse, row_id, false, NEG_INF);
            continue;
        }
        int lim = p.Nk;  // keys [0, lim) are allowed for this row
        if (p.k_len) lim = min(max(__ldg(p.k_len + u.b), 0), p.Nk);
        if (p.causal) lim = min(lim, row + 1 + (p.Nk - p.N));

        RowState st;
        for (int j = 0; j < n; ++j, ++gs) {
            const uint32_t buf = gs & 1;
            const uint32_t t_s = tmem + lane_off + buf * 128u;
            ok = mbar_wait(&bars[C::kBarSFull + buf], (gs >> 1) & 1, abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();

            float s[BN];
            uint32_t pk0[32], pk1[32];
            float2 ls = make_float2(0.f, 0.f);
            load_score_row(t_s, s);
            const float m_new = masked_row_max(s, (u.lo + j) * BN, lim, p.scale_log2);
            float alpha;
            const bool resc = update_reference(st, j, m_new, p.tau, alpha);
            // the products before this tile's predecessor are complete (the
            // commit behind S ready covers them): consume their phases
            const bool any_resc = __any_sync(0xffffffffu, resc);
            ok = wait_pv_upto<D>(bars, waited, (long long)gs - (any_resc ? 1 : 2), abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (any_resc) {
                tc_fence_after();
                rescale_o_row<D>(t_o, alpha);
            }
            exp_half_p<0>(s, p.scale_log2, -st.m_ref, pk0, ls);
            tmem_st32(t_s + 0, pk0);
            exp_half_p<1>(s, p.scale_log2, -st.m_ref, pk1, ls);
            tmem_st32(t_s + 32, pk1);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[C::kBarPFull + buf]);
            st.l += ls.x + ls.y;
            st.lr += rounded_sum(pk0, pk1);
        }
        if (ok) {
            ok = wait_pv_upto<D>(bars, waited, (long long)gs - 1, abort_flag, to);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (!ok) {
            if (row_valid) fill_row<D, O_BF16>(p.o, p.lse, row_id, true, __int_as_float(0x7fc00000));
            break;
        }
        tc_fence_after();
        write_row<D, O_BF16>(t_o, p.o, p.lse, row_id, row_valid, st.lr, 1.f, st.m_ref + log2f(st.l));
        tc_fence_before();
        mbar_arrive(&bars[C::kBarOFree]);
        ++tl;
    }
    return ok;
}

// ------------------------------------------------------------------ MMA issuer
template <int D>
__device__ __forceinline__ bool mma_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                         const UnitQueue &uq, uint32_t tmem, uint32_t q_addr, uint32_t ring_addr) {
    using C = Cfg1<D>;
    const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
    const uint32_t idesc_pv = idesc_bf16_f32(BM, 128, true);
    const uint64_t q_desc = sw128_desc(q_addr, 16, 1024);
    const uint64_t k_desc = sw128_desc(ring_addr, 16, 1024);
    const uint64_t v_desc = sw128_desc(ring_addr, kBlockBytes, 1024);
    const uint64_t to = p.timeout_ns;
    uint32_t tq = 0;   // non-empty units (q_full phase)
    uint32_t g = 0;    // ring position
    uint32_t gs = 0;   // score tiles issued: buffer gs % 2
    uint32_t gpv = 0;  // P V products issued: P buffer and o_done barrier gpv % 2
    uint32_t tl = 0;   // units with work (o_free phase)

    auto take = [&](uint32_t &slot) -> bool {
        slot = g % C::kSlots;
        const bool r = mbar_wait(&bars[C::kBarFull + slot], (g / C::kSlots) & 1, abort_flag, to);
        ++g;
        return r;
    };
    // S_b = sum over the halves h of Q_h K_h^T (K_j's halves in consecutive ring slots)
    auto qk = [&]() -> bool {
        uint32_t sl[C::kHalves];
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
            if (!take(sl[h])) return false;
        tc_fence_after();
        const uint32_t d = tmem + (gs & 1) * 128u;
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
            mma_ss_k128(d, q_desc + ((h * kHalfBytes) >> 4), k_desc + ((sl[h] * kHalfBytes) >> 4), idesc_qk,
                        h > 0 ? 1u : 0u);
        tc_commit(&bars[C::kBarSFull + (gs & 1)]);
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) tc_commit(&bars[C::kBarEmpty + sl[h]]);
        ++gs;
        return true;
    };
    auto pv = [&](bool first) -> bool {
        const uint32_t buf = gpv & 1;
        if (!mbar_wait(&bars[C::kBarPFull + buf], (gpv >> 1) & 1, abort_flag, to)) return false;
        if (first && tl > 0 && !mbar_wait(&bars[C::kBarOFree], (tl - 1) & 1, abort_flag, to)) return false;
        uint32_t sl[C::kHalves];
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
            if (!take(sl[h])) return false;
        tc_fence_after();
        const uint32_t a = tmem + buf * 128u;
        // O_h (+)= P V_h: columns [128 h, 128 h + 128) of O
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
            mma_ts_k128(tmem + kColO + 128u * h, a, v_desc + ((sl[h] * kHalfBytes) >> 4), idesc_pv,
                        first ? 0u : 1u);
        tc_commit(&bars[C::kBarODone + buf]);
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) tc_commit(&bars[C::kBarEmpty + sl[h]]);
        ++gpv;
        return true;
    };

    bool ok = true;
    for (int k = 0; ok; ++k) {
        int n = 0;  // dynamic: the key-tile count comes with the id (the TMA warp decoded the unit)
        const int t = p.dynamic ? unit_pop(uq, k, abort_flag, to, ok, &n) : unit_static(p, k);
        if (!ok || t < 0) break;
        if (!p.dynamic) n = decode_unit1(p, t).n[0];
        if (n == 0) continue;
        if (!mbar_wait(&bars[C::kBarQFull], tq & 1, abort_flag, to)) { ok = false; break; }
        ++tq;
        tc_fence_after();
        int jq = 0;  // score tiles of this unit issued
        auto qk_next = [&]() -> bool {
            if (!qk()) return false;
            if (++jq == n) tc_commit(&bars[C::kBarQEmpty]);  // Q no longer read in this unit
            return true;
        };
        if (!qk_next()) { ok = false; break; }
        if (n > 1 && !qk_next()) { ok = false; break; }
        for (int j = 0; j < n; ++j) {
            if (!pv(j == 0)) { ok = false; break; }
            if (j + 2 < n && !qk_next()) { ok = false; break; }
        }
        ++tl;
    }
    return ok;
}

// ------------------------------------------------------------------ TMA producer
template <int D>
__device__ __forceinline__ void load_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                          const UnitQueue &uq, uint8_t *sQ, uint8_t *ring) {
    using C = Cfg1<D>;
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
    const uint64_t to = p.timeout_ns;
    uint32_t tq = 0, g = 0;
    // test only: the ring load this CTA never issues (its ring position), or none
    const uint32_t drop = (blockIdx.x == 0 && p.drop_load > 0) ? (uint32_t)(p.drop_load - 1) : 0xFFFFFFFFu;
    bool ok = true;
    // key tile `kt` of K or V as D / 128 half tiles (d columns [128 h, 128 h + 128))
    auto load_tile = [&](const CUtensorMap *map, int kt, int bh_kv) -> bool {
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
            const uint32_t slot = g % C::kSlots, round = g / C::kSlots;
            if (round > 0 && !mbar_wait(&bars[C::kBarEmpty + slot], (round - 1) & 1, abort_flag, to)) return false;
            if (g != drop) {
                mbar_arrive_expect_tx(&bars[C::kBarFull + slot], kHalfBytes);
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    tma_load_3d(ring + slot * kHalfBytes + c * kBlockBytes, map, &bars[C::kBarFull + slot],
                                h * 128 + c * 64, kt * BN, bh_kv);
            }
            ++g;
        }
        return true;
    };
    for (int k = 0; ok; ++k) {
        const int t = p.dynamic ? unit_take(p, uq, k, abort_flag, to, ok) : unit_static(p, k);
        if (!ok) break;
        if (t < 0) {
            if (p.dynamic) unit_publish(uq, k, -1, 0, 0);
            break;
        }
        const UnitCoord u = decode_unit1(p, t);
        if (p.dynamic) unit_publish(uq, k, t, u.n[0], 0);
        const int n = u.n[0];
        if (n == 0) continue;
        if (tq > 0 && !mbar_wait(&bars[C::kBarQEmpty], (tq - 1) & 1, abort_flag, to)) {
            ok = false;
            break;
        }
        mbar_arrive_expect_tx(&bars[C::kBarQFull], C::kHalves * kHalfBytes);
#pragma unroll
        for (int c = 0; c < 2 * C::kHalves; ++c)
            tma_load_3d(sQ + c * kBlockBytes, &p.tm_q, &bars[C::kBarQFull], c * 64, u.blk * kUnitRows, u.bh);
        ++tq;
        // the order the MMA issuer takes them: K_0, K_1, V_0, K_2, V_1, ..., V_{n-1}
        if (!load_tile(&p.tm_k, u.lo, u.bh_kv)) { ok = false; break; }
        if (n > 1 && !load_tile(&p.tm_k, u.lo + 1, u.bh_kv)) { ok = false; break; }
        for (int j = 0; j < n && ok; ++j) {
            if (!load_tile(&p.tm_v, u.lo + j, u.bh_kv)) ok = false;
            else if (j + 2 < n && !load_tile(&p.tm_k, u.lo + j + 2, u.bh_kv)) ok = false;
        }
    }
    if (!ok) record_timeout(p);
    // drain: every copy this thread issued has landed before the CTA may exit
    if (tq > 0) mbar_wait_drain(&bars[C::kBarQFull], (tq - 1) & 1);
    const uint32_t nr = g < (uint32_t)C::kSlots ? g : (uint32_t)C::kSlots;
    for (uint32_t i = 0; i < nr; ++i) {
        const uint32_t gi = g - 1 - i;
        if (gi != drop) mbar_wait_drain(&bars[C::kBarFull + gi % C::kSlots], (gi / C::kSlots) & 1);
    }
}

}  // namespace d256

template <int D, bool O_BF16>
__global__ void __launch_bounds__(d256::kThreads, 1) fa_fwd_onetile_kernel(const __grid_constant__ FwdParams p) {
    using namespace d256;
    using C = Cfg1<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *ring = smem + C::kOffRing;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    volatile int *claimed = reinterpret_cast<volatile int *>(smem + C::kOffClaimed);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const UnitQueue uq{reinterpret_cast<volatile int *>(smem + C::kOffUnitIds), &bars[C::kBarUnitFull], &bars[C::kBarUnitFree]};
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            const bool per_row = (i >= C::kBarPFull && i < C::kBarPFull + 2) || i == C::kBarOFree;
            const bool unit_free = i >= C::kBarUnitFree && i < C::kBarUnitFree + kUnitQueue;
            mbar_init(&bars[i], unit_free ? 129u : (per_row ? 128u : 1u));
        }
        *abort_flag = 0;
        *claimed = p.dynamic ? (sched_claim(p.sched, p.timeout_ns) ? 1 : 0) : 1;
        fence_mbar_init();
    }
    if (warp == d256::kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (!*claimed) {  // the scheduler slot stayed in use by another launch: no work, report it
        if (threadIdx.x == 0) record_status(p.status, kStatusSchedBusy);
        if (warp == d256::kMmaWarp) tmem_dealloc(tmem, kTmemCols);
        return;
    }

    if (warp < d256::kSoftmaxWarps) {
        if (!d256::softmax_role<D, O_BF16>(p, bars, abort_flag, uq, tmem, warp, lane)) record_timeout(p);
    } else if (warp == d256::kMmaWarp) {
        if (lane == 0) {
            if (!d256::mma_role<D>(p, bars, abort_flag, uq, tmem, smem_u32(sQ), smem_u32(ring))) record_timeout(p);
            tc_commit(&bars[C::kBarDrain]);
            mbar_wait_drain(&bars[C::kBarDrain], 0);
        }
    } else if (warp == d256::kLoadWarp) {
        if (lane == 0) d256::load_role<D>(p, bars, abort_flag, uq, sQ, ring);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == d256::kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && p.dynamic) sched_release(p.sched);
}

}  // namespace fa

// fa_fwd_pair_kernel.cuh -- the fused attention forward on CTA pairs (d = 128,
// bf16 operands).
//
// The computation is that of fa_fwd_kernel.cuh (page "FlashAttention (ES)":
// the Attention equation of section "El problema de la atencion estandar",
// computed with the tiling, online softmax and single fused kernel of section
// "Innovaciones clave de FlashAttention"); what differs is how it maps onto
// Blackwell:
//
//   * a cluster of two CTAs on two SMs runs each product as one tcgen05
//     cta_group::2 product of M = 256 query rows: CTA r holds its 128 query
//     rows of the 256-row work unit, keys [64 r, 64 r + 64) of each K tile
//     and value columns [64 r, 64 r + 64) of each V tile, so each SM loads and
//     reads half of every K and V tile (the tensor cores exchange the halves);
//   * per CTA, TMEM holds two score buffers S_0, S_1 (consecutive key tiles),
//     the output accumulator O and the probabilities P in columns of their
//     own: Q K_{j+2}^T may be issued as soon as the softmax has read S(j),
//     and the softmax of tile j+1 never waits for the P V of tile j;
//   * each query row is shared by two softmax warps on one SM sub-partition,
//     one per 64-key half of the tile, which exchange their row maxima (and,
//     at the end of a unit, their sums) through shared memory; each warp
//     reads key tile j+1 and posts its half maximum before it computes the
//     exponentials of tile j, so the exchange overlaps them.
//
// TMEM (each CTA, 512 columns allocated as a pair): S_0 [0,128), S_1
// [128,256), O [256,384), P [384,448) (bf16 pairs).  Warps 0-7 softmax (warp
// w: TMEM lanes 32 (w % 4) ..., key half w / 4), warp 8 issues every product
// (CTA 0 only), warp 9 issues the TMA loads of this CTA's halves, warps 10-11
// idle.  Work units (b, h, 256-row block, key split) are taken by the pairs in
// a static snake order.  Every wait is bounded in wall time; on time-out the
// CTA raises its abort flag, records FA_ERR_DEVICE_TIMEOUT, marks the rows of
// its unit NaN and leaves (its partner's waits then run out as well).
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {
namespace pair {

constexpr int kThreads = 384;
constexpr int kSoftmaxWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S_0 [0,128), S_1 [128,256)
constexpr uint32_t kColO = 256;  // O [256,384)
constexpr uint32_t kColP = 384;  // P [384,448): 128 keys as bf16 pairs
constexpr int kD = 128;

struct PCfg {
    static constexpr int kQBytes = BM * kD * 2;     // this CTA's 128 query rows: two 16 KB column blocks
    static constexpr int kKBytes = 64 * kD * 2;     // 64 keys x 128: two 8 KB column blocks
    static constexpr int kVBytes = BN * 64 * 2;     // 128 keys x 64 value columns: one 16 KB block
    static constexpr int kKStages = 5;
    static constexpr int kVStages = 5;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kKStages * kKBytes;
    static constexpr int kOffMax = kOffV + kVStages * kVBytes;  // [2 tile parity][2 halves][128] float
    static constexpr int kOffSum = kOffMax + 2 * 2 * BM * 4;    // [2 halves][2 (l, lr)][128] float
    static constexpr int kOffBar = kOffSum + 2 * 2 * BM * 4;
    static constexpr int kBarQFull = 0;                         // CTA 0: both Q tiles landed
    static constexpr int kBarQEmpty = 1;                        // both: the unit's last Q K^T done
    static constexpr int kBarKFull = 2;                         // [kKStages] CTA 0
    static constexpr int kBarKEmpty = kBarKFull + kKStages;     // [kKStages] both
    static constexpr int kBarVFull = kBarKEmpty + kKStages;     // [kVStages] CTA 0
    static constexpr int kBarVEmpty = kBarVFull + kVStages;     // [kVStages] both
    static constexpr int kBarSFull = kBarVEmpty + kVStages;     // [2] both: S_b written
    static constexpr int kBarSFree = kBarSFull + 2;             // [2] CTA 0: S_b read by all 16 softmax warps
    static constexpr int kBarPFull = kBarSFree + 2;             // CTA 0: P of all 16 softmax warps in TMEM
    static constexpr int kBarPvDone = kBarPFull + 1;            // both: P V complete
    static constexpr int kBarOFree = kBarPvDone + 1;            // CTA 0: O read by all 16 softmax warps
    static constexpr int kBarXMax = kBarOFree + 1;              // [4] per sub-partition: both halves' maxima
    static constexpr int kBarXSum = kBarXMax + 4;               // [4] per sub-partition: both halves' sums
    static constexpr int kBarDrain = kBarXSum + 4;
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 4;
    static constexpr int kSmemUsed = kOffAbort + 4;
    static constexpr int kSmemBytes = kSmemUsed + 1024;  // + slack to align the base to 1024 bytes
    static_assert(kQBytes % 1024 == 0 && kKBytes % 1024 == 0 && kVBytes % 1024 == 0, "1024-byte tile alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
    static_assert(2 * kSmemBytes > 233472, "one CTA per SM: TMEM is allocated whole");
};

// Unit k of this pair: the snake order of unit_index over pairs.
__device__ __forceinline__ int pair_unit(const FwdParams &p, int k) {
    const int G = gridDim.x >> 1, c = blockIdx.x >> 1;
    const int t = k * G + ((k & 1) ? (G - 1 - c) : c);
    return t < p.n_units ? t : -1;
}

// ------------------------------------------------------------------ softmax
template <bool O_BF16>
__device__ __forceinline__ bool softmax_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                             uint8_t *smem, uint32_t tmem, uint32_t rank, int warp, int lane) {
    using C = PCfg;
    const int wq = warp & 3, h = warp >> 2;  // sub-partition (row group) and key half
    const int r = wq * 32 + lane;            // row of this CTA's tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t t_o = tmem + lane_off + kColO + 64u * h;
    const uint32_t t_p = tmem + lane_off + kColP + 32u * h;
    float *xmax = reinterpret_cast<float *>(smem + C::kOffMax);
    float *xsum = reinterpret_cast<float *>(smem + C::kOffSum);
    const uint32_t s_free0[2] = {cluster_addr(&bars[C::kBarSFree], 0), cluster_addr(&bars[C::kBarSFree + 1], 0)};
    const uint32_t p_full0 = cluster_addr(&bars[C::kBarPFull], 0);
    const uint32_t o_free0 = cluster_addr(&bars[C::kBarOFree], 0);
    const uint64_t to = p.timeout_ns;
    uint32_t gs = 0;        // score tiles consumed (S buffer gs % 2)
    uint32_t pv_known = 0;  // P V products known to be complete
    uint32_t gu = 0;        // units with work (sum exchange phase)
    auto ensure_pv = [&](uint32_t n) -> bool {  // the first n P V products are complete
        if (pv_known >= n) return true;
        const bool w = mbar_wait(&bars[C::kBarPvDone], (n - 1) & 1, abort_flag, to);
        pv_known = n;
        return __all_sync(0xffffffffu, w);
    };
    // both warps of the sub-partition have written their half's value for this round
    auto exchange = [&](uint64_t *bar, uint32_t phase) -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
        return __all_sync(0xffffffffu, mbar_wait(bar, phase & 1, abort_flag, to));
    };
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = pair_unit(p, k);
        if (t < 0) break;
        const UnitCoord u = decode_unit(p, t, nullptr);
        const int row = u.blk * kUnitRows + (int)rank * BM + r;
        const bool row_valid = row < p.N;
        const size_t row_id = ((size_t)u.split * p.B * p.H + u.bh) * p.N + row;
        if (u.nmax == 0) {  // no allowed key for the unit's rows
            if (row_valid && h == 0) fill_row<kD, O_BF16>(p.o, p.lse, row_id, false, __int_as_float(0xff800000));
            continue;
        }
        int lim = p.Nk;  // keys [0, lim) are allowed for this row
        if (p.k_len) lim = min(max(__ldg(p.k_len + u.b), 0), p.Nk);
        if (p.causal) lim = min(lim, row + 1 + (p.Nk - p.N));
        RowState st;
        // S half-row of key tile j (score tile g overall) into s, its S buffer
        // released, masked, and this half's maximum posted to the partner warp
        auto read_half = [&](uint32_t g, int j, float (&s)[64]) -> bool {
            const uint32_t buf = g & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[C::kBarSFull + buf], (g >> 1) & 1, abort_flag, to)))
                return false;
            tc_fence_after();
            const uint32_t t_s = tmem + lane_off + kColS + 128u * buf + 64u * h;
            tmem_ld32f(t_s, s);
            tmem_ld32f(t_s + 32, s + 32);
            tmem_ld_wait();
            tmem_reg_fence_f<64>(s);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(s_free0[buf]);  // S_buf may take the key tile after next
            const int kv0 = (u.lo + j) * BN + 64 * h;  // masking step on this half's 64 keys
            if (kv0 + 64 > lim) mask_scores<0>(s, kv0, lim);
            xmax[(g & 1) * 2 * BM + h * BM + r] = max64(s) * p.scale_log2;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[C::kBarXMax + wq]);
            return true;
        };
        // key tile j from `cur`: the row maximum of both halves, the reference
        // update, the next tile read into `nxt` (its maximum travels to the
        // partner while this tile's exponentials run), then P and the sums
        auto tile = [&](float (&cur)[64], float (&nxt)[64], int j) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[C::kBarXMax + wq], gs & 1, abort_flag, to))) return false;
            const float m_new = fmaxf(xmax[(gs & 1) * 2 * BM + r], xmax[(gs & 1) * 2 * BM + BM + r]);
            float alpha;
            const bool resc = update_reference(st, j, m_new, p.tau, alpha);
            if (j + 1 < u.nmax && !read_half(gs + 1, j + 1, nxt)) return false;
            if (__any_sync(0xffffffffu, resc)) {  // O (this half's 64 columns) *= alpha once P V(j-1) is done
                if (!ensure_pv(gs)) return false;
                tc_fence_after();
                rescale_o_row<64>(t_o, alpha);
            }
            uint32_t pk[32];
            float2 ls = make_float2(0.f, 0.f);
            exp_half_p<0>(cur, p.scale_log2, -st.m_ref, pk, ls);
            if (!ensure_pv(gs)) return false;  // P V(j-1) has read P
            tc_fence_after();
            tmem_st32(t_p, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(p_full0);
            st.l += ls.x + ls.y;
            float b4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 32; ++i) b4[i & 3] = add_bf16x2_to(b4[i & 3], pk[i]);
            st.lr += (b4[0] + b4[1]) + (b4[2] + b4[3]);
            ++gs;
            return true;
        };
        float sa[64], sb[64];  // two score buffers in registers, alternating by key tile
        ok = read_half(gs, 0, sa);
        for (int j = 0; j < u.nmax && ok; j += 2) {
            ok = tile(sa, sb, j);
            if (ok && j + 1 < u.nmax) ok = tile(sb, sa, j + 1);
        }
        if (ok) ok = ensure_pv(gs);  // every product of this unit
        if (ok) {  // both halves' sums, added in the same order by both
            xsum[h * 2 * BM + r] = st.l;
            xsum[h * 2 * BM + BM + r] = st.lr;
            ok = exchange(&bars[C::kBarXSum + wq], gu);
        }
        if (!ok) {
            if (row_valid && h == 0) fill_row<kD, O_BF16>(p.o, p.lse, row_id, true, __int_as_float(0x7fc00000));
            break;
        }
        const float l = xsum[r] + xsum[2 * BM + r];
        const float lr = xsum[BM + r] + xsum[2 * BM + BM + r];
        ++gu;
        tc_fence_after();
        // this half's 64 output columns; lse from the first half
        const bool empty = !(lr > 0.f);
        const float inv_l = empty ? 0.f : 1.f / lr;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            uint32_t v[32];
            tmem_ld32(t_o + ch * 32, v);
            tmem_ld_wait();
            tmem_reg_fence(v);
            if (row_valid) store_row_chunk<kD, O_BF16>(p.o, row_id, 2 * h + ch, v, inv_l);
        }
        if (row_valid && h == 0)
            p.lse[row_id] = empty ? __int_as_float(0xff800000) : (st.m_ref + log2f(l)) * 0.69314718055994530942f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(o_free0);
    }
    return ok;
}

// ------------------------------------------------------------------ MMA issuer (CTA 0)
__device__ __forceinline__ bool mma_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag, uint32_t tmem,
                                         uint32_t q_addr, uint32_t k_addr, uint32_t v_addr) {
    using C = PCfg;
    const uint32_t idesc_qk = idesc_bf16_f32(2 * BM, BN, false);
    const uint32_t idesc_pv = idesc_bf16_f32(2 * BM, kD, true);
    const uint64_t q_desc = sw128_desc(q_addr, 16, 1024);
    const uint64_t k_desc = sw128_desc(k_addr, 16, 1024);
    const uint64_t v_desc = sw128_desc(v_addr, C::kVBytes, 1024);
    const uint64_t to = p.timeout_ns;
    uint32_t tq = 0, tl = 0;    // units with work (q_full, o_free phases)
    uint32_t gk = 0, gv = 0;    // K and V ring positions
    uint32_t gq = 0, gp = 0;    // Q K^T and P V products issued
    // S_{gq % 2} = Q K^T for the next key tile in the K ring
    auto issue_qk = [&]() -> bool {
        const uint32_t kst = gk % C::kKStages, buf = gq & 1;
        if (!mbar_wait(&bars[C::kBarKFull + kst], (gk / C::kKStages) & 1, abort_flag, to)) return false;
        if (gq >= 2 && !mbar_wait(&bars[C::kBarSFree + buf], ((gq - 2) >> 1) & 1, abort_flag, to)) return false;
        tc_fence_after();
        mma2_ss_k128_b8k(tmem + kColS + 128u * buf, q_desc, k_desc + ((kst * C::kKBytes) >> 4), idesc_qk, 0u);
        tc_commit_pair(&bars[C::kBarSFull + buf], 3);
        tc_commit_pair(&bars[C::kBarKEmpty + kst], 3);
        ++gk;
        ++gq;
        return true;
    };
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = pair_unit(p, k);
        if (t < 0) break;
        const UnitCoord u = decode_unit(p, t, nullptr);
        const int n = u.nmax;
        if (n == 0) continue;
        if (!mbar_wait(&bars[C::kBarQFull], tq & 1, abort_flag, to)) { ok = false; break; }
        ++tq;
        tc_fence_after();
        for (int j = 0; j < 2 && j < n && ok; ++j) ok = issue_qk();
        if (!ok) break;
        if (n <= 2) tc_commit_pair(&bars[C::kBarQEmpty], 3);
        for (int j = 0; j < n; ++j) {
            // the scores of key tile j + 2 (their S buffer is free once the
            // softmax has read tile j, which it does while still working on
            // tile j - 1), then O (+)= P V for key tile j
            if (j + 2 < n) {
                if (!(ok = issue_qk())) break;
                if (j + 2 == n - 1) tc_commit_pair(&bars[C::kBarQEmpty], 3);
            }
            if (!mbar_wait(&bars[C::kBarPFull], gp & 1, abort_flag, to)) { ok = false; break; }
            if (j == 0 && tl > 0 && !mbar_wait(&bars[C::kBarOFree], (tl - 1) & 1, abort_flag, to)) { ok = false; break; }
            const uint32_t vst = gv % C::kVStages;
            if (!mbar_wait(&bars[C::kBarVFull + vst], (gv / C::kVStages) & 1, abort_flag, to)) { ok = false; break; }
            tc_fence_after();
            mma2_ts_k128(tmem + kColO, tmem + kColP, v_desc + ((vst * C::kVBytes) >> 4), idesc_pv, j > 0 ? 1u : 0u);
            tc_commit_pair(&bars[C::kBarPvDone], 3);
            tc_commit_pair(&bars[C::kBarVEmpty + vst], 3);
            ++gv;
            ++gp;
        }
        ++tl;
    }
    return ok;
}

// ------------------------------------------------------------------ TMA producer (both CTAs)
// tm_k here is a map with 64-row boxes (this CTA's 64 keys of a tile).
__device__ __forceinline__ void load_role(const FwdParams &p, const CUtensorMap *tm_k64, uint64_t *bars,
                                          volatile int *abort_flag, uint32_t rank, uint8_t *sQ, uint8_t *sK,
                                          uint8_t *sV) {
    using C = PCfg;
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(tm_k64);
    prefetch_tensormap(&p.tm_v);
    const uint64_t to = p.timeout_ns;
    const uint32_t q_full0 = cluster_addr(&bars[C::kBarQFull], 0);
    uint32_t tq = 0, gk = 0, gv = 0;
    // test only: the K load (ring position) the first pair never issues, in
    // both CTAs, so that no copy is ever in flight toward it
    const uint32_t drop = ((blockIdx.x >> 1) == 0 && p.drop_load > 0) ? (uint32_t)(p.drop_load - 1) : 0xFFFFFFFFu;
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = pair_unit(p, k);
        if (t < 0) break;
        const UnitCoord u = decode_unit(p, t, nullptr);
        const int n = u.nmax;
        if (n == 0) continue;
        if (tq > 0 && !mbar_wait(&bars[C::kBarQEmpty], (tq - 1) & 1, abort_flag, to)) { ok = false; break; }
        if (rank == 0) mbar_arrive_expect_tx(&bars[C::kBarQFull], 2 * C::kQBytes);
#pragma unroll
        for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(sQ + c * (BM * 128), &p.tm_q, q_full0, c * 64, u.blk * kUnitRows + (int)rank * BM, u.bh);
        ++tq;
        for (int j = 0; j < n && ok; ++j) {
            const int kt = u.lo + j;
            {
                const uint32_t st = gk % C::kKStages, round = gk / C::kKStages;
                if (round > 0 && !mbar_wait(&bars[C::kBarKEmpty + st], (round - 1) & 1, abort_flag, to)) {
                    ok = false;
                    break;
                }
                if (gk != drop) {
                    if (rank == 0) mbar_arrive_expect_tx(&bars[C::kBarKFull + st], 2 * C::kKBytes);
                    const uint32_t full0 = cluster_addr(&bars[C::kBarKFull + st], 0);
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d_pair(sK + st * C::kKBytes + c * (64 * 128), tm_k64, full0, c * 64,
                                         kt * BN + 64 * (int)rank, u.bh_kv);
                }
                ++gk;
            }
            {
                const uint32_t st = gv % C::kVStages, round = gv / C::kVStages;
                if (round > 0 && !mbar_wait(&bars[C::kBarVEmpty + st], (round - 1) & 1, abort_flag, to)) {
                    ok = false;
                    break;
                }
                if (rank == 0) mbar_arrive_expect_tx(&bars[C::kBarVFull + st], 2 * C::kVBytes);
                tma_load_3d_pair(sV + st * C::kVBytes, &p.tm_v, cluster_addr(&bars[C::kBarVFull + st], 0),
                                 64 * (int)rank, kt * BN, u.bh_kv);
                ++gv;
            }
        }
    }
    if (!ok) record_timeout(p);
    if (rank != 0) return;  // the pair's copies complete on CTA 0's barriers: CTA 0 drains them
    if (tq > 0) mbar_wait_drain(&bars[C::kBarQFull], (tq - 1) & 1);
    const uint32_t nk = gk < (uint32_t)C::kKStages ? gk : (uint32_t)C::kKStages;
    for (uint32_t i = 0; i < nk; ++i) {
        const uint32_t g = gk - 1 - i;
        if (g != drop) mbar_wait_drain(&bars[C::kBarKFull + g % C::kKStages], (g / C::kKStages) & 1);
    }
    const uint32_t nv = gv < (uint32_t)C::kVStages ? gv : (uint32_t)C::kVStages;
    for (uint32_t i = 0; i < nv; ++i) {
        const uint32_t g = gv - 1 - i;
        mbar_wait_drain(&bars[C::kBarVFull + g % C::kVStages], (g / C::kVStages) & 1);
    }
}

}  // namespace pair

struct PairParams {
    FwdParams p;
    CUtensorMap tm_k64;  // K with 64-row boxes: one CTA's half of a key tile
};

template <bool O_BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::kThreads, 1)
    fa_fwd_pair_kernel(const __grid_constant__ PairParams pp) {
    using C = pair::PCfg;
    const FwdParams &p = pp.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            // CTA 0's s_free, p_full and o_free count one arrival per softmax
            // warp of both CTAs; the exchange barriers the two warps of a
            // sub-partition; everything else one arrival (or one commit)
            const bool pair_warps = i == C::kBarSFree || i == C::kBarSFree + 1 || i == C::kBarPFull || i == C::kBarOFree;
            const bool exch = i >= C::kBarXMax && i < C::kBarDrain;
            mbar_init(&bars[i], pair_warps ? 2u * pair::kSoftmaxWarps : (exch ? 2u : 1u));
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == pair::kMmaWarp) {
        tmem_alloc_pair(tmem_slot, pair::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < pair::kSoftmaxWarps) {
        setmaxnreg_inc<kSoftmaxRegs>();
        if (!pair::softmax_role<O_BF16>(p, bars, abort_flag, smem, tmem, rank, warp, lane)) record_timeout(p);
    } else {
        setmaxnreg_dec<kControlRegs>();
    }
    if (warp == pair::kMmaWarp) {
        if (lane == 0 && rank == 0) {
            if (!pair::mma_role(p, bars, abort_flag, tmem, smem_u32(sQ), smem_u32(sK), smem_u32(sV)))
                record_timeout(p);
            tc_commit_pair(&bars[C::kBarDrain], 1);  // no product may still run when TMEM is released
            mbar_wait_drain(&bars[C::kBarDrain], 0);
        }
    } else if (warp == pair::kLoadWarp) {
        if (lane == 0) pair::load_role(p, &pp.tm_k64, bars, abort_flag, rank, sQ, sK, sV);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while its partner may still signal its barriers
    if (warp == pair::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, pair::kTmemCols);
    }
}

}  // namespace fa

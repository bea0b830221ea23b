// fa_fwd_kernel.cuh -- fused exact attention forward for sm_100a.
//
// One launch computes O = softmax(Q K^T * scale + mask) V and the per-row
// logsumexp (page "FlashAttention (ES)", section "El problema de la atencion
// estandar"), following the three techniques of section "Innovaciones clave de
// FlashAttention":
//   * tiling ("Tiling y procesamiento por bloques"): a work unit is one
//     256-row query block of one (b, h), split into two 128-row tiles A and
//     B; the 128-key K and V tiles stream from HBM into shared memory through
//     TMA and mbarrier rings and each feeds both query tiles; the score tile
//     S = Q K_j^T never leaves the SM;
//   * online softmax ("Calculo de Softmax en linea"): each row keeps a
//     reference maximum m and two running sums of exp2 terms; a new tile's
//     terms are taken relative to m, and when m must grow the accumulated
//     output and sums are multiplied by 2^(m_old - m_new);
//   * one fused kernel ("Fusion de operaciones en un unico kernel de CUDA"):
//     Q K^T, masking, softmax and the product with V run in this one kernel,
//     which writes only O and lse.
//
// Blackwell mapping (one CTA per SM, persistent over work units), 12 warps:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread t of a
//              warpgroup owns row t of its tile; it reads its S row from
//              tensor memory (TMEM), masks, updates m and the sums, writes the
//              bf16 probabilities P back over the S row in TMEM, rescales its
//              O row in TMEM when m moved, and runs the epilogue for its row;
//   warp 8     MMA issuer (one thread): S_X = Q_X K_j^T (both operands in
//              shared memory) and O_X += P_X V_j (P from TMEM, V_j from shared
//              memory), tcgen05.mma with fp32 accumulation in TMEM;
//   warp 9     TMA producer (one thread): Q_A and Q_B once per unit, K_j and
//              V_j through separate rings (warps 10-11 idle).
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256, 256+D),
// O_B [256+D, 256+2D); at d = 128 with bf16 inputs P_X occupies the first 64
// columns of S_X (two bf16 per 32-bit column); at d = 64 it has columns of its
// own (kSepP) and with E4M3 inputs it sits in shared memory (kSmemP), and
// the MMA order is that of the separate-P loop in mma_role.
//
// MMA issue order inside a unit (P over S), for key tiles j = 1, 2, ...:
//     P_A V_{j-1},  Q_A K_j^T,  P_B V_{j-1},  Q_B K_j^T
// so the tensor core works on one tile while the other tile's softmax runs.
// tcgen05.mma operations issued by one thread execute in issue order, which
// makes two things safe: Q_X K_j^T overwrites the S_X columns holding P_X only
// after P_X V_{j-1} has read them, and the commit that signals "S_X(j) ready"
// also covers P_X V_{j-1}, so the softmax may rescale O_X as soon as S_X(j)
// arrives.
//
// Every wait is bounded in wall time.  On time-out the CTA raises a shared
// abort flag, records FA_ERR_DEVICE_TIMEOUT in the optional status word,
// drains its in-flight copies and MMAs (again bounded), frees TMEM and exits.
#pragma once

#include "fa_softmax_row.cuh"

namespace fa {

constexpr int kQTiles = 2;     // query tiles per work unit
constexpr int kUnitRows = BM * kQTiles;
constexpr int kSoftmaxWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;   // warps 10-11 only complete the third warpgroup
constexpr int kThreads = 384;
// Register split (setmaxnreg): the launch gives 384 x 168; the two softmax
// warpgroups take 224 each and the MMA/TMA warpgroup keeps 56:
// 256 * 224 + 128 * 56 = 64512 = 384 * 168, and 224 + 224 + 56 <= 512 per lane
// on every SM sub-partition (one warp of each warpgroup per sub-partition).
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168, "register split exceeds the launch");
constexpr uint32_t kTmemCols = 512;
constexpr int kUnitQueue = 4;  // depth of the shared-memory queue of work-unit ids
// Largest batch for which the unit order sorts the batch elements by their key
// tiles (a table of this many ints in shared memory).
constexpr int kSortMaxB = 128;
constexpr int kStatusTimeout = 5;    // FA_ERR_DEVICE_TIMEOUT
constexpr int kStatusSchedBusy = 7;  // FA_ERR_SCHED_BUSY
// Separate P columns (d = 64): O_A and O_B take 64 TMEM columns each, which
// leaves 128 columns for P_A [384, 448) and P_B [448, 512).  P then no longer
// overwrites S, so Q_X K_{j+1}^T may run as soon as the softmax has read
// S_X(j) (barrier s_free) instead of after P_X V_j: the softmax of a tile no
// longer waits for the P V -> Q K^T chain of its own previous tile.  The
// price: a rescale of O_X and the store of P_X(j+1) first wait for P_X V_j
// (barrier pv_done, one phase per product).
template <int D>
constexpr bool kSepP = (D == 64);
// E4M3: P (one byte per key, 16 KB per tile) goes to shared memory instead of
// over S in TMEM, and P_X V reads it from there (both operands in shared
// memory); as with separate P columns, Q_X K_{j+1}^T may then run as soon as
// the softmax has read S_X(j), and the store of the next P waits for P_X V_j.
template <bool F8>
constexpr bool kSmemP = F8;
// S released once read (barrier s_free), each P_X V signalled (pv_done):
// separate P columns (d = 64) or P in shared memory (E4M3).
template <int D, bool F8>
constexpr bool kSepChain = (kSepP<D> && !F8) || kSmemP<F8>;

__device__ __forceinline__ uint32_t col_s(uint32_t x) { return x * 128u; }                  // S_X, P_X
__device__ __forceinline__ uint32_t col_o(uint32_t x, uint32_t d) { return 256u + x * d; }  // O_X
__device__ __forceinline__ uint32_t col_p_sep(uint32_t x) { return 384u + x * 64u; }         // P_X (d = 64)

struct FwdParams {
    CUtensorMap tm_q, tm_k, tm_v;  // 3-D maps over [B*H][N][D] (Q) and [B*H_kv][Nk][D] (K, V) bf16;
                                   // box {64, 128, 1}; 128-byte swizzle
    CUtensorMap tm_o;              // d = 64, fp32 O: 3-D map over o as [n_splits*B*H][N][64] fp32,
                                   // box {32, 32, 1}, 128-byte swizzle (the epilogue's TMA stores)
    void *o;                       // [n_splits][B, H, N, D] fp32 or bf16 (n_splits > 1: fp32 partials)
    float *lse;                    // [n_splits][B, H, N]
    const int32_t *k_len;          // [B] or nullptr
    int32_t *status;               // device status word or nullptr
    int B, H, N;                   // N queries
    int Nk;                        // keys; query i sits at key position i + Nk - N
    int H_kv;                      // key/value heads; query head h uses key/value head h / group
    int group;                     // H / H_kv
    int n_blocks;                  // ceil(N / 256)
    int n_splits;                  // key-range splits per query block (1: none)
    int split_tiles;               // key tiles per split
    int n_units;                   // B * H * n_blocks * n_splits
    int band_blocks;               // query blocks per band of the unit order (see decode_unit)
    int dynamic;                   // units handed out by the counter (1) or in the static snake order (0)
    int sort_b;                    // 1: key-padded non-causal units go batch element by batch element,
                                   // most key tiles first (B <= kSortMaxB; dynamic)
    uint32_t *sched;               // this launch's scheduler slot: [0] next unit, [1] CTAs done,
                                   // [2, 4) owner (64-bit grid id + 1 of the launch using it, 0: free)
    int causal;
    float scale_log2;              // scale * log2(e)
    float tau;                     // rescale threshold in log2 units (<= 0: rescale on any growth)
    float out_scale;               // factor on O (the value scale of E4M3 inputs; 1 for bf16)
    uint64_t timeout_ns;
    int drop_load;                 // test only (0: off): CTA 0's TMA producer never issues its
                                   // drop_load-th K-tile load (d = 256: ring load), so the
                                   // wait for it runs out and the time-out path runs
};

// F8: Q, K and V in E4M3 (one byte per element, d = 128 only), products on
// tcgen05 kind::f8f6f4; otherwise bf16 and kind::f16.
template <int D, bool F8 = false>
struct Cfg {
    static_assert(!F8 || D == 128, "E4M3 operands: d = 128 only");
    static constexpr int kElemBytes = F8 ? 1 : 2;
    static constexpr int kChunks = D * kElemBytes / 128;  // 128-byte column blocks per row
    static constexpr int kChunkElems = 128 / kElemBytes;  // elements of a row in one column block
    static constexpr int kChunkBytes = BM * 128;           // one column block of a 128-row tile
    static constexpr int kTileBytes = BM * D * kElemBytes; // one 128 x D tile
    static constexpr int kKStages = F8 ? 4 : (D == 128) ? 3 : 4;
    static constexpr int kVStages = F8 ? 4 : (D == 128) ? 2 : 3;  // d = 64: a stage gives way to the O stages
    static constexpr int kOffQ = 0;                                   // Q_A, Q_B
    static constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;
    static constexpr int kOffP = kOffV + kVStages * kTileBytes;  // P_A, P_B (kSmemP)
    static constexpr int kOffBar = kOffP + (kSmemP<F8> ? kQTiles * kTileBytes : 0);
    // barrier slots
    static constexpr int kBarQFull = 0;
    static constexpr int kBarQEmpty = 1;
    static constexpr int kBarKFull = 2;
    static constexpr int kBarKEmpty = kBarKFull + kKStages;
    static constexpr int kBarVFull = kBarKEmpty + kKStages;
    static constexpr int kBarVEmpty = kBarVFull + kVStages;
    static constexpr int kBarSFull = kBarVEmpty + kVStages;  // [2], per query tile
    static constexpr int kBarPFull = kBarSFull + 2;          // [2]
    static constexpr int kBarOFinal = kBarPFull + 2;         // [2]
    static constexpr int kBarOFree = kBarOFinal + 2;         // [2]
    static constexpr int kBarSFree = kBarOFree + 2;          // [2] S_X read by the softmax (separate P)
    static constexpr int kBarPvDone = kBarSFree + 2;         // [2] P_X V complete (separate P)
    static constexpr int kBarUnitFull = kBarPvDone + 2;      // [kUnitQueue]
    static constexpr int kBarUnitFree = kBarUnitFull + kUnitQueue;  // [kUnitQueue]
    static constexpr int kBarDrain = kBarUnitFree + kUnitQueue;
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 4;
    static constexpr int kOffClaimed = kOffAbort + 4;                // scheduler slot claimed (int)
    static constexpr int kOffUnitIds = kOffClaimed + 4;              // [kUnitQueue][4] ints
    static constexpr int kOffBOrder = kOffUnitIds + 16 * kUnitQueue;  // [kSortMaxB] ints
    // d = 64: per softmax warp D / 32 boxes of [32 rows][32 fp32 columns] in the
    // 128-byte swizzle, the source of the fp32 O epilogue's TMA stores
    static constexpr bool kStageO = kSepP<D> && !F8;
    static constexpr int kStageBytes = (D / 32) * 4096;
    static constexpr int kOffStage = (kOffBOrder + 4 * kSortMaxB + 1023) & ~1023;  // swizzled TMA boxes
    static constexpr int kSmemUsed = kOffStage + (kStageO ? kSoftmaxWarps * kStageBytes : 0);
    static constexpr int kSmemBytes = kSmemUsed + 1024;  // + slack to align the base to 1024 bytes
    static_assert(kChunkBytes % 1024 == 0 && kTileBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kOffStage % 1024 == 0, "the O stage holds 128-byte-swizzled TMA boxes");
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
    static_assert(2 * kSmemBytes > 233472, "one CTA per SM: TMEM is allocated whole");
};

struct UnitCoord {
    int bh, b, blk, split;
    int bh_kv;  // key/value head row of K and V: b * H_kv + h / group
    int lo;     // first key tile of this unit's key range
    int n[2];   // key tiles of query tile A and B: tiles [lo, lo + n[x])
    int nmax;
};

// Static schedule (the backward kernel): work unit k of this CTA is taken from
// bands of gridDim.x consecutive units, walked in alternating direction.
__device__ __forceinline__ int unit_index(int k) {
    const int G = gridDim.x, c = blockIdx.x;
    return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// ------------------------------------------------------------------ work distribution
// Units are handed out dynamically, in index order, from a per-launch counter
// in global memory: whichever CTA is free takes the next one, so the causal
// units' unequal costs even out at the end of the launch.  Inside a CTA the
// TMA warp (which runs ahead) takes the ids and passes them to the other
// roles through a small shared-memory queue.
struct UnitQueue {
    volatile int *ids;  // [kUnitQueue][4]: unit id, then two words the producer may attach
    uint64_t *full;     // [kUnitQueue], one arrival: the producer has written the entry
    uint64_t *free;     // [kUnitQueue], one arrival per consuming thread
    const int *b_order; // batch elements longest first (FwdParams::sort_b), else nullptr
};


// Producer (one thread), step 1: the id of this CTA's k-th unit, or -1 when
// none is left (ok turns false when the wait for a free entry times out).
__device__ __forceinline__ int unit_take(const UnitQueue &q, uint32_t *counter, int n_units, bool dynamic, int k,
                                         volatile int *abort_flag, uint64_t timeout_ns, bool &ok) {
    const int slot = k % kUnitQueue;
    if (k >= kUnitQueue && !mbar_wait(&q.free[slot], ((k / kUnitQueue) - 1) & 1, abort_flag, timeout_ns)) {
        ok = false;
        return -1;
    }
    // dynamic: the first unit of CTA c is unit c (no wait at the start), the
    // rest come from the counter after the gridDim.x units taken that way;
    // static: the snake order of unit_index
    const int t = !dynamic ? unit_index(k)
                           : (k == 0 ? (int)blockIdx.x : (int)gridDim.x + (int)atomicAdd(counter, 1u));
    return t < n_units ? t : -1;
}

// Producer, step 2: publish entry k (id t, -1 included so that consumers stop,
// and two attached words).
__device__ __forceinline__ int unit_take(const FwdParams &p, const UnitQueue &q, int k, volatile int *abort_flag,
                                         uint64_t timeout_ns, bool &ok) {
    return unit_take(q, p.sched, p.n_units, p.dynamic != 0, k, abort_flag, timeout_ns, ok);
}

// Static order: every role computes its k-th unit itself (no queue).
__device__ __forceinline__ int unit_static(const FwdParams &p, int k) {
    const int t = unit_index(k);
    return t < p.n_units ? t : -1;
}

__device__ __forceinline__ void unit_publish(const UnitQueue &q, int k, int t, int a, int b) {
    volatile int *e = q.ids + 4 * (k % kUnitQueue);
    e[0] = t;
    e[1] = a;
    e[2] = b;
    mbar_arrive(&q.full[k % kUnitQueue]);  // release: the entry is visible to whoever acquires the phase
}

// Consumer: entry k (returns the id, -1: no more units; a and b the attached
// words); ok turns false if the wait times out or the CTA is aborting.
__device__ __forceinline__ int unit_pop(const UnitQueue &q, int k, volatile int *abort_flag, uint64_t timeout_ns,
                                        bool &ok, int *a = nullptr, int *b = nullptr) {
    const int slot = k % kUnitQueue;
    if (!mbar_wait(&q.full[slot], (k / kUnitQueue) & 1, abort_flag, timeout_ns)) {
        ok = false;
        return -1;
    }
    volatile int *e = q.ids + 4 * slot;
    const int t = e[0];
    if (a) *a = e[1];
    if (b) *b = e[2];
    mbar_arrive(&q.free[slot]);
    return t;
}

// Scheduler slots are shared by all launches on a device (taken round-robin
// by the host), so two launches in flight at once may meet on one slot (more
// launches in flight than slots, or one CUDA graph replayed on several
// streams).  Every CTA therefore claims the slot for its grid before it takes
// a unit: the owner word holds the grid id + 1 of the launch using the slot
// (0: free), set by the first CTA of the launch to arrive and cleared by the
// last to leave.  A CTA that finds another launch's grid id there waits,
// bounded in wall time; the launches serialise on the slot instead of
// sharing its counter.  Returns false when the limit passes (the CTA then
// skips its work and reports FA_ERR_SCHED_BUSY).
__device__ __forceinline__ bool sched_claim(uint32_t *sched, uint64_t timeout_ns) {
    unsigned long long *owner = reinterpret_cast<unsigned long long *>(sched + 2);
    const unsigned long long me = grid_id() + 1ull;
    uint64_t t0 = 0;
    for (;;) {
        const unsigned long long old = atomicCAS(owner, 0ull, me);
        if (old == 0ull || old == me) {
            __threadfence();
            return true;
        }
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        else if (now - t0 > timeout_ns) return false;
        __nanosleep(1000);
    }
}

// The last CTA to finish resets the launch's scheduler words for the next
// launch that uses them (every CTA has taken its last id by then), and only
// then frees the slot.
__device__ __forceinline__ void sched_release(uint32_t *sched) {
    __threadfence();
    if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
        atomicExch(sched, 0u);
        atomicExch(sched + 1, 0u);
        __threadfence();
        atomicExch(reinterpret_cast<unsigned long long *>(sched + 2), 0ull);
    }
}

// Stores `code` in the optional status word unless an earlier error is there.
__device__ __forceinline__ void record_status(int32_t *status, int code) {
    if (status) atomicCAS(reinterpret_cast<int *>(status), 0, code);
}

// Unit numbering: the query blocks of every (b, h) are cut into bands of
// band_blocks consecutive blocks, longest (causal) first; units go band by
// band, head-major inside a band, longest block first within a head, key
// splits innermost.  A band of one block is block-major order (the best
// balance), a band of all blocks head-major order (the CTAs at work share few
// heads' K and V in L2); the host picks the band so that the heads in flight
// fit in L2.  Query tile x of the unit covers the key tiles of the unit's
// split that some row of the tile may attend to.
__device__ __forceinline__ void band_decode(const FwdParams &p, int r, int &bh, int &blk) {
    const int BH = p.B * p.H;
    const int band = r / (p.band_blocks * BH);
    const int in_band = r - band * p.band_blocks * BH;
    const int bsz = min(p.band_blocks, p.n_blocks - band * p.band_blocks);
    bh = in_band / bsz;
    blk = p.n_blocks - 1 - (band * p.band_blocks + (in_band - bh * bsz));
}

__device__ __forceinline__ UnitCoord decode_unit(const FwdParams &p, int t, const int *b_order) {
    UnitCoord u;
    u.split = t % p.n_splits;
    band_decode(p, t / p.n_splits, u.bh, u.blk);
    u.b = u.bh / p.H;
    if (b_order) {  // batch elements with more key tiles first
        const int h = u.bh - u.b * p.H;
        u.b = b_order[u.b];
        u.bh = u.b * p.H + h;
    }
    u.bh_kv = u.b * p.H_kv + (u.bh - u.b * p.H) / p.group;
    u.lo = u.split * p.split_tiles;
    int kv_lim = p.Nk;
    if (p.k_len) kv_lim = min(max(__ldg(p.k_len + u.b), 0), p.Nk);
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const int first = u.blk * kUnitRows + x * BM;
        int e = kv_lim;  // keys [0, e) may be attended to by some row of the tile
        if (p.causal) e = max(0, min(e, first + BM + (p.Nk - p.N)));
        const int tiles = (first < p.N) ? (e + BN - 1) / BN : 0;
        u.n[x] = max(0, min(tiles, u.lo + p.split_tiles) - u.lo);
    }
    u.nmax = max(u.n[0], u.n[1]);
    return u;
}

__device__ __forceinline__ void record_timeout(const FwdParams &p) {
    if (p.status) atomicCAS(reinterpret_cast<int *>(p.status), 0, kStatusTimeout);
}

// Bounded wait that ignores the abort flag: used to drain in-flight work (TMA
// copies and MMAs that were issued and will complete within microseconds).
// Its limit is fixed and generous, independent of the caller's time limit,
// so that a short timeout_ms never lets a CTA exit with copies in flight.
constexpr uint64_t kDrainTimeoutNs = 1000000000ull;
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    int dummy = 0;
    return mbar_wait(bar, parity, &dummy, kDrainTimeoutNs);
}

// ------------------------------------------------------------------ softmax
// One warpgroup, query tile x; thread owns row (warp % 4) * 32 + lane.
// E4M3 probabilities are taken relative to m_ref - kF8Shift (so that they lie
// in (0, 2^(7 + tau)], tau <= 1.75: below E4M3's largest value 448, and
// normal in E4M3 down to 2^-13 of the reference).
constexpr float kF8Shift = 7.f;

template <int D, bool O_BF16, bool F8>
__device__ __forceinline__ bool softmax_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                             const UnitQueue &uq, uint32_t tmem, int x, int warp, int lane,
                                             uint8_t *stage, uint8_t *sP) {
    using C = Cfg<D, F8>;
    const int row_in_tile = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float NEG_INF = __int_as_float(0xff800000);
    uint64_t *s_full = &bars[C::kBarSFull + x];
    uint64_t *p_full = &bars[C::kBarPFull + x];
    uint64_t *o_final = &bars[C::kBarOFinal + x];
    uint64_t *o_free = &bars[C::kBarOFree + x];
    uint64_t *s_free = &bars[C::kBarSFree + x];
    uint64_t *pv_done = &bars[C::kBarPvDone + x];
    constexpr bool kSep = kSepChain<D, F8>;
    const uint32_t t_s = tmem + lane_off + col_s(x);
    const uint32_t t_o = tmem + lane_off + col_o(x, D);
    const uint32_t t_p = tmem + lane_off + ((kSepP<D> && !F8) ? col_p_sep(x) : col_s(x));
    uint32_t gs = 0;  // S tiles of this query tile consumed so far (s_full / p_full phase)
    uint32_t tl = 0;  // units in which this query tile had work (o_final / o_free phase)
    uint32_t pv_known = 0;  // separate P: P_X V products known to be complete
    bool store_pending = false;  // TMA epilogue (lane 0): a store may still be reading the stage
    // separate P: wait until the first n P_X V products are complete (phases
    // complete in order, and product n cannot start before this thread stores
    // P_X(n), so the parity of phase n - 1 is unambiguous)
    auto ensure_pv = [&](uint32_t n) -> bool {
        if (pv_known >= n) return true;
        const bool w = mbar_wait(pv_done, (n - 1) & 1, abort_flag, p.timeout_ns);
        pv_known = n;
        return __all_sync(0xffffffffu, w);
    };
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = p.dynamic ? unit_pop(uq, k, abort_flag, p.timeout_ns, ok) : unit_static(p, k);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || t < 0) break;
        const UnitCoord u = decode_unit(p, t, uq.b_order);
        const int row = u.blk * kUnitRows + x * BM + row_in_tile;
        const bool row_valid = row < p.N;
        // output row: [split][B*H][N] (the split index is 0 without key splits)
        const size_t row_id = ((size_t)u.split * p.B * p.H + u.bh) * p.N + row;
        const int n = u.n[x];
        if (n == 0) {  // no allowed key for these rows: O = 0, lse = -inf
            if (row_valid) fill_row<D, O_BF16>(p.o, p.lse, row_id, false, NEG_INF);
            continue;
        }
        int lim = p.Nk;  // keys [0, lim) are allowed for this row
        if (p.k_len) lim = min(max(__ldg(p.k_len + u.b), 0), p.Nk);
        if (p.causal) lim = min(lim, row + 1 + (p.Nk - p.N));

        RowState st;  // lr: dividing O by it makes O an exact convex combination of V rows
                      // (a lone dominant weight is not rounded away)
        for (int j = 0; j < n; ++j, ++gs) {
            ok = mbar_wait(s_full, gs & 1, abort_flag, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();

            float s[BN];
            uint32_t pk0[32], pk1[32];          // P for keys [0,64) and [64,128), two bf16 per column
            float2 ls = make_float2(0.f, 0.f);  // this tile's unrounded sum (packed pair)
            load_score_row(t_s, s);
            if constexpr (kSep) {  // S_X is in registers: its columns may take the next Q_X K^T
                tc_fence_before();
                mbar_arrive(s_free);
            }
            const float m_new = masked_row_max(s, (u.lo + j) * BN, lim, p.scale_log2);
            float alpha;
            const bool resc = update_reference(st, j, m_new, p.tau, alpha);
            if (__any_sync(0xffffffffu, resc)) {
                // O_X holds P_X V for key tiles < j and nothing is adding to it:
                // the commit that released S_X(j) covered the last such product
                // (separate P: the wait below does), and the next one waits for
                // this tile's P.  Scale in place.
                if constexpr (kSep) {
                    if (!(ok = ensure_pv(gs))) break;
                    tc_fence_after();
                }
                rescale_o_row<D>(t_o, alpha);
            }
            if constexpr (F8) {
                exp_e4m3(s, p.scale_log2, kF8Shift - st.m_ref, pk0, ls);
                // P_X(j - 1) must have been read by its product before it is replaced
                if (!(ok = ensure_pv(gs))) break;
                // this row of P_X: 128 bytes of the K-major tile in the 128-byte swizzle
                uint8_t *prow = sP + x * C::kTileBytes + row_in_tile * 128;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<uint4 *>(prow + ((u ^ (row_in_tile & 7)) << 4)) =
                        make_uint4(pk0[4 * u], pk0[4 * u + 1], pk0[4 * u + 2], pk0[4 * u + 3]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
            } else if constexpr (kSep) {
                exp_half_p<0>(s, p.scale_log2, -st.m_ref, pk0, ls);
                // P_X(j - 1) must have been read by its product before it is replaced
                if (!(ok = ensure_pv(gs))) break;
                tc_fence_after();
                tmem_st32(t_p + 0, pk0);
                exp_half_p<1>(s, p.scale_log2, -st.m_ref, pk1, ls);
                tmem_st32(t_p + 32, pk1);
            } else {
                exp_half_p<0>(s, p.scale_log2, -st.m_ref, pk0, ls);
                tmem_st32(t_s + 0, pk0);  // P overwrites scores already in registers
                exp_half_p<1>(s, p.scale_log2, -st.m_ref, pk1, ls);
                tmem_st32(t_s + 32, pk1);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full);
            // the sums after the "P ready" signal, so that the tensor core gets P
            // sooner: the unrounded one (lse) and, bf16 only, the sum of the
            // rounded probabilities from the packed pairs still in registers
            st.l += ls.x + ls.y;
            if constexpr (!F8) st.lr += rounded_sum(pk0, pk1);
        }
        if (ok) {
            if constexpr (kSep) {
                ok = ensure_pv(gs);  // every product of this unit
            } else {
                ok = mbar_wait(o_final, tl & 1, abort_flag, p.timeout_ns);
                ok = __all_sync(0xffffffffu, ok);
            }
        }
        if (!ok) {  // abandon this unit: mark its rows
            if (row_valid) fill_row<D, O_BF16>(p.o, p.lse, row_id, true, __int_as_float(0x7fc00000));
            break;
        }
        tc_fence_after();
        // a row whose allowed keys all lie outside this unit's key range (key
        // splits) has nothing summed: O = 0, lse = -inf for it.  E4M3: O over
        // the unrounded sum (the rounded and unrounded sums differ only by the
        // unbiased roundings of the weights, each at most 2^-4 relative for
        // the large ones)
        if constexpr (C::kStageO && !O_BF16) {
            // the warp's 32 rows are consecutive output rows starting at lane 0's
            const size_t first_row_id = row_id - lane;
            const int n_valid = min(32, p.N - (row - lane));
            write_rows_tma<D>(t_o, stage, lane, &p.tm_o, row - lane, u.split * p.B * p.H + u.bh, p.lse, first_row_id,
                              n_valid, st.lr, st.m_ref + log2f(st.l), store_pending);
        } else {
            write_row<D, O_BF16>(t_o, p.o, p.lse, row_id, row_valid, F8 ? st.l : st.lr, F8 ? p.out_scale : 1.f,
                                 st.m_ref - (F8 ? kF8Shift : 0.f) + log2f(st.l));
        }
        tc_fence_before();
        mbar_arrive(o_free);
        ++tl;
    }
    if constexpr (C::kStageO && !O_BF16) {
        if (lane == 0 && store_pending) bulk_wait_group0();  // every O store has completed
    }
    return ok;
}

// ------------------------------------------------------------------ MMA issuer
template <int D, bool F8>
__device__ __forceinline__ bool mma_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                         const UnitQueue &uq, uint32_t tmem, uint32_t q_addr, uint32_t k_addr,
                                         uint32_t v_addr, uint32_t p_addr) {
    using C = Cfg<D, F8>;
    const uint32_t idesc_qk = F8 ? idesc_e4m3_f32(BM, BN, false) : idesc_bf16_f32(BM, BN, false);
    const uint32_t idesc_pv = F8 ? idesc_e4m3_f32(BM, D, true) : idesc_bf16_f32(BM, D, true);
    // Descriptors differ only in their start-address field (bits [0,14), in
    // 16-byte units), so each operand's descriptor is a base plus an offset.
    const uint64_t q_desc = sw128_desc(q_addr, 16, 1024);
    const uint64_t k_desc = sw128_desc(k_addr, 16, 1024);
    const uint64_t v_desc = sw128_desc(v_addr, C::kChunkBytes, 1024);
    const uint64_t p_desc = sw128_desc(p_addr, 16, 1024);  // P_A, P_B in shared memory (kSmemP), K-major
    uint32_t tq = 0;              // non-empty units (q_full phase)
    uint32_t gk = 0, gv = 0;      // K and V ring positions
    uint32_t gp0 = 0, gp1 = 0;    // P_X V products issued (p_full phase)
    uint32_t tl0 = 0, tl1 = 0;    // units in which tile X had work (o_free phase)
    const uint64_t to = p.timeout_ns;

    // S_X = Q_X K^T for the key tile in ring slot kslot
    auto qk = [&](int x, uint32_t kslot) {
        const uint64_t qd = q_desc + ((x * C::kTileBytes) >> 4);
        const uint64_t kd = k_desc + ((kslot * C::kTileBytes) >> 4);
        if constexpr (F8) mma_e4m3_ss_k128(tmem + col_s(x), qd, kd, idesc_qk, 0u);
        else if constexpr (D == 128) mma_ss_k128(tmem + col_s(x), qd, kd, idesc_qk, 0u);
        else mma_ss_k64(tmem + col_s(x), qd, kd, idesc_qk, 0u);
        tc_commit(&bars[C::kBarSFull + x]);
    };
    // O_X (+)= P_X V for the value tile in ring slot vslot; `first` starts a
    // fresh accumulator, `last` ends the unit for tile X
    auto pv = [&](int x, uint32_t &gpx, uint32_t tlx, uint32_t vslot, bool first, bool last) -> bool {
        const uint64_t vd = v_desc + ((vslot * C::kTileBytes) >> 4);
        if (!mbar_wait(&bars[C::kBarPFull + x], gpx & 1, abort_flag, to)) return false;
        ++gpx;
        if (first && tlx > 0 && !mbar_wait(&bars[C::kBarOFree + x], (tlx - 1) & 1, abort_flag, to)) return false;
        tc_fence_after();
        mma_ts_k128(tmem + col_o(x, D), tmem + col_s(x), vd, idesc_pv, first ? 0u : 1u);
        if (last) tc_commit(&bars[C::kBarOFinal + x]);
        return true;
    };

    // separate P (d = 64): per key tile j, Q_A K_j^T and Q_B K_j^T as soon as
    // the softmax has read S_X(j - 1), then P_A V_{j-1} and P_B V_{j-1}
    uint32_t gq0 = 0, gq1 = 0;    // Q_X K^T products issued (s_free phase)
    auto qk_sep = [&](int x, uint32_t &gqx, uint32_t kslot) -> bool {
        if (gqx > 0 && !mbar_wait(&bars[C::kBarSFree + x], (gqx - 1) & 1, abort_flag, to)) return false;
        ++gqx;
        tc_fence_after();
        qk(x, kslot);
        return true;
    };
    auto pv_sep = [&](int x, uint32_t &gpx, uint32_t tlx, uint32_t vslot, bool first) -> bool {
        if (!mbar_wait(&bars[C::kBarPFull + x], gpx & 1, abort_flag, to)) return false;
        ++gpx;
        if (first && tlx > 0 && !mbar_wait(&bars[C::kBarOFree + x], (tlx - 1) & 1, abort_flag, to)) return false;
        tc_fence_after();
        if constexpr (F8)
            mma_e4m3_ss_pv_k128(tmem + col_o(x, D), p_desc + ((x * C::kTileBytes) >> 4),
                                v_desc + ((vslot * C::kTileBytes) >> 4), idesc_pv, first ? 0u : 1u);
        else
            mma_ts_k128(tmem + col_o(x, D), tmem + col_p_sep(x), v_desc + ((vslot * C::kTileBytes) >> 4), idesc_pv,
                        first ? 0u : 1u);
        tc_commit(&bars[C::kBarPvDone + x]);
        return true;
    };

    bool ok = true;
    for (int k = 0; ok; ++k) {
        UnitCoord u;  // dynamic: the key-tile counts come with the id (the TMA warp decoded the unit)
        const int t = p.dynamic ? unit_pop(uq, k, abort_flag, to, ok, &u.n[0], &u.n[1]) : unit_static(p, k);
        if (!ok || t < 0) break;
        if (!p.dynamic) u = decode_unit(p, t, uq.b_order);
        u.nmax = max(u.n[0], u.n[1]);
        if (u.nmax == 0) continue;
        if (!mbar_wait(&bars[C::kBarQFull], tq & 1, abort_flag, to)) { ok = false; break; }
        ++tq;
        tc_fence_after();
        if constexpr (kSepChain<D, F8>) {
            for (int j = 0; j <= u.nmax && ok; ++j) {
                if (j < u.nmax) {
                    const uint32_t kslot = gk % C::kKStages;
                    if (!mbar_wait(&bars[C::kBarKFull + kslot], (gk / C::kKStages) & 1, abort_flag, to)) {
                        ok = false;
                        break;
                    }
                    if (j < u.n[0] && !qk_sep(0, gq0, kslot)) { ok = false; break; }
                    if (j < u.n[1] && !qk_sep(1, gq1, kslot)) { ok = false; break; }
                    tc_commit(&bars[C::kBarKEmpty + kslot]);
                    ++gk;
                    if (j == u.nmax - 1) tc_commit(&bars[C::kBarQEmpty]);
                }
                if (j > 0) {
                    const uint32_t vslot = gv % C::kVStages;
                    if (!mbar_wait(&bars[C::kBarVFull + vslot], (gv / C::kVStages) & 1, abort_flag, to)) {
                        ok = false;
                        break;
                    }
                    if (j - 1 < u.n[0] && !pv_sep(0, gp0, tl0, vslot, j == 1)) { ok = false; break; }
                    if (j - 1 < u.n[1] && !pv_sep(1, gp1, tl1, vslot, j == 1)) { ok = false; break; }
                    tc_commit(&bars[C::kBarVEmpty + vslot]);
                    ++gv;
                }
            }
        } else {
          for (int j = 0; j <= u.nmax; ++j) {
            // products with V_{j-1}, interleaved with the scores of key tile j
            const bool have_k = j < u.nmax;
            const uint32_t kslot = gk % C::kKStages, vslot = gv % C::kVStages;
            if (have_k && !mbar_wait(&bars[C::kBarKFull + kslot], (gk / C::kKStages) & 1, abort_flag, to)) {
                ok = false;
                break;
            }
            if (j > 0 && !mbar_wait(&bars[C::kBarVFull + vslot], (gv / C::kVStages) & 1, abort_flag, to)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (j > 0 && j - 1 < u.n[0] && !pv(0, gp0, tl0, vslot, j == 1, j == u.n[0])) { ok = false; break; }
            if (have_k && j < u.n[0]) qk(0, kslot);
            if (j > 0 && j - 1 < u.n[1] && !pv(1, gp1, tl1, vslot, j == 1, j == u.n[1])) { ok = false; break; }
            if (have_k && j < u.n[1]) qk(1, kslot);
            if (j > 0) {
                tc_commit(&bars[C::kBarVEmpty + vslot]);
                ++gv;
            }
            if (have_k) {
                tc_commit(&bars[C::kBarKEmpty + kslot]);
                ++gk;
                if (j == u.nmax - 1) tc_commit(&bars[C::kBarQEmpty]);
            }
          }
        }
        tl0 += u.n[0] > 0;
        tl1 += u.n[1] > 0;
    }
    return ok;
}

// ------------------------------------------------------------------ TMA producer
template <int D, bool F8>
__device__ __forceinline__ void load_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                          const UnitQueue &uq, uint8_t *sQ, uint8_t *sK, uint8_t *sV) {
    using C = Cfg<D, F8>;
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
    const uint64_t to = p.timeout_ns;
    uint32_t tq = 0, gk = 0, gv = 0;
    // test only: the K load this CTA never issues (its ring position), or none
    const uint32_t drop = (blockIdx.x == 0 && p.drop_load > 0) ? (uint32_t)(p.drop_load - 1) : 0xFFFFFFFFu;
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = p.dynamic ? unit_take(p, uq, k, abort_flag, to, ok) : unit_static(p, k);
        if (!ok) break;
        if (t < 0) {
            if (p.dynamic) unit_publish(uq, k, -1, 0, 0);
            break;
        }
        const UnitCoord u = decode_unit(p, t, uq.b_order);
        if (p.dynamic) unit_publish(uq, k, t, u.n[0], u.n[1]);
        if (u.nmax == 0) continue;
        if (tq > 0 && !mbar_wait(&bars[C::kBarQEmpty], (tq - 1) & 1, abort_flag, to)) {
            ok = false;
            break;
        }
        mbar_arrive_expect_tx(&bars[C::kBarQFull], kQTiles * C::kTileBytes);
#pragma unroll
        for (int x = 0; x < kQTiles; ++x)
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_3d(sQ + x * C::kTileBytes + c * C::kChunkBytes, &p.tm_q, &bars[C::kBarQFull],
                            c * C::kChunkElems, u.blk * kUnitRows + x * BM, u.bh);
        ++tq;
        for (int j = 0; j < u.nmax && ok; ++j) {
            {
                const uint32_t slot = gk % C::kKStages, round = gk / C::kKStages;
                if (round > 0 && !mbar_wait(&bars[C::kBarKEmpty + slot], (round - 1) & 1, abort_flag, to)) {
                    ok = false;
                    break;
                }
                if (gk != drop) {
                    mbar_arrive_expect_tx(&bars[C::kBarKFull + slot], C::kTileBytes);
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(sK + slot * C::kTileBytes + c * C::kChunkBytes, &p.tm_k,
                                    &bars[C::kBarKFull + slot], c * C::kChunkElems, (u.lo + j) * BN, u.bh_kv);
                }
                ++gk;
            }
            {
                const uint32_t slot = gv % C::kVStages, round = gv / C::kVStages;
                if (round > 0 && !mbar_wait(&bars[C::kBarVEmpty + slot], (round - 1) & 1, abort_flag, to)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars[C::kBarVFull + slot], C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(sV + slot * C::kTileBytes + c * C::kChunkBytes, &p.tm_v, &bars[C::kBarVFull + slot],
                                c * C::kChunkElems, (u.lo + j) * BN, u.bh_kv);
                ++gv;
            }
        }
    }
    if (!ok) record_timeout(p);
    // drain: every copy this thread issued has landed before the CTA may exit
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

template <int D, bool O_BF16, bool F8 = false>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_sm100_kernel(const __grid_constant__ FwdParams p) {
    using C = Cfg<D, F8>;
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

    int *b_order = reinterpret_cast<int *>(smem + C::kOffBOrder);
    const UnitQueue uq{reinterpret_cast<volatile int *>(smem + C::kOffUnitIds), &bars[C::kBarUnitFull],
                       &bars[C::kBarUnitFree], p.sort_b ? b_order : nullptr};
    if (p.sort_b) {
        // rank of batch element t among all by (key tiles descending, index):
        // its key tiles first go to the table, then every thread t < B counts
        // the elements ahead of it and writes t at its rank
        const int t = threadIdx.x;
        int tiles = 0, rank = 0;
        if (t < p.B) {
            tiles = (min(max(__ldg(p.k_len + t), 0), p.Nk) + BN - 1) / BN;
            b_order[t] = tiles;
        }
        __syncthreads();
        if (t < p.B)
            for (int i = 0; i < p.B; ++i) {
                const int ti = b_order[i];
                rank += (ti > tiles) || (ti == tiles && i < t);
            }
        __syncthreads();
        if (t < p.B) b_order[rank] = t;
    }
    volatile int *claimed = reinterpret_cast<volatile int *>(smem + C::kOffClaimed);
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            const bool per_row = (i >= C::kBarPFull && i < C::kBarPFull + 2) ||
                                 (i >= C::kBarOFree && i < C::kBarOFree + 2) ||
                                 (i >= C::kBarSFree && i < C::kBarSFree + 2);
            // a queued unit id is read by the 256 softmax threads and the MMA thread
            const bool unit_free = i >= C::kBarUnitFree && i < C::kBarUnitFree + kUnitQueue;
            mbar_init(&bars[i], unit_free ? 2u * 128u + 1u : (per_row ? 128u : 1u));
        }
        *abort_flag = 0;
        *claimed = p.dynamic ? (sched_claim(p.sched, p.timeout_ns) ? 1 : 0) : 1;
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
    if (!*claimed) {  // the scheduler slot stayed in use by another launch: no work, report it
        if (threadIdx.x == 0) record_status(p.status, kStatusSchedBusy);
        if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
        return;
    }

    if (warp < kSoftmaxWarps) {
        setmaxnreg_inc<kSoftmaxRegs>();
        uint8_t *stage = smem + C::kOffStage + warp * C::kStageBytes;
        if (!softmax_role<D, O_BF16, F8>(p, bars, abort_flag, uq, tmem, warp >> 2, warp, lane, stage,
                                         smem + C::kOffP))
            record_timeout(p);
    } else {
        setmaxnreg_dec<kControlRegs>();
    }
    if (warp == kMmaWarp) {
        if (lane == 0) {
            if (!mma_role<D, F8>(p, bars, abort_flag, uq, tmem, smem_u32(sQ), smem_u32(sK), smem_u32(sV),
                                 smem_u32(smem + C::kOffP)))
                record_timeout(p);
            // drain: no MMA may still be running when TMEM is released
            tc_commit(&bars[C::kBarDrain]);
            mbar_wait_drain(&bars[C::kBarDrain], 0);
        }
    } else if (warp == kLoadWarp) {
        if (lane == 0) load_role<D, F8>(p, bars, abort_flag, uq, sQ, sK, sV);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && p.dynamic) sched_release(p.sched);
}

}  // namespace fa

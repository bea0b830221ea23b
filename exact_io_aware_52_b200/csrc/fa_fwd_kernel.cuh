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
// O_B [256+D, 256+2D); P_X occupies the first 64 columns of S_X (two bf16 per
// 32-bit column).
//
// MMA issue order inside a unit, for key tiles j = 1, 2, ...:
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

#include "sm100_ptx.cuh"

namespace fa {

constexpr int BM = 128;        // query rows per tile (tcgen05 M)
constexpr int BN = 128;        // keys per tile
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
constexpr int kStatusTimeout = 5;  // FA_ERR_DEVICE_TIMEOUT
// Of every kPolyPeriod key pairs of a score row, the last kPolyPairs take
// their exponentials from the FMA-pipe polynomial, the rest from MUFU ex2.
// Measured on workload 4 (B200, 300 launches): 0 of 4 -> 2.30 ms, 1 of 4 ->
// 2.44 ms, 2 of 4 -> 2.49 ms: the softmax is not MUFU-throughput bound here,
// so the polynomial's extra instructions only cost; it stays off.
constexpr int kPolyPeriod = 4;
constexpr int kPolyPairs = 0;
// P to bf16: round to nearest even (cvt) when false; truncation (keep the
// high half of each fp32 word, one byte permute per pair) when true.
constexpr bool kPackTruncate = false;
// The tile's sum of the bf16-rounded probabilities (two mixed-precision adds
// per pair) is taken after "P ready", from the packed pairs, instead of
// between the exponentials, so that the tensor core gets P sooner; the
// unrounded sum (one packed add per pair) stays beside the exponentials.
constexpr bool kLateSums = true;
static_assert(!kLateSums || (kPolyPairs == 0 && !kPackTruncate), "late sums: MUFU exponentials, rounded P");
// P V in two halves of 64 keys: the softmax releases P for keys [0, 64) as
// soon as it is in TMEM, so the tensor core multiplies that half while the
// softmax computes the other, and only P V for keys [64, 128) plus the next
// Q K^T remain between "P ready" and the next "S ready".  Measured on B200
// (300 launches each): d = 64 (B8 H12 N1024 causal) 48.5 -> 47.1 us; d = 128
// (B1 H32 N16384 causal) 2.249 -> 2.306 ms, where the extra store wait in the
// middle of the softmax costs more than the overlap gains.  On for d = 64 only.
template <int D>
constexpr bool kSplitPV = (D == 64);
// The V ring slot of key tile j-1 is released right after the last P_X V_{j-1}
// product is issued (before Q_B K_j^T) instead of at the end of the step.
// Measured on B200 (300 launches): E4M3 (B1 H32 N16384 causal) 1.852 ->
// 1.788 ms; bf16 d = 128 unchanged, d = 64 (B8 H12 N1024 causal) 43.0 ->
// 44.0 us.  On for E4M3 only.
template <bool F8>
constexpr bool kEarlyVRelease = F8;

__device__ __forceinline__ uint32_t col_s(uint32_t x) { return x * 128u; }                  // S_X, P_X
__device__ __forceinline__ uint32_t col_o(uint32_t x, uint32_t d) { return 256u + x * d; }  // O_X

struct FwdParams {
    CUtensorMap tm_q, tm_k, tm_v;  // 3-D maps over [B*H][N][D] (Q) and [B*H_kv][Nk][D] (K, V) bf16;
                                   // box {64, 128, 1}; 128-byte swizzle
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
    uint32_t *sched;               // this launch's scheduler words: [0] next unit, [1] CTAs done
    int causal;
    float scale_log2;              // scale * log2(e)
    float tau;                     // rescale threshold in log2 units (<= 0: rescale on any growth)
    float out_scale;               // factor on O (the value scale of E4M3 inputs; 1 for bf16)
    uint64_t timeout_ns;
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
    static constexpr int kVStages = F8 ? 4 : (D == 128) ? 2 : 4;
    static constexpr int kOffQ = 0;                                   // Q_A, Q_B
    static constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
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
    static constexpr int kBarPHalf = kBarOFree + 2;          // [2] P of keys [0, 64) in TMEM
    static constexpr int kBarUnitFull = kBarPHalf + 2;       // [kUnitQueue]
    static constexpr int kBarUnitFree = kBarUnitFull + kUnitQueue;  // [kUnitQueue]
    static constexpr int kBarDrain = kBarUnitFree + kUnitQueue;
    static constexpr int kNumBars = kBarDrain + 1;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 4;
    static constexpr int kOffUnitIds = kOffAbort + 4;                // [kUnitQueue][4] ints
    static constexpr int kSmemUsed = kOffUnitIds + 16 * kUnitQueue;
    static constexpr int kSmemBytes = kSmemUsed + 1024;  // + slack to align the base to 1024 bytes
    static_assert(kChunkBytes % 1024 == 0 && kTileBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
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

// The last CTA to finish resets the launch's scheduler words for the next
// launch that uses them (every CTA has taken its last id by then).
__device__ __forceinline__ void sched_release(uint32_t *sched) {
    __threadfence();
    if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
        atomicExch(sched, 0u);
        atomicExch(sched + 1, 0u);
    }
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

__device__ __forceinline__ UnitCoord decode_unit(const FwdParams &p, int t) {
    UnitCoord u;
    u.split = t % p.n_splits;
    band_decode(p, t / p.n_splits, u.bh, u.blk);
    u.b = u.bh / p.H;
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

// Bounded wait that ignores the abort flag: used to drain in-flight work.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    int dummy = 0;
    return mbar_wait(bar, parity, &dummy, timeout_ns);
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

// Probabilities of keys [64H, 64H+64) of one score row against reference -neg_m
// (log2 units): p = 2^(s * scale_log2 - m), summed unrounded into `ls` and as
// the bf16 values the tensor core will use into `lrs`, and packed as bf16
// pairs into pk (column c holds keys 64H + 2c and 64H + 2c + 1).
template <int H>
__device__ __forceinline__ void exp_half(const float *s, float scale_log2, float neg_m, uint32_t (&pk)[32],
                                         float2 &ls, float &lrs) {
    const float2 sl2 = make_float2(scale_log2, scale_log2);
    const float2 nm = make_float2(neg_m, neg_m);
    float2 a[4] = {ls, make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float b[4] = {lrs, 0.f, 0.f, 0.f};
    float2 b2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
        const float2 xx = __ffma2_rn(make_float2(s[64 * H + c], s[64 * H + c + 1]), sl2, nm);
        const bool poly = ((c >> 1) % kPolyPeriod) >= kPolyPeriod - kPolyPairs;
        const float2 pp = poly ? exp2_poly2(xx) : make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
        a[(c >> 1) & 3] = __fadd2_rn(a[(c >> 1) & 3], pp);
        uint32_t pb;
        if constexpr (kPackTruncate) {
            pb = __byte_perm(__float_as_uint(pp.x), __float_as_uint(pp.y), 0x7632);
            b2[(c >> 1) & 3] = __fadd2_rn(b2[(c >> 1) & 3], make_float2(__uint_as_float(pb << 16),
                                                                        __uint_as_float(pb & 0xFFFF0000u)));
        } else {
            pb = pack_bf16x2(pp.x, pp.y);
            b[(c >> 1) & 3] = add_bf16x2_to(b[(c >> 1) & 3], pb);
        }
        pk[c >> 1] = pb;
    }
    ls = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
    const float2 bb = __fadd2_rn(__fadd2_rn(b2[0], b2[1]), __fadd2_rn(b2[2], b2[3]));
    lrs = ((b[0] + b[1]) + (b[2] + b[3])) + (bb.x + bb.y);
}

// Probabilities of keys [64H, 64H+64) as in exp_half, without the rounded
// sum: pk holds the bf16 pairs, `ls` gains the unrounded values.
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
        const float2 p1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
        a[(c >> 2) & 3] = __fadd2_rn(a[(c >> 2) & 3], __fadd2_rn(p0, p1));
        pk[c >> 2] = pack_e4m3x4(p0.x, p0.y, p1.x, p1.y);
    }
    ls = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
}

// ------------------------------------------------------------------ softmax
// One warpgroup, query tile x; thread owns row (warp % 4) * 32 + lane.
// E4M3 probabilities are taken relative to m_ref - kF8Shift (so that they lie
// in (0, 2^8] with eager rescaling, inside E4M3's normal range down to 2^-14
// of the row maximum).
constexpr float kF8Shift = 8.f;

template <int D, bool O_BF16, bool F8>
__device__ __forceinline__ bool softmax_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                             const UnitQueue &uq, uint32_t tmem, int x, int warp, int lane) {
    using C = Cfg<D, F8>;
    const int row_in_tile = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float LN2 = 0.69314718055994530942f;
    const float NEG_INF = __int_as_float(0xff800000);
    uint64_t *s_full = &bars[C::kBarSFull + x];
    uint64_t *p_full = &bars[C::kBarPFull + x];
    uint64_t *p_half = &bars[C::kBarPHalf + x];
    uint64_t *o_final = &bars[C::kBarOFinal + x];
    uint64_t *o_free = &bars[C::kBarOFree + x];
    const uint32_t t_s = tmem + lane_off + col_s(x);
    const uint32_t t_o = tmem + lane_off + col_o(x, D);
    uint32_t gs = 0;  // S tiles of this query tile consumed so far (s_full / p_full phase)
    uint32_t tl = 0;  // units in which this query tile had work (o_final / o_free phase)
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = p.dynamic ? unit_pop(uq, k, abort_flag, p.timeout_ns, ok) : unit_static(p, k);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || t < 0) break;
        const UnitCoord u = decode_unit(p, t);
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

        float m_ref = 0.f;  // reference maximum, log2 units
        float l = 0.f;      // running sum of 2^(x - m_ref), unrounded: gives lse
        float lr = 0.f;     // running sum of bf16(2^(x - m_ref)), the weights the tensor core
                            // multiplies V by: dividing O by it makes O an exact convex
                            // combination of V rows (a lone dominant weight is not rounded away)
        for (int j = 0; j < n; ++j, ++gs) {
            ok = mbar_wait(s_full, gs & 1, abort_flag, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();

            const int kv0 = (u.lo + j) * BN;
            const bool masked = kv0 + BN > lim;  // masking step: keys at or beyond the row's limit
            float s[BN];
            uint32_t pk0[32], pk1[32];          // P for keys [0,64) and [64,128), two bf16 per column
            float2 ls = make_float2(0.f, 0.f);  // this tile's unrounded sum (packed pair)
            float lrs = 0.f;                    // this tile's rounded (bf16) sum
            // the row's 128 scores: four 32-column TMEM loads, one wait
            tmem_ld32f(t_s + 0, s);
            tmem_ld32f(t_s + 32, s + 32);
            tmem_ld32f(t_s + 64, s + 64);
            tmem_ld32f(t_s + 96, s + 96);
            tmem_ld_wait();
            tmem_reg_fence_f<BN>(s);
            if (masked) {
                mask_scores<0>(s, kv0, lim);
                mask_scores<1>(s, kv0, lim);
            }
            const float m_new = fmaxf(max64(s), max64(s + 64)) * p.scale_log2;
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
            if (__any_sync(0xffffffffu, resc)) {
                // O_X holds P_X V for key tiles < j and nothing is adding to it:
                // the commit that released S_X(j) covered the last such product,
                // and the next one waits for this tile's P.  Scale in place.
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
            if constexpr (F8) {
                exp_e4m3(s, p.scale_log2, kF8Shift - m_ref, pk0, ls);
                tmem_st32(t_s + 0, pk0);  // P overwrites scores already in registers
            } else if constexpr (kLateSums) {
                exp_half_p<0>(s, p.scale_log2, -m_ref, pk0, ls);
                tmem_st32(t_s + 0, pk0);  // P overwrites scores already in registers
                if constexpr (kSplitPV<D>) {
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(p_half);
                }
                exp_half_p<1>(s, p.scale_log2, -m_ref, pk1, ls);
                tmem_st32(t_s + 32, pk1);
            } else {
                exp_half<0>(s, p.scale_log2, -m_ref, pk0, ls, lrs);
                tmem_st32(t_s + 0, pk0);  // P overwrites scores already in registers
                if constexpr (kSplitPV<D>) {
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(p_half);
                }
                exp_half<1>(s, p.scale_log2, -m_ref, pk1, ls, lrs);
                tmem_st32(t_s + 32, pk1);
            }
            if constexpr (!F8 && kLateSums) {
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full);
                l += ls.x + ls.y;
                lr += rounded_sum(pk0, pk1);
            } else {
                l += ls.x + ls.y;
                lr += lrs;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full);
            }
        }
        if (ok) {
            ok = mbar_wait(o_final, tl & 1, abort_flag, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (!ok) {  // abandon this unit: mark its rows
            if (row_valid) fill_row<D, O_BF16>(p.o, p.lse, row_id, true, __int_as_float(0x7fc00000));
            break;
        }
        tc_fence_after();
        // a row whose allowed keys all lie outside this unit's key range (key
        // splits) has nothing summed: O = 0, lse = -inf for it
        // E4M3: O over the unrounded sum (with eager rescaling the row maximum's
        // weight 2^8 is exact in E4M3, so the rounded and unrounded sums differ
        // only by the unbiased rounding of the smaller weights)
        const float norm = F8 ? l : lr;
        const bool empty = !(norm > 0.f);
        const float inv_l = empty ? 0.f : (F8 ? p.out_scale : 1.f) / norm;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t r[32];
            tmem_ld32(t_o + ch * 32, r);
            tmem_ld_wait();
            tmem_reg_fence(r);
            if (row_valid) store_row_chunk<D, O_BF16>(p.o, row_id, ch, r, inv_l);
        }
        if (row_valid) p.lse[row_id] = empty ? NEG_INF : (m_ref - (F8 ? kF8Shift : 0.f) + log2f(l)) * LN2;
        tc_fence_before();
        mbar_arrive(o_free);
        ++tl;
    }
    return ok;
}

// ------------------------------------------------------------------ MMA issuer
template <int D, bool F8>
__device__ __forceinline__ bool mma_role(const FwdParams &p, uint64_t *bars, volatile int *abort_flag,
                                         const UnitQueue &uq, uint32_t tmem, uint32_t q_addr, uint32_t k_addr,
                                         uint32_t v_addr) {
    using C = Cfg<D, F8>;
    const uint32_t idesc_qk = F8 ? idesc_e4m3_f32(BM, BN, false) : idesc_bf16_f32(BM, BN, false);
    const uint32_t idesc_pv = F8 ? idesc_e4m3_f32(BM, D, true) : idesc_bf16_f32(BM, D, true);
    // Descriptors differ only in their start-address field (bits [0,14), in
    // 16-byte units), so each operand's descriptor is a base plus an offset.
    const uint64_t q_desc = sw128_desc(q_addr, 16, 1024);
    const uint64_t k_desc = sw128_desc(k_addr, 16, 1024);
    const uint64_t v_desc = sw128_desc(v_addr, C::kChunkBytes, 1024);
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
        if constexpr (F8) {
            if (!mbar_wait(&bars[C::kBarPFull + x], gpx & 1, abort_flag, to)) return false;
            ++gpx;
            if (first && tlx > 0 && !mbar_wait(&bars[C::kBarOFree + x], (tlx - 1) & 1, abort_flag, to)) return false;
            tc_fence_after();
            mma_e4m3_ts_k128(tmem + col_o(x, D), tmem + col_s(x), vd, idesc_pv, first ? 0u : 1u);
        } else if constexpr (kSplitPV<D>) {
            // keys [0, 64): P columns [0, 32), V rows [0, 64); then keys [64, 128)
            if (!mbar_wait(&bars[C::kBarPHalf + x], gpx & 1, abort_flag, to)) return false;
            if (first && tlx > 0 && !mbar_wait(&bars[C::kBarOFree + x], (tlx - 1) & 1, abort_flag, to)) return false;
            tc_fence_after();
            mma_ts_k64(tmem + col_o(x, D), tmem + col_s(x), vd, idesc_pv, first ? 0u : 1u);
            if (!mbar_wait(&bars[C::kBarPFull + x], gpx & 1, abort_flag, to)) return false;
            ++gpx;
            tc_fence_after();
            mma_ts_k64(tmem + col_o(x, D), tmem + col_s(x) + 32, vd + (4 * 2048 >> 4), idesc_pv, 1u);
        } else {
            if (!mbar_wait(&bars[C::kBarPFull + x], gpx & 1, abort_flag, to)) return false;
            ++gpx;
            if (first && tlx > 0 && !mbar_wait(&bars[C::kBarOFree + x], (tlx - 1) & 1, abort_flag, to)) return false;
            tc_fence_after();
            mma_ts_k128(tmem + col_o(x, D), tmem + col_s(x), vd, idesc_pv, first ? 0u : 1u);
        }
        if (last) tc_commit(&bars[C::kBarOFinal + x]);
        return true;
    };

    bool ok = true;
    for (int k = 0; ok; ++k) {
        UnitCoord u;  // dynamic: the key-tile counts come with the id (the TMA warp decoded the unit)
        const int t = p.dynamic ? unit_pop(uq, k, abort_flag, to, ok, &u.n[0], &u.n[1]) : unit_static(p, k);
        if (!ok || t < 0) break;
        if (!p.dynamic) u = decode_unit(p, t);
        u.nmax = max(u.n[0], u.n[1]);
        if (u.nmax == 0) continue;
        if (!mbar_wait(&bars[C::kBarQFull], tq & 1, abort_flag, to)) { ok = false; break; }
        ++tq;
        tc_fence_after();
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
            if (kEarlyVRelease<F8> && j > 0) {
                tc_commit(&bars[C::kBarVEmpty + vslot]);
                ++gv;
            }
            if (have_k && j < u.n[1]) qk(1, kslot);
            if (!kEarlyVRelease<F8> && j > 0) {
                tc_commit(&bars[C::kBarVEmpty + vslot]);
                ++gv;
            }
            if (have_k) {
                tc_commit(&bars[C::kBarKEmpty + kslot]);
                ++gk;
                if (j == u.nmax - 1) tc_commit(&bars[C::kBarQEmpty]);
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
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int t = p.dynamic ? unit_take(p, uq, k, abort_flag, to, ok) : unit_static(p, k);
        if (!ok) break;
        if (t < 0) {
            if (p.dynamic) unit_publish(uq, k, -1, 0, 0);
            break;
        }
        const UnitCoord u = decode_unit(p, t);
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
                mbar_arrive_expect_tx(&bars[C::kBarKFull + slot], C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(sK + slot * C::kTileBytes + c * C::kChunkBytes, &p.tm_k, &bars[C::kBarKFull + slot],
                                c * C::kChunkElems, (u.lo + j) * BN, u.bh_kv);
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
    if (tq > 0) mbar_wait_drain(&bars[C::kBarQFull], (tq - 1) & 1, to);
    const uint32_t nk = gk < (uint32_t)C::kKStages ? gk : (uint32_t)C::kKStages;
    for (uint32_t i = 0; i < nk; ++i) {
        const uint32_t g = gk - 1 - i;
        mbar_wait_drain(&bars[C::kBarKFull + g % C::kKStages], (g / C::kKStages) & 1, to);
    }
    const uint32_t nv = gv < (uint32_t)C::kVStages ? gv : (uint32_t)C::kVStages;
    for (uint32_t i = 0; i < nv; ++i) {
        const uint32_t g = gv - 1 - i;
        mbar_wait_drain(&bars[C::kBarVFull + g % C::kVStages], (g / C::kVStages) & 1, to);
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

    const UnitQueue uq{reinterpret_cast<volatile int *>(smem + C::kOffUnitIds), &bars[C::kBarUnitFull],
                       &bars[C::kBarUnitFree]};
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            const bool per_row = (i >= C::kBarPFull && i < C::kBarPFull + 2) ||
                                 (i >= C::kBarOFree && i < C::kBarOFree + 2) ||
                                 (i >= C::kBarPHalf && i < C::kBarPHalf + 2);
            // a queued unit id is read by the 256 softmax threads and the MMA thread
            const bool unit_free = i >= C::kBarUnitFree && i < C::kBarUnitFree + kUnitQueue;
            mbar_init(&bars[i], unit_free ? 2u * 128u + 1u : (per_row ? 128u : 1u));
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
        setmaxnreg_inc<kSoftmaxRegs>();
        if (!softmax_role<D, O_BF16, F8>(p, bars, abort_flag, uq, tmem, warp >> 2, warp, lane)) record_timeout(p);
    } else {
        setmaxnreg_dec<kControlRegs>();
    }
    if (warp == kMmaWarp) {
        if (lane == 0) {
            if (!mma_role<D, F8>(p, bars, abort_flag, uq, tmem, smem_u32(sQ), smem_u32(sK), smem_u32(sV)))
                record_timeout(p);
            // drain: no MMA may still be running when TMEM is released
            tc_commit(&bars[C::kBarDrain]);
            mbar_wait_drain(&bars[C::kBarDrain], 0, p.timeout_ns);
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

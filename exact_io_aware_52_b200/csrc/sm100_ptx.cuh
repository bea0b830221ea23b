// sm100_ptx.cuh -- inline-PTX wrappers for the sm_100a features the attention
// kernel uses: mbarriers (with time-bounded waits), TMA tensor loads, tensor
// memory (TMEM) allocation and load/store, and tcgen05 MMA with its shared
// memory and instruction descriptors.  Written from the PTX ISA's descriptions
// of these instructions; nothing here is specific to attention.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace fa {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// The temporal launch number of this grid in its context: distinct for every
// kernel launch, CUDA-graph replays included.
__device__ __forceinline__ uint64_t grid_id() {
    uint64_t g;
    asm volatile("mov.u64 %0, %%gridid;" : "=l"(g));
    return g;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of `bar` with parity `parity` to complete, for at most
// `timeout_ns` nanoseconds of wall time.  Returns false (after raising
// *abort_flag) on time-out, or when another thread of the CTA has already
// raised *abort_flag.  The clock is only read after the first failed poll, so
// a wait that is already satisfied costs one try_wait.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          uint64_t timeout_ns) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------- registers
// Per-warpgroup register reallocation; executed by all 128 threads of a
// warpgroup.  The increases of some warpgroups must be covered by the
// decreases of others within the registers the block was launched with.
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- TMA
// 3-D tiled bulk tensor load global -> shared, completion signalled on `bar`
// as transaction bytes.  `map` is the generic address of a __grid_constant__
// CUtensorMap.  The innermost coordinate c0 must be a multiple of 16 bytes'
// worth of elements (8 for bf16); every caller passes multiples of 64.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Element-wise add of a shared-memory tile into global memory through a
// tensor map (TMA reduce, fp32 add for an fp32 map), tracked by the issuing
// thread's bulk async-group.  Out-of-range rows of the box are skipped.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap *map, const void *src, int c0, int c1, int c2) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
        " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1),
        "r"(c2)
        : "memory");
}
// Copy of a shared-memory tile to global memory through a tensor map (TMA
// store), tracked by the issuing thread's bulk async-group.  Elements of the
// box outside the tensor are not written.  The innermost coordinate c0 must
// be a multiple of 16 bytes' worth of elements and no coordinate negative.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group"
        " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1),
        "r"(c2)
        : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every committed bulk group of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- TMEM
// Whole-warp operations.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation previously issued by THIS
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// columns [col, col+32) of TMEM lane (lane_base + t).  The registers are valid
// only after tmem_ld_wait(); tmem_reg_fence() then re-defines them after the
// wait so the compiler cannot hoist their uses above it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// As tmem_ld32, into 32 consecutive floats.
__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float *f) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3]), "=f"(f[4]), "=f"(f[5]), "=f"(f[6]), "=f"(f[7]),
          "=f"(f[8]), "=f"(f[9]), "=f"(f[10]), "=f"(f[11]), "=f"(f[12]), "=f"(f[13]), "=f"(f[14]),
          "=f"(f[15]), "=f"(f[16]), "=f"(f[17]), "=f"(f[18]), "=f"(f[19]), "=f"(f[20]), "=f"(f[21]),
          "=f"(f[22]), "=f"(f[23]), "=f"(f[24]), "=f"(f[25]), "=f"(f[26]), "=f"(f[27]), "=f"(f[28]),
          "=f"(f[29]), "=f"(f[30]), "=f"(f[31])
        : "r"(taddr));
}

template <int N>
__device__ __forceinline__ void tmem_reg_fence_f(float *f) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(f[i])::"memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void tmem_reg_fence(uint32_t (&r)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i])::"memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- tcgen05.mma
// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile.
//   start : shared address of the first element (the tile base is 1024-byte
//           aligned; K-major operands may start 32/64/96 bytes into a row)
//   lbo   : leading-dimension byte offset (K-major swizzled: unused, 16;
//           MN-major: distance between 64-element column blocks)
//   sbo   : stride-dimension byte offset (distance between 8-row groups)
// Bit layout: [0,14) start>>4, [16,30) lbo>>4, [32,46) sbo>>4, [46,48)
// descriptor version 1, [49,52) base offset 0, [61,64) swizzle mode
// (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t start, uint32_t lbo, uint32_t sbo) {
    uint64_t desc = 0;
    desc |= (uint64_t)((start >> 4) & 0x3FFFu);
    desc |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    desc |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    desc |= (uint64_t)1 << 46;
    desc |= (uint64_t)2 << 61;
    return desc;
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator.
//   [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format
//   (1 = bf16), bit 15 A major (0 = K), bit 16 B major (0 = K, 1 = MN),
//   [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], issued by one thread; A is K-major in TMEM
// (lane = row, each 32-bit column packs two consecutive K elements).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// A whole K loop of tcgen05.mma issued back to back from one asm block, the
// per-step descriptors formed in-line (base + start-address offset in 16-byte
// units) so the issuing thread needs no registers for them.
//
// S (+)= A B^T over K = 16 * steps with both operands K-major, 128-byte
// swizzled, stored as 64-element column blocks of `block_bytes` each: step kk
// starts (kk / 4) * block_bytes + (kk % 4) * 32 bytes into both A and B.
// The first step overwrites D when `accumulate` is 0.
#define FA_SS_STEP(OFF)                                      \
    "add.s64 da, %1, " #OFF ";\n\t"                          \
    "add.s64 db, %2, " #OFF ";\n\t"                          \
    "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, pt;\n\t"
__device__ __forceinline__ void mma_ss_k64(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    // K = 64: one column block, offsets 0, 32, 64, 96 bytes
    asm volatile(
        "{\n\t.reg .b64 da, db;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        FA_SS_STEP(2) FA_SS_STEP(4) FA_SS_STEP(6)
        "}" ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_ss_k128(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    // K = 128: two column blocks of 16384 bytes (1024 in 16-byte units)
    asm volatile(
        "{\n\t.reg .b64 da, db;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        FA_SS_STEP(2) FA_SS_STEP(4) FA_SS_STEP(6)
        FA_SS_STEP(1024) FA_SS_STEP(1026) FA_SS_STEP(1028) FA_SS_STEP(1030)
        "}" ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
#undef FA_SS_STEP

// O (+)= P V over 128 keys (8 steps of K = 16): P in TMEM from column a_tmem
// (8 columns per step), V MN-major in shared memory, 16 key rows of 128 bytes
// per step (2048 bytes = 128 in 16-byte units).
#define FA_TS_STEP(TA, DB)                                   \
    "add.u32 ta, %1, " #TA ";\n\t"                           \
    "add.s64 db, %2, " #DB ";\n\t"                           \
    "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, pt;\n\t"
__device__ __forceinline__ void mma_ts_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .b64 db;\n\t.reg .b32 ta;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        FA_TS_STEP(8, 128) FA_TS_STEP(16, 256) FA_TS_STEP(24, 384) FA_TS_STEP(32, 512)
        FA_TS_STEP(40, 640) FA_TS_STEP(48, 768) FA_TS_STEP(56, 896)
        "}" ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D (+)= A B over K = 128 with both operands MN-major in shared memory (A's
// rows and B's columns contiguous, 128-byte swizzle): 8 steps of K = 16, each
// 16 K-rows of 128 bytes (2048 bytes = 128 in 16-byte units) into both.
#define FA_SSMN_STEP(OFF)                                    \
    "add.s64 da, %1, " #OFF ";\n\t"                          \
    "add.s64 db, %2, " #OFF ";\n\t"                          \
    "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, pt;\n\t"
__device__ __forceinline__ void mma_ss_mn_k128(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .b64 da, db;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        FA_SSMN_STEP(128) FA_SSMN_STEP(256) FA_SSMN_STEP(384) FA_SSMN_STEP(512)
        FA_SSMN_STEP(640) FA_SSMN_STEP(768) FA_SSMN_STEP(896)
        "}" ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
#undef FA_SSMN_STEP

// bf16 x bf16 -> fp32 instruction descriptor with a chosen major-ness of A.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
    return idesc_bf16_f32(M, N, b_mn_major) | ((a_mn_major ? 1u : 0u) << 15);
}

// O (+)= P V over 64 keys (4 steps of K = 16): a_tmem and b_desc point at the
// first of the 64 keys (P column a_tmem, V key row b_desc).
__device__ __forceinline__ void mma_ts_k64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .b64 db;\n\t.reg .b32 ta;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        FA_TS_STEP(8, 128) FA_TS_STEP(16, 256) FA_TS_STEP(24, 384)
        "}" ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
#undef FA_TS_STEP

// ---------------------------------------------------------------- 8-bit operands
// Instruction descriptor of tcgen05.mma kind::f8f6f4 with both operands E4M3
// (format code 0) and fp32 accumulation: as idesc_bf16_f32 with the A and B
// format fields left at 0.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool b_mn_major) {
    return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// S (+)= A B^T over K = 128 E4M3 elements: both operands K-major, 128-byte
// rows (one 128-element row per swizzle row), 4 steps of K = 32 = 32 bytes.
#define FA_F8SS_STEP(OFF)                                    \
    "add.s64 da, %1, " #OFF ";\n\t"                          \
    "add.s64 db, %2, " #OFF ";\n\t"                          \
    "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %3, pt;\n\t"
__device__ __forceinline__ void mma_e4m3_ss_k128(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .b64 da, db;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t"
        FA_F8SS_STEP(2) FA_F8SS_STEP(4) FA_F8SS_STEP(6)
        "}" ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
#undef FA_F8SS_STEP

// O (+)= P V over 128 keys of E4M3: P in TMEM (four keys per 32-bit column,
// 8 columns per step of K = 32), V MN-major in shared memory, 32 key rows of
// 128 bytes per step (4096 bytes = 256 in 16-byte units).
#define FA_F8TS_STEP(TA, DB)                                 \
    "add.u32 ta, %1, " #TA ";\n\t"                           \
    "add.s64 db, %2, " #DB ";\n\t"                           \
    "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [ta], db, %3, pt;\n\t"
__device__ __forceinline__ void mma_e4m3_ts_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .b64 db;\n\t.reg .b32 ta;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t"
        FA_F8TS_STEP(8, 256) FA_F8TS_STEP(16, 512) FA_F8TS_STEP(24, 768)
        "}" ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
#undef FA_F8TS_STEP

// O (+)= P V over 128 keys of E4M3 with P in shared memory: P K-major (one
// 128-byte swizzle row of 128 keys per query row, 32 bytes per step of K = 32),
// V MN-major as in mma_e4m3_ts_k128 (4096 bytes = 256 in 16-byte units per step).
#define FA_F8SSPV_STEP(DA, DB)                               \
    "add.s64 da, %1, " #DA ";\n\t"                          \
    "add.s64 db, %2, " #DB ";\n\t"                          \
    "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %3, pt;\n\t"
__device__ __forceinline__ void mma_e4m3_ss_pv_k128(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                    uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .b64 da, db;\n\t.reg .pred p, pt;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.u32 pt, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t"
        FA_F8SSPV_STEP(2, 256) FA_F8SSPV_STEP(4, 512) FA_F8SSPV_STEP(6, 768)
        "}" ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
#undef FA_F8SSPV_STEP

// Four fp32 values rounded to E4M3 (nearest even, saturating) and packed into
// one 32-bit word, a in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x for two lanes on the FMA pipe (the MUFU ex2 unit is the other source of
// exponentials; splitting the work between the two pipes keeps either from
// capping the tile rate).  Cody-Waite style reduction x = n + f with
// n = round(x) taken from the low mantissa bits of x + 1.5*2^23 and
// f in [-1/2, 1/2]; 2^f by a degree-4 polynomial with p(0) = 1 whose
// coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez
// exchange, fitted for this file; max relative error 3.6e-6 evaluated in
// fp32); 2^n enters by adding n to the exponent field.  Inputs below -127
// are clamped there, giving +0 up to the polynomial's error; inputs must be
// below 128.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    const float2 magic = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
    x.x = fmaxf(x.x, -127.f);
    x.y = fmaxf(x.y, -127.f);
    const float2 t = __fadd2_rn(x, magic);  // round(x) + magic, exact integer arithmetic
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));  // exact: |f| <= 1/2
    float2 q = __ffma2_rn(make_float2(0.009782912209630013f, 0.009782912209630013f), f,
                          make_float2(0.055976882576942444f, 0.055976882576942444f));
    q = __ffma2_rn(q, f, make_float2(0.24020710587501526f, 0.24020710587501526f));
    q = __ffma2_rn(q, f, make_float2(0.6931136250495911f, 0.6931136250495911f));
    q = __ffma2_rn(q, f, make_float2(1.f, 1.f));
    // low bits of t hold n (two's complement within the mantissa): bits(t) << 23 == n << 23
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// Packs two floats as bf16 (round to nearest even): `lo` in bits [0,16),
// `hi` in bits [16,32).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// acc + lo(u) + hi(u), each bf16 half of the packed pair widened exactly and
// added in fp32 (mixed-precision add, one instruction per half).
__device__ __forceinline__ float add_bf16x2_to(float acc, uint32_t u) {
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %1;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\t"
        "add.rn.f32.bf16 %0, hi, %0;\n\t}"
        : "+f"(acc)
        : "r"(u));
    return acc;
}

// The two bf16 halves of a packed pair, widened exactly to float.
__device__ __forceinline__ float bf16x2_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16x2_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

}  // namespace fa

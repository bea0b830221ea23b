/*
 * fa_selftest.h -- single-CTA checks of the sm_100a building blocks of the
 * attention kernel (libfa_selftest.so).  Each call launches one small kernel
 * on `stream` (a cudaStream_t), synchronises it and returns 0 on success, 1 on
 * a bad argument, 4 on a CUDA error.  Device-side time-outs store 5 in
 * *status (caller-zeroed device int32).  All pointers are device pointers,
 * 16-byte aligned, owned by the caller.
 *
 * These exercise the tiling step of the page "FlashAttention (ES)", section
 * "Tiling y procesamiento por bloques" (TMA into shared memory), and the two
 * matrix products of section "Fusion de operaciones en un unico kernel de
 * CUDA" (Q K^T and the product with V) on the tensor cores.
 */
#ifndef EXACT_IO_AWARE_52_FA_SELFTEST_H
#define EXACT_IO_AWARE_52_FA_SELFTEST_H

#include <stdint.h>

#if defined(__GNUC__)
#define FA_SELFTEST_EXPORT __attribute__((visibility("default")))
#else
#define FA_SELFTEST_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* TMA-load the bf16 tile src[128][64] with 128-byte swizzle and copy the raw
 * 16384-byte shared-memory image to dst. */
FA_SELFTEST_EXPORT int fa_selftest_tma_sw128(const void *src, void *dst, int32_t *status, void *stream);

/* s[128][128] (fp32) = a[128][K] * b[128][K]^T with tcgen05.mma, a and b bf16
 * K-major in shared memory; K in {64, 128}. */
FA_SELFTEST_EXPORT int fa_selftest_mma_ss(const void *a, const void *b, float *s, int K, int32_t *status,
                                          void *stream);

/* o[128][D] (fp32) = p[128][128] * v[128][D] with tcgen05.mma, p (bf16) staged
 * in tensor memory, v (bf16) MN-major in shared memory; D in {64, 128}. */
FA_SELFTEST_EXPORT int fa_selftest_mma_ts(const void *p, const void *v, float *o, int D, int32_t *status,
                                          void *stream);

/* s[128][128] (fp32) = a[128][128] * b[128][128]^T with tcgen05.mma
 * kind::f8f6f4, a and b E4M3 (one byte each) K-major in shared memory. */
FA_SELFTEST_EXPORT int fa_selftest_mma_e4m3_ss(const void *a, const void *b, float *s, int32_t *status,
                                               void *stream);

/* o[128][128] (fp32) = E4M3(p)[128][128] * v[128][128]: p given in fp32 is
 * rounded to E4M3 (nearest even, saturating) and packed four per TMEM column
 * by the kernel's packer; v E4M3 MN-major in shared memory. */
FA_SELFTEST_EXPORT int fa_selftest_mma_e4m3_ts(const float *p, const void *v, float *o, int32_t *status,
                                               void *stream);

/* y[i] = 2^x[i] (fp32, n even) through the FMA-pipe polynomial exponential the
 * kernel uses for part of its softmax weights (the online softmax of section
 * "Calculo de Softmax en linea"); inputs below -127 give +0. */
FA_SELFTEST_EXPORT int fa_selftest_exp2_poly(const float *x, float *y, int n, void *stream);

/* Measurement, not a check: the exponential unit's rate as the softmax sees
 * it.  One CTA per SM, 4 * warps_per_subpartition warps (1..8 per SM
 * sub-partition); every thread runs `iters` (1..100000) passes of 128
 * exponentials (mix = 0: independent ex2 only; mix = 1: the softmax's mix of
 * one FFMA2, two ex2, one FADD2 and one bf16 pack per pair of keys).
 * *cycles_per_pass (host) receives the mean clock cycles of one warp's pass;
 * 128 * 32 * warps_per_subpartition / *cycles_per_pass is then the ex2 lanes
 * per clock one sub-partition delivered.  Allocates and frees two small
 * device buffers; synchronises `stream`.  Returns 0, 1 for a bad argument,
 * 4 for a CUDA error. */
FA_SELFTEST_EXPORT int fa_selftest_mufu_rate(int warps_per_subpartition, int mix, int iters,
                                             double *cycles_per_pass, void *stream);

/* Wait on a barrier nothing arrives at, with a limit of timeout_ms; the wait
 * must give up and store 5 in *status. */
FA_SELFTEST_EXPORT int fa_selftest_wait_timeout(int32_t *status, uint32_t timeout_ms, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_52_FA_SELFTEST_H */

/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention forward pass.
 *
 * The operation (page "FlashAttention (ES)", section "El problema de la
 * atencion estandar", the Attention equation; masking from section "Fusion de
 * operaciones en un unico kernel de CUDA"):
 *
 *     O   = softmax(Q K^T * scale + mask) V
 *     lse = log( sum over allowed keys of exp(scale * q . k) )   (natural log)
 *
 * computed by one fused kernel launch that tiles Q, K and V through shared
 * memory (section "Tiling y procesamiento por bloques"), keeps a running row
 * maximum and running sum of exponentials (section "Calculo de Softmax en
 * linea") and writes only O and lse (section "Fusion de operaciones en un
 * unico kernel de CUDA"): no N x N buffer, no workspace of any kind.
 *
 * Layout (all tensors contiguous, row-major):
 *   q       : bf16  [B, H, N, d]      (one N x d matrix per (b, h))
 *   k, v    : bf16  [B, H_kv, N_k, d] (fa_fwd: H_kv = H and N_k = N; fa_fwd_ex
 *             may group heads -- query head h attends with key/value head
 *             h / (H / H_kv), the multi-query attention of section
 *             "FlashAttention-2 (2023)" -- and may give more keys than queries,
 *             the cached-keys setting of section "Soluciones especializadas":
 *             query i then sits at key position i + N_k - N)
 *   o       : fp32  [B, H, N, d]  (fa_fwd; fa_fwd_ex may select bf16)
 *   lse     : fp32  [B, H, N]
 *   k_len   : int32 [B]  (fa_fwd_ex only; key j of batch b is masked iff
 *             j >= k_len[b]; values are clamped to [0, N_k] on the device)
 * Mask: causal masks key j for query i when j > i + N_k - N (j > i when
 * N_k = N).  A row with no allowed key gets O = 0, lse = -inf.
 *
 * Ownership: the caller owns every buffer.  The library allocates, frees and
 * synchronises nothing (except fa_read_device_status and fa_fwd_host, which
 * say so), holds no state beyond a per-device cache of properties (and the two
 * copy streams of fa_fwd_host) and the driver's tensor-map entry point, and is
 * safe to call from several threads.
 *
 * Errors: argument errors are returned synchronously and launch nothing.
 * Device-side errors (a pipeline wait that exceeded its time limit) are
 * written to the optional device status word.  All calls are asynchronous on
 * `stream` (a cudaStream_t; NULL is the legacy default stream).
 */
#ifndef EXACT_IO_AWARE_52_FA_H
#define EXACT_IO_AWARE_52_FA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_EXPORT __attribute__((visibility("default")))
#else
#define FA_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARGUMENT = 1, /* NULL pointer, negative size, bad scale, bad dtype */
    FA_ERR_MISALIGNED = 2,       /* a pointer not 16-byte aligned (TMA requirement)   */
    FA_ERR_UNSUPPORTED = 3,      /* d not in {64, 128, 256}, or the device is not sm_100 */
    FA_ERR_CUDA = 4,             /* a CUDA runtime/driver call or the launch failed   */
    FA_ERR_DEVICE_TIMEOUT = 5,   /* (device status word) a pipeline wait timed out     */
    FA_ERR_WORKSPACE_LIMIT = 6,  /* fa_fwd_static_workspace: the splits need more than
                                    FA_STATIC_WORKSPACE_BYTES of scratch                */
    FA_ERR_SCHED_BUSY = 7        /* (device status word) the launch's scheduler slot stayed
                                    in use by another in-flight launch for longer than the
                                    wait limit; the launch did no work                  */
} fa_status;

typedef enum { FA_O_F32 = 0, FA_O_BF16 = 1 } fa_o_dtype;

/* Element type of q, k and v. */
typedef enum {
    FA_IN_BF16 = 0, /* bfloat16, the default                                        */
    FA_IN_E4M3 = 1  /* FP8 E4M3 (one byte; OCP "fn" variant: no infinities), d = 128 */
} fa_in_dtype;

/* Flags for fa_fwd_params.flags. */
enum {
    /* Rescale the running output whenever a row maximum grows, instead of
     * only when it grows by more than a factor 2^8 (bf16 inputs) or 2^1.75
     * (E4M3 inputs, whose weights must stay below E4M3's largest value), the
     * defaults.  Both are exact up to rounding; the default skips most
     * rescales, this one keeps the largest softmax weight of each row at
     * exactly 1 (E4M3: 2^7) before rounding. */
    FA_FLAG_EAGER_RESCALE = 1
};

/*
 * fa_fwd -- the attention forward pass, fp32 output, no key padding.
 *   q, k, v : device bf16 [B, H, N, d], 16-byte aligned
 *   o       : device fp32 [B, H, N, d], 16-byte aligned
 *   lse     : device fp32 [B, H, N]
 *   B, H, N : >= 0 (B*H*N == 0 is a no-op returning FA_OK)
 *   d       : 64, 128 or 256
 *   causal  : 0 or 1
 *   scale   : finite, > 0 (the definition's 1/sqrt(d_k))
 *   stream  : cudaStream_t
 * Equivalent to fa_fwd_ex with k_len = NULL, o_dtype = FA_O_F32, flags = 0,
 * no status word and the default time limit.
 */
FA_EXPORT fa_status fa_fwd(const void *q, const void *k, const void *v, float *o, float *lse,
                 int B, int H, int N, int d, int causal, float scale, void *stream);

typedef struct {
    const void *q, *k, *v;   /* device, in_dtype: q [B, H, N, d]; k, v [B, H_kv, N_k, d] */
    void *o;                 /* device [B, H, N, d], fp32 or bf16 per o_dtype         */
    float *lse;              /* device fp32 [B, H, N]                                 */
    const int32_t *k_len;    /* device int32 [B], or NULL (no key padding)           */
    int32_t *dev_status;     /* device int32 word or NULL; the kernel stores a
                                fa_status there on a device-side error (first error
                                wins); the caller zeroes it before the launch        */
    int B, H, N, d;
    int causal;
    float scale;
    int o_dtype;             /* fa_o_dtype                                            */
    int flags;               /* FA_FLAG_* bits, 0 by default                          */
    uint32_t timeout_ms;     /* per-wait time limit on the device; 0 = 2000 ms        */
    int H_kv;                /* key/value heads (k, v are [B, H_kv, N_k, d]); 0 means H;
                                must divide H (1 = multi-query attention)             */
    int N_k;                 /* keys; 0 means N (queries); query i sits at key
                                position i + N_k - N                                  */
    int num_splits;          /* 0 or 1: one pass over each row's keys.  S > 1: the key
                                range is cut into S contiguous parts processed in
                                parallel (more work units when B*H*ceil(N/256) is
                                below the SM count), their partial results written
                                to `workspace` and merged by a second kernel          */
    void *workspace;         /* device scratch, 16-byte aligned, at least
                                fa_fwd_workspace_bytes(p) bytes; unused when
                                num_splits <= 1.  Owned by the caller; the library
                                writes every byte it reads from it in the same call   */
    size_t workspace_bytes;  /* size of workspace                                     */
    int in_dtype;            /* fa_in_dtype of q, k, v                                */
    float descale_q, descale_k, descale_v;
                             /* E4M3 inputs: the values are q * descale_q, k * descale_k,
                                v * descale_v (per-tensor scales; 0 means 1).  Ignored
                                for bf16.  The products Q K^T and P V run on E4M3 with
                                fp32 accumulation; P is rounded to E4M3 before P V;
                                the softmax is fp32.  Finite and >= 0.                */
    int test_drop_load;      /* test only; 0 (off) in every normal call.  n > 0: the TMA
                                producer of the kernel's first CTA never issues its n-th
                                key-tile load (d = 256: its n-th K/V half-tile load), so
                                the pipeline wait for that tile runs out after timeout_ms
                                and the time-out path (status word, NaN rows, drain,
                                exit) runs with no copy in flight.  Must be >= 0.       */
} fa_fwd_params;

/*
 * fa_fwd_workspace_bytes -- device scratch bytes fa_fwd_ex needs for *p
 * (0 when p->num_splits <= 1): the partial outputs of the key splits, fp32
 * [S][B, H, N, d] and [S][B, H, N].  Host arithmetic only; 0 for a NULL p.
 */
FA_EXPORT size_t fa_fwd_workspace_bytes(const fa_fwd_params *p);

/*
 * fa_fwd_suggest_splits -- a key-split count for *p on the current device.
 * Returns 1 when the unsplit grid already gives every SM two work units or
 * the keys fit one 128-key tile; otherwise the count in [1, key tiles] that
 * minimises a cost model of whole waves of (query block, split) units over
 * the SMs plus the partials' HBM round trip.  Returns 0 on error (NULL, a
 * non-positive size, no CUDA device).
 */
FA_EXPORT int fa_fwd_suggest_splits(const fa_fwd_params *p);

/*
 * fa_fwd_ex -- the forward pass with key padding, output dtype and a status
 * word.  Causal problems hand their work units out through a per-launch
 * counter held by the library (64 slots per device, taken round-robin by
 * causal fa_fwd / fa_fwd_ex / fa_bwd launches).  Each launch's CTAs claim its
 * slot for their grid before taking a unit, so launches that meet on a slot
 * (more than 64 in flight at once on one device, or one CUDA graph replayed
 * on several streams) run one after the other instead of sharing a counter;
 * a launch whose wait for its slot outlasts timeout_ms does no work and
 * stores FA_ERR_SCHED_BUSY in *dev_status.
 *
 * On a device-side timeout the kernel stores FA_ERR_DEVICE_TIMEOUT in
 * *dev_status and stops: the CTA that timed out writes NaN to the rows of the
 * unit it was working on, but its remaining units are never written, and
 * with key splits the merge still runs over whatever partials the workspace
 * holds.  After FA_ERR_DEVICE_TIMEOUT the whole of o and lse is undefined;
 * the error is seen only through the status word, so pass one when the
 * result matters.
 *
 * The library caches device addresses (its scheduler words, and the scratch
 * array of fa_fwd_static_workspace) per device ordinal for the life of the
 * process.  Do not reset a device (cudaDeviceReset) between calls into this
 * library: the module is reloaded at a possibly different address and the
 * cached addresses would be stale.
 */
FA_EXPORT fa_status fa_fwd_ex(const fa_fwd_params *p, void *stream);

typedef struct {
    const void *q, *k, *v;   /* host, dev.in_dtype, shapes as in dev (pinned for async copies) */
    const int32_t *k_len;    /* host int32 [B] or NULL                                */
    void *o;                 /* host output, dtype per dev.o_dtype                    */
    float *lse;              /* host fp32 [B, H, N]                                   */
    fa_fwd_params dev;       /* device buffers of the same shapes (q, k, v, o, lse,
                                and k_len when k_len is not NULL) plus the options    */
} fa_fwd_host_params;

/*
 * fa_fwd_host -- end-to-end call on HOST buffers: copies q, k, v (and k_len)
 * host -> device into the caller's device buffers, runs fa_fwd_ex, copies o
 * and lse device -> host, and synchronises `stream` before returning.
 * A call whose copies total 64 MB or more, and that gives every SM at least
 * two work units per piece, is cut into up to 8 pieces: whole batch elements
 * (B > 1) or whole groups of query heads sharing a key/value head (B = 1).
 * Piece c's copies in run on a copy-in stream, its fa_fwd_ex on `stream` once
 * they have landed, and its copies out on a copy-out stream once the kernel is
 * done, so that copies in both directions and the kernels of different pieces
 * overlap (the two streams are created once per device and kept).  The
 * result equals the single call's bit for bit (each piece is a valid
 * fa_fwd_ex problem with the caller's options; a call that cannot be cut that
 * way runs whole).  Host buffers should be pinned for the copies to overlap.
 * Work queued earlier on `stream` completes before the first copy.  If
 * dev.dev_status is set, a device-side error found after the copies is
 * returned as its fa_status.
 */
FA_EXPORT fa_status fa_fwd_host(const fa_fwd_host_params *p, void *stream);

/*
 * fa_read_device_status -- synchronises `stream`, reads the device status
 * word and returns it as a fa_status (FA_ERR_CUDA if the read fails).
 */
FA_EXPORT fa_status fa_read_device_status(const int32_t *dev_status, void *stream);

/* Human-readable name of a status code (static string, never NULL). */
FA_EXPORT const char *fa_status_string(fa_status s);

/* Library version as an integer MAJOR*10000 + MINOR*100 + PATCH. */
FA_EXPORT int fa_version(void);

/*
 * Backward pass: the gradients of the forward's O with respect to q, k and v
 * for a given dO.  The pages report training speed-ups of the method (page
 * "FlashAttention (ES)", section "Resultados empiricos") but give no
 * backward algorithm; this is the derivative of the definition of section
 * "El problema de la atencion estandar", with P recomputed from q, k and the
 * forward's lse:
 *     dV = P^T dO,  dP = dO V^T,  dS = scale * P o (dP - D),  D_i = dO_i . O_i,
 *     dQ = dS K,    dK = dS^T Q
 * (o the elementwise product).  Masks, N_k, grouped heads and k_len are those
 * of the forward; dK and dV of a key/value head sum over its query heads.
 */
typedef struct {
    const void *q, *k, *v;   /* device bf16: q [B, H, N, d]; k, v [B, H_kv, N_k, d]    */
    const void *o;           /* device forward output [B, H, N, d], fp32 or bf16 (o_dtype) */
    const void *dout;        /* device bf16 [B, H, N, d]: gradient of the loss w.r.t. O  */
    const float *lse;        /* device fp32 [B, H, N] from the forward with the same inputs */
    float *dq;               /* device fp32 [B, H, N, d], overwritten                   */
    float *dk, *dv;          /* device fp32 [B, H_kv, N_k, d], overwritten              */
    const int32_t *k_len;    /* device int32 [B] or NULL, as in fa_fwd_params           */
    int32_t *dev_status;     /* device status word or NULL, as in fa_fwd_params         */
    int B, H, N, d;          /* d in {64, 128}                                          */
    int causal;
    float scale;
    int o_dtype;             /* fa_o_dtype of o                                         */
    uint32_t timeout_ms;     /* per-wait time limit on the device; 0 = 2000 ms          */
    int H_kv, N_k;           /* 0 means H and N                                         */
    void *workspace;         /* device scratch of at least fa_bwd_workspace_bytes(p),
                                16-byte aligned, owned by the caller                    */
    size_t workspace_bytes;
} fa_bwd_params;

/* Scratch bytes fa_bwd needs for *p: D, fp32 [B, H, N].  0 for a NULL p. */
FA_EXPORT size_t fa_bwd_workspace_bytes(const fa_bwd_params *p);

/*
 * fa_bwd -- two launches on `stream`: D and a zeroed dQ, then the gradients
 * (dQ accumulated in fp32 by TMA reduce-adds, one key tile per work unit).
 * All pointers except k_len and dev_status must be 16-byte aligned.  Errors
 * as for fa_fwd_ex (d not in {64, 128}: FA_ERR_UNSUPPORTED).  dq, dk and dv
 * are deterministic up to the order of the fp32 additions into dq.
 */
FA_EXPORT fa_status fa_bwd(const fa_bwd_params *p, void *stream);

/* Size of the library's fixed device scratch array (64 MiB), per device. */
#define FA_STATIC_WORKSPACE_BYTES (64u * 1024u * 1024u)

/*
 * fa_fwd_static_workspace -- fa_fwd_ex with the key-split scratch taken from
 * a fixed device array inside the library instead of p->workspace, so that
 * the call allocates no memory.  The pages have no counterpart: their
 * forward pass has no key splits and hence no scratch; this is an interface
 * convenience of this library.
 *
 * p is read as by fa_fwd_ex except that p->workspace and p->workspace_bytes
 * are ignored.  With p->num_splits > 1 the scratch is a file-scope device
 * array of FA_STATIC_WORKSPACE_BYTES; a problem whose splits need more
 * (fa_fwd_workspace_bytes(p) > FA_STATIC_WORKSPACE_BYTES) is rejected with
 * FA_ERR_WORKSPACE_LIMIT before anything is launched.  With num_splits <= 1
 * no scratch is used and the call is fa_fwd_ex.
 *
 * The array is one per device and every call on that device uses it:
 * calls whose executions overlap (on different streams, or from different
 * host threads) race on it and their results are undefined.  Serialise them,
 * e.g. on one stream.  Nothing in it has to start at zero.
 *
 * The first call with num_splits > 1 on a device looks the array's address
 * up (cudaGetSymbolAddress, with that device current) and caches it; make
 * that first call before any stream capture.  Errors: those of fa_fwd_ex,
 * FA_ERR_WORKSPACE_LIMIT, and FA_ERR_CUDA if the lookup fails.
 */
FA_EXPORT fa_status fa_fwd_static_workspace(const fa_fwd_params *p, void *stream);

/*
 * Test hooks (not for production use): the scheduler slot the next causal
 * launch from this process will take, and a synchronous read (get4) and/or
 * overwrite (set4) of a slot's four words on the current device ([0] next
 * unit, [1] CTAs done, [2..3] the 64-bit owner, little-endian; all zero when
 * the slot is free).  They let a test hold a slot the way an in-flight
 * launch would, without a second launch.  Errors: FA_ERR_INVALID_ARGUMENT
 * for a slot outside [0, 64), FA_ERR_UNSUPPORTED / FA_ERR_CUDA from the
 * device.
 */
FA_EXPORT int fa_testhook_sched_next_slot(void);
FA_EXPORT fa_status fa_testhook_sched_slot(int slot, const uint32_t *set4, uint32_t *get4);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_52_FA_H */

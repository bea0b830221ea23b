/*
 * fp64 CPU oracle for the exact attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library) never links, loads or calls it, and the two share no code.
 *
 * What it computes is the plain definition of scaled dot-product attention,
 * Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V, from the page
 * "FlashAttention (ES)", section "El problema de la atencion estandar"
 * (the Attention equation), written out row by row:
 *
 *   1. the bf16 input bits are widened exactly to double;
 *   2. the full score row s_j = sigma * sum_t q_it k_jt is materialised for
 *      every key j in [0, N) (sigma is the float scale the GPU receives,
 *      widened to double);
 *   3. the masking step named in section "Fusion de operaciones en un unico
 *      kernel de CUDA" removes keys outside the allowed set
 *      A_i = { j : (not causal or j <= i) and j < L_b };
 *   4. a max-subtracted softmax over A_i: m = max s_j, e_j = exp(s_j - m),
 *      l = sum e_j, p_j = e_j / l;
 *   5. O_i = sum_j p_j v_j and lse_i = m + ln l (natural log of
 *      sum_j exp(s_j) over A_i).  An empty A_i gives O_i = 0, lse_i = -inf.
 *
 * Queries and keys may differ in number (N_q queries against N_k keys, the
 * cached-keys setting of section "Soluciones especializadas"): query i then
 * sits at key position i + N_k - N_q, and the causal mask allows key j iff
 * j <= i + N_k - N_q (with N_q = N_k this is j <= i).
 *
 * Grouped keys and values (the multi-query attention that section
 * "FlashAttention-2 (2023)" says the method was extended to): with H_kv
 * key/value heads, query head h attends with key/value head h / (H / H_kv);
 * H_kv = H is ordinary multi-head attention, H_kv = 1 multi-query attention.
 *
 * There is no tiling, no online recurrence and no reordering beyond this
 * definition: one score row at a time, in key order.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Exact widening of a bf16 bit pattern: bf16 is the top half of an IEEE
 * binary32, so shifting the 16 bits up gives the same value as a float. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * attn_oracle_f64
 *   q       : bf16 bit patterns, contiguous [B, H, N, d]   (N queries)
 *   k, v    : bf16 bit patterns, contiguous [B, H_kv, Nk, d] (Nk keys); H_kv divides H
 *   k_len   : NULL, or int32[B]; key j of batch b is masked iff j >= k_len[b]
 *             (values outside [0, Nk] are clamped to it)
 *   causal  : nonzero masks key j for query i when j > i + Nk - N
 *   scale   : the float multiplier applied to q.k (1/sqrt(d_k) in the
 *             definition); widened to double
 *   rows    : NULL (every row, in order) or n_rows flat row ids
 *             r = (b*H + h)*N + i
 *   o       : double [n_rows, d]      lse : double [n_rows]
 *   nthreads: OpenMP threads (<= 0: library default)
 * Returns 0, or -1 on a bad argument, -2 on allocation failure.
 */
int attn_oracle_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    const int32_t *k_len, int B, int H, int H_kv, int N, int Nk, int d,
                    int causal, float scale, const int64_t *rows,
                    int64_t n_rows, double *o, double *lse, int nthreads) {
    if (B < 0 || H < 0 || N < 0 || d <= 0) return -1;
    if (H_kv <= 0 || H % H_kv != 0) return -1;
    if (Nk < 0) return -1;
    if (!q || !k || !v || !o || !lse) return (n_rows == 0) ? 0 : -1;
    const int64_t total_rows = (int64_t)B * H * N;
    if (!rows) n_rows = total_rows;
    const double sigma = (double)scale;
    int bad = 0;
    int oom = 0;
    const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();

#pragma omp parallel num_threads(nt)
    {
        double *s = (double *)malloc(sizeof(double) * (Nk > 0 ? (size_t)Nk : 1));
        double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
        if (!s || !qrow) {
#pragma omp atomic write
            oom = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < n_rows; ++t) {
            if (!s || !qrow) continue;
            const int64_t r = rows ? rows[t] : t;
            if (r < 0 || r >= total_rows) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int64_t bh = r / N;
            const int i = (int)(r % N);
            const int b = (int)(bh / H);
            const int h = (int)(bh % H);
            const int64_t bh_kv = (int64_t)b * H_kv + h / (H / H_kv); /* this head's key/value head */
            int L = Nk;
            if (k_len) {
                L = k_len[b];
                if (L < 0) L = 0;
                if (L > Nk) L = Nk;
            }
            const uint16_t *qi = q + r * d;
            const uint16_t *kb = k + bh_kv * (int64_t)Nk * d;
            const uint16_t *vb = v + bh_kv * (int64_t)Nk * d;
            double *oi = o + t * d;

            /* step 1-2: widened query row, full score row over every key */
            for (int c = 0; c < d; ++c) qrow[c] = bf16_bits_to_double(qi[c]);
            for (int j = 0; j < Nk; ++j) {
                const uint16_t *kj = kb + (int64_t)j * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += qrow[c] * bf16_bits_to_double(kj[c]);
                s[j] = sigma * acc;
            }
            /* step 3: allowed set A_i */
            int allowed_end = L;                    /* keys [0, L) survive padding */
            if (causal && (int64_t)i + 1 + Nk - N < allowed_end)
                allowed_end = (int)((int64_t)i + 1 + Nk - N);      /* j <= i + Nk - N */
            /* step 4: max-subtracted softmax over A_i = [0, allowed_end) */
            if (allowed_end <= 0) {
                for (int c = 0; c < d; ++c) oi[c] = 0.0;
                lse[t] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int j = 0; j < allowed_end; ++j)
                if (s[j] > m) m = s[j];
            double l = 0.0;
            for (int j = 0; j < allowed_end; ++j) {
                s[j] = exp(s[j] - m);   /* e_j, overwriting the score row */
                l += s[j];
            }
            /* step 5: O_i = sum_j (e_j / l) v_j */
            for (int c = 0; c < d; ++c) oi[c] = 0.0;
            for (int j = 0; j < allowed_end; ++j) {
                const double p = s[j] / l;
                const uint16_t *vj = vb + (int64_t)j * d;
                for (int c = 0; c < d; ++c) oi[c] += p * bf16_bits_to_double(vj[c]);
            }
            lse[t] = m + log(l);
        }
        free(s);
        free(qrow);
    }
    if (oom) return -2;
    return bad ? -1 : 0;
}

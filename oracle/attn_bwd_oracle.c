/*
 * fp64 CPU oracle for the gradients of exact attention (the backward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library) never links, loads or calls it, and the two share no code.
 *
 * The pages report training speed-ups of the method (page "FlashAttention
 * (ES)", section "Resultados empiricos") but give no backward algorithm,
 * so what is computed here is the plain derivative of the forward definition
 * of section "El problema de la atencion estandar".  With
 *     S = sigma Q K^T (+ mask),  P = softmax_rows(S),  O = P V
 * and dO the gradient of a loss with respect to O, the chain rule (through the
 * row softmax, whose Jacobian is diag(p) - p p^T) gives
 *     dV = P^T dO
 *     dP = dO V^T
 *     dS_ij = P_ij (dP_ij - D_i),   D_i = sum_c dO_ic O_ic
 *     dQ = sigma dS K
 *     dK = sigma dS^T Q
 * Masked (query, key) pairs have P = 0 and contribute nothing; a row with no
 * allowed key has O = 0 and zero gradients.  The mask, the N_q / N_k alignment
 * and the grouped key/value heads are those of the forward oracle
 * (attn_oracle.c); dK and dV of a key/value head are sums over the query heads
 * that use it.  Everything is recomputed from Q, K, V and dO in double, one
 * score row at a time, in key order.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * attn_bwd_oracle_f64
 *   q, dout : bf16 bit patterns [B, H, N, d]
 *   k, v    : bf16 bit patterns [B, H_kv, Nk, d]; H_kv divides H
 *   k_len   : NULL or int32[B] (key j of batch b masked iff j >= k_len[b], clamped to [0, Nk])
 *   causal  : nonzero masks key j for query i when j > i + Nk - N
 *   scale   : the float multiplier sigma of q.k, widened to double
 *   dq      : out, double [B, H, N, d]
 *   dk, dv  : out, double [B, H_kv, Nk, d]
 * Returns 0, or -1 on bad sizes or a failed allocation.
 */
int attn_bwd_oracle_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                        const int32_t *k_len, int B, int H, int H_kv, int N, int Nk, int d, int causal,
                        float scale, double *dq, double *dk, double *dv, int nthreads) {
    if (B < 0 || H <= 0 || H_kv <= 0 || H % H_kv || N < 0 || Nk < 0 || d <= 0) return -1;
    const double sigma = (double)scale;
    const int group = H / H_kv;
    const int64_t n_groups = (int64_t)B * H_kv;
    int failed = 0;
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : failed)
    {
        double *p = malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double *dp = malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double *qi = malloc(sizeof(double) * d);
        double *doi = malloc(sizeof(double) * d);
        double *oi = malloc(sizeof(double) * d);
        if (!p || !dp || !qi || !doi || !oi) failed = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t g = 0; g < n_groups; ++g) {
            if (failed) continue;
            const int b = (int)(g / H_kv);
            const int hk = (int)(g % H_kv);
            const uint16_t *kb = k + g * (int64_t)Nk * d;
            const uint16_t *vb = v + g * (int64_t)Nk * d;
            double *dkb = dk + g * (int64_t)Nk * d;
            double *dvb = dv + g * (int64_t)Nk * d;
            memset(dkb, 0, sizeof(double) * (size_t)Nk * d);
            memset(dvb, 0, sizeof(double) * (size_t)Nk * d);
            int L = Nk;
            if (k_len) {
                L = k_len[b];
                if (L < 0) L = 0;
                if (L > Nk) L = Nk;
            }
            for (int h = hk * group; h < (hk + 1) * group; ++h) {
                const int64_t bh = (int64_t)b * H + h;
                for (int i = 0; i < N; ++i) {
                    const int64_t r = bh * N + i;
                    double *dqi = dq + r * d;
                    for (int c = 0; c < d; ++c) {
                        qi[c] = bf16_to_double(q[r * d + c]);
                        doi[c] = bf16_to_double(dout[r * d + c]);
                        dqi[c] = 0.0;
                    }
                    int end = L;  /* allowed keys: [0, end) */
                    if (causal && (int64_t)i + 1 + Nk - N < end) end = (int)((int64_t)i + 1 + Nk - N);
                    if (end <= 0) continue;
                    /* P row: max-subtracted softmax of the scaled scores */
                    double m = -INFINITY;
                    for (int j = 0; j < end; ++j) {
                        const uint16_t *kj = kb + (int64_t)j * d;
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += qi[c] * bf16_to_double(kj[c]);
                        p[j] = sigma * acc;
                        if (p[j] > m) m = p[j];
                    }
                    double l = 0.0;
                    for (int j = 0; j < end; ++j) {
                        p[j] = exp(p[j] - m);
                        l += p[j];
                    }
                    for (int j = 0; j < end; ++j) p[j] /= l;
                    /* O row and D_i = dO_i . O_i */
                    for (int c = 0; c < d; ++c) oi[c] = 0.0;
                    for (int j = 0; j < end; ++j) {
                        const uint16_t *vj = vb + (int64_t)j * d;
                        for (int c = 0; c < d; ++c) oi[c] += p[j] * bf16_to_double(vj[c]);
                    }
                    double Di = 0.0;
                    for (int c = 0; c < d; ++c) Di += doi[c] * oi[c];
                    /* dP_ij = dO_i . v_j ; dS_ij = P_ij (dP_ij - D_i) */
                    for (int j = 0; j < end; ++j) {
                        const uint16_t *vj = vb + (int64_t)j * d;
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += doi[c] * bf16_to_double(vj[c]);
                        dp[j] = p[j] * (acc - Di);
                    }
                    /* dQ_i = sigma sum_j dS_ij k_j ; dK_j += sigma dS_ij q_i ; dV_j += P_ij dO_i */
                    for (int j = 0; j < end; ++j) {
                        const uint16_t *kj = kb + (int64_t)j * d;
                        double *dkj = dkb + (int64_t)j * d;
                        double *dvj = dvb + (int64_t)j * d;
                        const double ds = sigma * dp[j];
                        for (int c = 0; c < d; ++c) {
                            dqi[c] += ds * bf16_to_double(kj[c]);
                            dkj[c] += ds * qi[c];
                            dvj[c] += p[j] * doi[c];
                        }
                    }
                }
            }
        }
        free(p);
        free(dp);
        free(qi);
        free(doi);
        free(oi);
    }
    return failed ? -1 : 0;
}

/*
 * attn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of multi-head causal scaled-dot-product
 * self-attention, forward and backward.  It exists so that the tests, the
 * smoke check and the CPU-baseline leg of the benchmark can check and time
 * the CUDA path; the product path never calls it, links it or loads it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (per batch b and head h, all arithmetic in double):
 *
 *   Forward -- "Stanford CS336 walkthrough" (lmnt.cn), section 5.1 model.py,
 *   CausalSelfAttention.forward: the scores are q @ k^T times 1/sqrt(d)
 *   (the caller passes that factor as `scale`); positions above the diagonal
 *   are filled with -inf (section 3.3 of the same page: the upper triangle is
 *   set to negative infinity so that its softmax weight is zero; the mask
 *   buffer is torch.tril(ones), so the diagonal is kept -- "Train Your Own
 *   LLM from Scratch" (fishgap.com), section 1, the register_buffer line);
 *   a softmax along each row; then y = att @ v.  Dropout is the identity
 *   (p = 0.0 in every configuration the pages print).
 *
 *   Optional document mask -- "How to build an LLM by hand" (agmtopy.github.io),
 *   section 5.5 on BOS-aligned best-fit packing: several documents share one
 *   row.  Reading: a token sees only earlier tokens of its own document.
 *   doc_start[b*T + i] is the first position of the document holding i, and
 *   i attends to j iff doc_start[i] <= j <= i.
 *
 *   Optional sliding window -- the same page, section 9 (gpt.py walkthrough),
 *   lists sliding-window attention among the model's attention features
 *   without stating its definition.  Reading: a window of w keys, the query's
 *   own position included: i attends to j iff i - w < j <= i (and the
 *   document rule, when both apply).  window <= 0 means no window.
 *
 *   Log-sum-exp -- the natural log of the softmax denominator of the SCALED
 *   scores: lse_i = max_j s_ij + log(sum_j exp(s_ij - max_j s_ij)).
 *
 *   Backward -- the pages only call loss.backward() (CS336 walkthrough,
 *   section 5.2 train.py).  The oracle differentiates the forward above by
 *   the chain rule, with the softmax Jacobian J = diag(p) - p p^T formed
 *   explicitly, entry by entry, for every row:
 *     dV_j  = sum_i p_ij dO_i
 *     dP_ij = <dO_i, v_j>
 *     dS_ij = sum_k J_i[j][k] dP_ik      (J_i[j][k] = p_ij [j==k] - p_ij p_ik)
 *     dQ_i  = scale * sum_j dS_ij k_j
 *     dK_j  = scale * sum_i dS_ij q_i
 *   This costs O(L^2) per row (O(T^3) per head); it deliberately does not use
 *   the rowsum(dO * O) shortcut that the CUDA path uses, so agreement between
 *   the two is a real check.
 *
 * Layout: every tensor is contiguous [B, H, T, d] (row-major, d fastest);
 * lse is [B, H, T]; doc_start is [B, T] int32 or NULL.
 *
 * Parallelism: OpenMP over the B*H independent (b, h) pairs only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARGS 1
#define ORACLE_ERR_NOMEM 2

int oracle_version(void) { return 1; }

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Is key position j visible from query position i?  (diagonal included) */
static int visible(const int32_t *doc_row, int window, int i, int j) {
    if (j > i) return 0;
    if (doc_row != NULL && j < doc_row[i]) return 0;
    if (window > 0 && j <= i - window) return 0;
    return 1;
}

static int check_args(const void *a, const void *b, const void *c, int B, int H, int T, int d) {
    if (a == NULL || b == NULL || c == NULL) return ORACLE_ERR_ARGS;
    if (B <= 0 || H <= 0 || T <= 0 || d <= 0) return ORACLE_ERR_ARGS;
    return ORACLE_OK;
}

/*
 * Softmax probabilities of row i of one head: p[0..i] (entries for invisible
 * j are exactly 0).  Returns the log-sum-exp of the scaled scores.
 * s is scratch of length >= i+1.
 */
static double softmax_row(const double *qh, const double *kh, int d, double scale,
                          const int32_t *doc_row, int window, int i, double *s, double *p) {
    const double *qi = qh + (size_t)i * d;
    double m = -INFINITY;
    for (int j = 0; j <= i; ++j) {
        if (!visible(doc_row, window, i, j)) { s[j] = -INFINITY; continue; }
        const double *kj = kh + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
        s[j] = scale * acc;
        if (s[j] > m) m = s[j];
    }
    /* m is finite: j == i is always visible. */
    double z = 0.0;
    for (int j = 0; j <= i; ++j) {
        p[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
        z += p[j];
    }
    for (int j = 0; j <= i; ++j) p[j] /= z;
    return m + log(z);
}

/*
 * Forward.  o: [B,H,T,d]; lse: [B,H,T] (may be NULL); probs: [B,H,T,T] or
 * NULL (the full attention matrix, invisible entries 0 -- for small tests).
 */
int oracle_attn_fwd_window(const double *q, const double *k, const double *v,
                           int B, int H, int T, int d, double scale,
                           const int32_t *doc_start, int window,
                           double *o, double *lse, double *probs) {
    if (check_args(q, k, v, B, H, T, d) || o == NULL) return ORACLE_ERR_ARGS;
    const long BH = (long)B * H;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)T);
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
        if (s == NULL || p == NULL) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                const long b = bh / H;
                const size_t off = (size_t)bh * T * d;
                const double *qh = q + off, *kh = k + off, *vh = v + off;
                double *oh = o + off;
                const int32_t *doc_row = doc_start ? doc_start + (size_t)b * T : NULL;
                for (int i = 0; i < T; ++i) {
                    double l = softmax_row(qh, kh, d, scale, doc_row, window, i, s, p);
                    if (lse) lse[(size_t)bh * T + i] = l;
                    double *oi = oh + (size_t)i * d;
                    for (int c = 0; c < d; ++c) oi[c] = 0.0;
                    for (int j = 0; j <= i; ++j) {
                        if (p[j] == 0.0) continue;
                        const double *vj = vh + (size_t)j * d;
                        for (int c = 0; c < d; ++c) oi[c] += p[j] * vj[c];
                    }
                    if (probs) {
                        double *prow = probs + ((size_t)bh * T + i) * T;
                        for (int j = 0; j < T; ++j) prow[j] = (j <= i) ? p[j] : 0.0;
                    }
                }
            }
        }
        free(s);
        free(p);
    }
    return err;
}

/*
 * Backward by the explicit softmax Jacobian.  dq, dk, dv: [B,H,T,d], fully
 * overwritten.
 */
int oracle_attn_bwd_window(const double *q, const double *k, const double *v,
                           const double *dout, int B, int H, int T, int d, double scale,
                           const int32_t *doc_start, int window,
                           double *dq, double *dk, double *dv) {
    if (check_args(q, k, v, B, H, T, d) || dout == NULL || dq == NULL || dk == NULL || dv == NULL)
        return ORACLE_ERR_ARGS;
    const long BH = (long)B * H;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)T);
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
        double *dp = (double *)malloc(sizeof(double) * (size_t)T);
        double *ds = (double *)malloc(sizeof(double) * (size_t)T);
        double *jrow = (double *)malloc(sizeof(double) * (size_t)T);
        if (!s || !p || !dp || !ds || !jrow) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                const long b = bh / H;
                const size_t off = (size_t)bh * T * d;
                const double *qh = q + off, *kh = k + off, *vh = v + off, *doh = dout + off;
                double *dqh = dq + off, *dkh = dk + off, *dvh = dv + off;
                const int32_t *doc_row = doc_start ? doc_start + (size_t)b * T : NULL;
                memset(dqh, 0, sizeof(double) * (size_t)T * d);
                memset(dkh, 0, sizeof(double) * (size_t)T * d);
                memset(dvh, 0, sizeof(double) * (size_t)T * d);
                for (int i = 0; i < T; ++i) {
                    softmax_row(qh, kh, d, scale, doc_row, window, i, s, p);
                    const double *doi = doh + (size_t)i * d;
                    const double *qi = qh + (size_t)i * d;
                    /* dV_j += p_ij dO_i ;  dP_ij = <dO_i, v_j> */
                    for (int j = 0; j <= i; ++j) {
                        const double *vj = vh + (size_t)j * d;
                        double *dvj = dvh + (size_t)j * d;
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) {
                            dvj[c] += p[j] * doi[c];
                            acc += doi[c] * vj[c];
                        }
                        dp[j] = acc;
                    }
                    /* dS_i = J_i dP_i with J_i[j][kk] = p_j [j==kk] - p_j p_kk, formed explicitly. */
                    for (int j = 0; j <= i; ++j) {
                        for (int kk = 0; kk <= i; ++kk)
                            jrow[kk] = (j == kk ? p[j] : 0.0) - p[j] * p[kk];
                        double acc = 0.0;
                        for (int kk = 0; kk <= i; ++kk) acc += jrow[kk] * dp[kk];
                        ds[j] = acc;
                    }
                    /* dQ_i = scale sum_j dS_ij k_j ;  dK_j += scale dS_ij q_i */
                    double *dqi = dqh + (size_t)i * d;
                    for (int j = 0; j <= i; ++j) {
                        if (ds[j] == 0.0) continue;
                        const double *kj = kh + (size_t)j * d;
                        double *dkj = dkh + (size_t)j * d;
                        const double g = scale * ds[j];
                        for (int c = 0; c < d; ++c) {
                            dqi[c] += g * kj[c];
                            dkj[c] += g * qi[c];
                        }
                    }
                }
            }
        }
        free(s);
        free(p);
        free(dp);
        free(ds);
        free(jrow);
    }
    return err;
}

/* Plain causal (or document-causal) attention: no window. */
int oracle_attn_fwd(const double *q, const double *k, const double *v,
                    int B, int H, int T, int d, double scale,
                    const int32_t *doc_start, double *o, double *lse, double *probs) {
    return oracle_attn_fwd_window(q, k, v, B, H, T, d, scale, doc_start, 0, o, lse, probs);
}

int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    int B, int H, int T, int d, double scale, const int32_t *doc_start,
                    double *dq, double *dk, double *dv) {
    return oracle_attn_bwd_window(q, k, v, dout, B, H, T, d, scale, doc_start, 0, dq, dk, dv);
}

/*
 * Plain fp64 CPU oracle for causal grouped-query attention with a learned
 * per-head attention sink, an optional sliding window and intra-document
 * (varlen) masking.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code with the CUDA path.
 *
 * What it computes, and where the pages name it:
 *   - Attention sinks: "gpt-oss implementation" (Megatron-LM issue 1739),
 *     section "Attention Mechanisms / Attention Sinks", which points to
 *     StreamingLLM; "Tricks from OpenAI gpt-oss you can use with
 *     transformers", kernels section ("Flash Attention 3 with support for
 *     attention sinks"); tpu-inference PR 861 ("gpt-oss"), where the kernel
 *     takes an `attention_sink` argument.  The pages name the sink but never
 *     write it out; the plain reading used here is the gpt-oss one: one
 *     extra logit s_h per query head that joins each row's softmax
 *     denominator and carries no value:
 *         out_i = sum_j exp(l_ij - m) v_j / (exp(s_h - m) + sum_j exp(l_ij - m)).
 *     s_h is added in logit space as is (it is not multiplied by `scale`).
 *   - Alternating sliding-window / full-causal layers: Megatron-LM issue
 *     1739, "Alternating Sliding-Window Attention Pattern"; the transformers
 *     blog, "Dynamic Sliding Window Layer & Cache"; torchtitan PR 1559,
 *     "FlexAttention sink/sliding".  Reading used: a window of W keys
 *     including the query itself, 0 <= i - j < W; W <= 0 means full causal.
 *   - Intra-document masking: Megatron-LM issue 1739, the request for
 *     "intra-doc masking (attention only within a document)".  Reading used:
 *     positions, causality and the window are document-local, and no
 *     attention crosses a cu_seqlens boundary.
 *   - Grouped-query attention: query head h reads key/value head
 *     floor(h / (Hq / Hkv)).
 *
 * The oracle is the definition written out: for every row it forms the
 * allowed key set, the scaled logits, their maximum (together with the sink),
 * the denominator, the output and lse = m + ln(Z) (the sink is inside lse).
 * The backward pass is the derivative of that definition:
 *   P_ij = exp(l_ij - lse_i), P_sink,i = exp(s_h - lse_i),
 *   D_i = sum_d dout_id out_id, dP_ij = dout_i . v_j,
 *   dS_ij = P_ij (dP_ij - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_{i,h in group} dS_ij q_i,
 *   dv_j = sum_{i,h in group} P_ij dout_i,  dsinks_h = -sum_i P_sink,i D_i.
 * (d out_i / d s_h = -P_sink,i out_i and d out_i / d l_ij = P_ij (v_j - out_i).)
 *
 * Layouts: q[T][Hq][D], k/v[T][Hkv][D], out[T][Hq][D], lse[Hq][T];
 * cu_seqlens[B+1] (host, int32) with cu_seqlens[0] = 0 and cu_seqlens[B] = T.
 * bf16 inputs are given as their 16-bit patterns and widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* Exact widening of a bf16 bit pattern: bf16 is the top half of an fp32. */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_bf16_to_f64(const uint16_t* src, double* dst, int64_t n) {
    if (n < 0 || (n > 0 && (!src || !dst))) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) dst[i] = bf16_bits_to_double(src[i]);
    return ORACLE_OK;
}

static int check_common(int T, int Hq, int Hkv, int D, int B, const int32_t* cu) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || B < 0 || !cu) return 0;
    if (Hq % Hkv != 0) return 0;
    if (cu[0] != 0 || cu[B] != T) return 0;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] < cu[b]) return 0;
    return 1;
}

/* Document that holds token t (cu is sorted). */
static int doc_of(const int32_t* cu, int B, int64_t t) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* First allowed key (absolute token index) for query token t in a document
 * starting at token a:  doc-local i = t - a, keys j with 0 <= i - j < W. */
static int64_t first_key(int64_t t, int64_t a, int window) {
    if (window <= 0) return a;
    int64_t lo = t - (int64_t)window + 1;
    return lo > a ? lo : a;
}

/* One row of the forward definition: query token t, query head h.
 * logits: scratch of at least (t - a + 1) doubles.
 * Writes out_row[D] and returns lse. */
static double fwd_row(int64_t t, int h, int64_t a, int Hq, int Hkv, int D,
                      const double* q, const double* k, const double* v,
                      double sink, int window, double scale,
                      double* logits, double* out_row) {
    const int G = Hq / Hkv;
    const int g = h / G;
    const int64_t j0 = first_key(t, a, window);
    const double* qi = q + (t * Hq + h) * (int64_t)D;

    /* l_ij = scale * q_i . k_j over the allowed keys */
    double m = sink;
    for (int64_t j = j0; j <= t; ++j) {
        const double* kj = k + (j * Hkv + g) * (int64_t)D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
        double l = scale * dot;
        logits[j - j0] = l;
        if (l > m) m = l;
    }
    /* Z = exp(s - m) + sum_j exp(l_ij - m); a sink of -inf contributes 0.
     * Every row has at least its own key, so m is finite. */
    double Z = exp(sink - m);
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int64_t j = j0; j <= t; ++j) {
        double p = exp(logits[j - j0] - m);
        Z += p;
        const double* vj = v + (j * Hkv + g) * (int64_t)D;
        for (int d = 0; d < D; ++d) out_row[d] += p * vj[d];
    }
    for (int d = 0; d < D; ++d) out_row[d] /= Z;
    return m + log(Z);
}

/* Forward over every (token, head) row, fp64 inputs. */
int oracle_fwd_f64(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                   const double* q, const double* k, const double* v, const double* sinks,
                   int window, double scale, double* out, double* lse, int nthreads) {
    if (!check_common(T, Hq, Hkv, D, B, cu_seqlens) || !sinks || !out || !lse) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v)) return ORACLE_ERR_ARG;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen) maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        if (!logits) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t row = 0; row < (int64_t)T * Hq; ++row) {
                int64_t t = row / Hq;
                int h = (int)(row % Hq);
                int64_t a = cu_seqlens[doc_of(cu_seqlens, B, t)];
                lse[(int64_t)h * T + t] = fwd_row(t, h, a, Hq, Hkv, D, q, k, v, sinks[h], window, scale,
                                                  logits, out + (t * Hq + h) * (int64_t)D);
            }
            free(logits);
        }
    }
    return err;
}

/* Forward for a chosen list of query tokens (all heads), fp64 inputs.
 * out_rows[n][Hq][D], lse_rows[Hq][n]. */
int oracle_fwd_rows_f64(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                        const double* q, const double* k, const double* v, const double* sinks,
                        int window, double scale, const int64_t* rows, int64_t nrows,
                        double* out_rows, double* lse_rows, int nthreads) {
    if (!check_common(T, Hq, Hkv, D, B, cu_seqlens) || !sinks || !rows || nrows < 0) return ORACLE_ERR_ARG;
    if (nrows > 0 && (!out_rows || !lse_rows || !q || !k || !v)) return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return ORACLE_ERR_ARG;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen) maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        if (!logits) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t idx = 0; idx < nrows * Hq; ++idx) {
                int64_t r = idx / Hq;
                int h = (int)(idx % Hq);
                int64_t t = rows[r];
                int64_t a = cu_seqlens[doc_of(cu_seqlens, B, t)];
                lse_rows[(int64_t)h * nrows + r] =
                    fwd_row(t, h, a, Hq, Hkv, D, q, k, v, sinks[h], window, scale, logits,
                            out_rows + (r * Hq + h) * (int64_t)D);
            }
            free(logits);
        }
    }
    return err;
}

/* Backward, fp64 inputs.  dout[T][Hq][D]; out_for_D: if non-NULL, the output
 * used to form D_i = dout_i . out_i (e.g. a bf16-rounded saved output);
 * if NULL, the oracle's own fp64 output is used.
 * Results: dq[T][Hq][D], dk/dv[T][Hkv][D], dsinks[Hq] (all overwritten). */
int oracle_bwd_f64(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                   const double* q, const double* k, const double* v, const double* sinks,
                   int window, double scale, const double* out_for_D, const double* dout,
                   double* dq, double* dk, double* dv, double* dsinks, int nthreads) {
    if (!check_common(T, Hq, Hkv, D, B, cu_seqlens) || !sinks || !dsinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen) maxlen = cu_seqlens[b + 1] - cu_seqlens[b];

    memset(dq, 0, sizeof(double) * (size_t)T * Hq * D);
    memset(dk, 0, sizeof(double) * (size_t)T * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)T * Hkv * D);
    /* Per (document, kv head) partial sink gradients, summed in a fixed
     * order at the end so the result does not depend on thread timing. */
    const int64_t ntask = (int64_t)B * Hkv;
    double* dsink_part = (double*)calloc((size_t)(ntask > 0 ? ntask : 1) * G, sizeof(double));
    if (!dsink_part) return ORACLE_ERR_NOMEM;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double* orow = (double*)malloc(sizeof(double) * (size_t)D);
        if (!logits || !orow) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
            /* One task = one document x one kv head: it owns dk/dv of that
             * document's keys for that head, so tasks never write the same
             * element. */
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < ntask; ++task) {
                int b = (int)(task / Hkv);
                int g = (int)(task % Hkv);
                int64_t a = cu_seqlens[b], e = cu_seqlens[b + 1];
                for (int64_t t = a; t < e; ++t) {
                    for (int hh = 0; hh < G; ++hh) {
                        int h = g * G + hh;
                        double lse = fwd_row(t, h, a, Hq, Hkv, D, q, k, v, sinks[h], window, scale,
                                             logits, orow);
                        const double* o = out_for_D ? out_for_D + (t * Hq + h) * (int64_t)D : orow;
                        const double* doi = dout + (t * Hq + h) * (int64_t)D;
                        const double* qi = q + (t * Hq + h) * (int64_t)D;
                        double* dqi = dq + (t * Hq + h) * (int64_t)D;
                        double Di = 0.0;
                        for (int d = 0; d < D; ++d) Di += doi[d] * o[d];
                        dsink_part[task * G + hh] -= exp(sinks[h] - lse) * Di;
                        int64_t j0 = first_key(t, a, window);
                        for (int64_t j = j0; j <= t; ++j) {
                            const double* kj = k + (j * Hkv + g) * (int64_t)D;
                            const double* vj = v + (j * Hkv + g) * (int64_t)D;
                            double P = exp(logits[j - j0] - lse);
                            double dP = 0.0;
                            for (int d = 0; d < D; ++d) dP += doi[d] * vj[d];
                            double dS = P * (dP - Di);
                            double* dkj = dk + (j * Hkv + g) * (int64_t)D;
                            double* dvj = dv + (j * Hkv + g) * (int64_t)D;
                            for (int d = 0; d < D; ++d) {
                                dqi[d] += scale * dS * kj[d];
                                dkj[d] += scale * dS * qi[d];
                                dvj[d] += P * doi[d];
                            }
                        }
                    }
                }
            }
        }
        free(logits);
        free(orow);
    }
    for (int h = 0; h < Hq; ++h) dsinks[h] = 0.0;
    for (int64_t task = 0; task < ntask; ++task) {
        int g = (int)(task % Hkv);
        for (int hh = 0; hh < G; ++hh) dsinks[g * G + hh] += dsink_part[task * G + hh];
    }
    free(dsink_part);
    return err;
}

/* The sink gradient alone, fp64 inputs:
 *   dsinks_h = -sum over every document and query token i of P_sink,i D_i,
 *   P_sink,i = exp(s_h - lse_i),  D_i = dout_i . out_i.
 * It needs each row's lse and output only, i.e. one forward pass, not the
 * whole backward.  out_for_D as for oracle_bwd_f64.  Each row's term is
 * formed independently; each head then sums its terms in ascending token
 * order. */
int oracle_bwd_dsinks_f64(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                          const double* q, const double* k, const double* v, const double* sinks,
                          int window, double scale, const double* out_for_D, const double* dout,
                          double* dsinks, int nthreads) {
    if (!check_common(T, Hq, Hkv, D, B, cu_seqlens) || !sinks || !dsinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v || !dout)) return ORACLE_ERR_ARG;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen) maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    double* term = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * Hq);
    if (!term) return ORACLE_ERR_NOMEM;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double* orow = (double*)malloc(sizeof(double) * (size_t)D);
        if (!logits || !orow) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t row = 0; row < (int64_t)T * Hq; ++row) {
                int64_t t = row / Hq;
                int h = (int)(row % Hq);
                int64_t a = cu_seqlens[doc_of(cu_seqlens, B, t)];
                double lse = fwd_row(t, h, a, Hq, Hkv, D, q, k, v, sinks[h], window, scale, logits, orow);
                const double* o = out_for_D ? out_for_D + (t * Hq + h) * (int64_t)D : orow;
                const double* doi = dout + (t * Hq + h) * (int64_t)D;
                double Di = 0.0;
                for (int d = 0; d < D; ++d) Di += doi[d] * o[d];
                term[(int64_t)h * T + t] = exp(sinks[h] - lse) * Di;
            }
        }
        free(logits);
        free(orow);
    }
    for (int h = 0; h < Hq; ++h) {
        double acc = 0.0;
        for (int64_t t = 0; t < T; ++t) acc -= term[(int64_t)h * T + t];
        dsinks[h] = acc;
    }
    free(term);
    return err;
}

/* Backward restricted to chosen query tokens: dq for every head of each
 * token in `rows` (fp64 inputs).  dq_i only needs row i's own probabilities,
 * so each row is the definition above evaluated for that row alone.
 * out_for_D as for oracle_bwd_f64.  dq_rows[n][Hq][D]. */
int oracle_bwd_dq_rows_f64(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                           const double* q, const double* k, const double* v, const double* sinks,
                           int window, double scale, const double* out_for_D, const double* dout,
                           const int64_t* rows, int64_t nrows, double* dq_rows, int nthreads) {
    if (!check_common(T, Hq, Hkv, D, B, cu_seqlens) || !sinks || !rows || nrows < 0) return ORACLE_ERR_ARG;
    if (nrows > 0 && (!q || !k || !v || !dout || !dq_rows)) return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen) maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double* orow = (double*)malloc(sizeof(double) * (size_t)D);
        if (!logits || !orow) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t idx = 0; idx < nrows * Hq; ++idx) {
                int64_t r = idx / Hq;
                int h = (int)(idx % Hq);
                int g = h / G;
                int64_t t = rows[r];
                int64_t a = cu_seqlens[doc_of(cu_seqlens, B, t)];
                double lse = fwd_row(t, h, a, Hq, Hkv, D, q, k, v, sinks[h], window, scale, logits, orow);
                const double* o = out_for_D ? out_for_D + (t * Hq + h) * (int64_t)D : orow;
                const double* doi = dout + (t * Hq + h) * (int64_t)D;
                double* dqi = dq_rows + (r * Hq + h) * (int64_t)D;
                double Di = 0.0;
                for (int d = 0; d < D; ++d) Di += doi[d] * o[d];
                for (int d = 0; d < D; ++d) dqi[d] = 0.0;
                int64_t j0 = first_key(t, a, window);
                for (int64_t j = j0; j <= t; ++j) {
                    const double* kj = k + (j * Hkv + g) * (int64_t)D;
                    const double* vj = v + (j * Hkv + g) * (int64_t)D;
                    double P = exp(logits[j - j0] - lse);
                    double dP = 0.0;
                    for (int d = 0; d < D; ++d) dP += doi[d] * vj[d];
                    double dS = P * (dP - Di);
                    for (int d = 0; d < D; ++d) dqi[d] += scale * dS * kj[d];
                }
            }
        }
        free(logits);
        free(orow);
    }
    return err;
}

/* Backward restricted to chosen key tokens: dk and dv for every key/value
 * head of each token in `keys` (fp64 inputs).  dk_j and dv_j sum over every
 * query row (and every head of the group) allowed to see key j; those rows'
 * lse_i and D_i come from their own forward rows.  keys must be sorted
 * ascending.  dk_rows/dv_rows [n][Hkv][D]. */
int oracle_bwd_dkv_rows_f64(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                            const double* q, const double* k, const double* v, const double* sinks,
                            int window, double scale, const double* out_for_D, const double* dout,
                            const int64_t* keys, int64_t nkeys, double* dk_rows, double* dv_rows, int nthreads) {
    if (!check_common(T, Hq, Hkv, D, B, cu_seqlens) || !sinks || !keys || nkeys < 0) return ORACLE_ERR_ARG;
    if (nkeys > 0 && (!q || !k || !v || !dout || !dk_rows || !dv_rows)) return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nkeys; ++r)
        if (keys[r] < 0 || keys[r] >= T || (r > 0 && keys[r] < keys[r - 1])) return ORACLE_ERR_ARG;
    if (nkeys == 0) return ORACLE_OK;
    const int G = Hq / Hkv;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen) maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    /* Query tokens that see at least one chosen key: a query t sees key j
     * when j <= t, they share a document, and t - j < window (if any). */
    char* need = (char*)calloc((size_t)(T > 0 ? T : 1), 1);
    double* lse_all = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * Hq);
    double* D_all = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * Hq);
    if (!need || !lse_all || !D_all) {
        free(need); free(lse_all); free(D_all);
        return ORACLE_ERR_NOMEM;
    }
    for (int64_t r = 0; r < nkeys; ++r) {
        int64_t j = keys[r];
        int64_t e = cu_seqlens[doc_of(cu_seqlens, B, j) + 1];
        int64_t hi = (window > 0 && j + window < e) ? j + window : e;
        for (int64_t t = j; t < hi; ++t) need[t] = 1;
    }
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    /* Pass 1: lse_i and D_i of every needed (query, head) row. */
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double* orow = (double*)malloc(sizeof(double) * (size_t)D);
        if (!logits || !orow) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t idx = 0; idx < (int64_t)T * Hq; ++idx) {
                int64_t t = idx / Hq;
                int h = (int)(idx % Hq);
                if (!need[t]) continue;
                int64_t a = cu_seqlens[doc_of(cu_seqlens, B, t)];
                double lse = fwd_row(t, h, a, Hq, Hkv, D, q, k, v, sinks[h], window, scale, logits, orow);
                const double* o = out_for_D ? out_for_D + (t * Hq + h) * (int64_t)D : orow;
                const double* doi = dout + (t * Hq + h) * (int64_t)D;
                double Di = 0.0;
                for (int d = 0; d < D; ++d) Di += doi[d] * o[d];
                lse_all[t * Hq + h] = lse;
                D_all[t * Hq + h] = Di;
            }
        }
        free(logits);
        free(orow);
    }
    /* Pass 2: each chosen key sums over its query rows in ascending order. */
    if (err == ORACLE_OK) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t idx = 0; idx < nkeys * Hkv; ++idx) {
            int64_t r = idx / Hkv;
            int g = (int)(idx % Hkv);
            int64_t j = keys[r];
            int64_t e = cu_seqlens[doc_of(cu_seqlens, B, j) + 1];
            int64_t hi = (window > 0 && j + window < e) ? j + window : e;
            const double* kj = k + (j * Hkv + g) * (int64_t)D;
            const double* vj = v + (j * Hkv + g) * (int64_t)D;
            double* dkj = dk_rows + (r * Hkv + g) * (int64_t)D;
            double* dvj = dv_rows + (r * Hkv + g) * (int64_t)D;
            for (int d = 0; d < D; ++d) dkj[d] = dvj[d] = 0.0;
            for (int64_t t = j; t < hi; ++t) {
                for (int hh = 0; hh < G; ++hh) {
                    int h = g * G + hh;
                    const double* qi = q + (t * Hq + h) * (int64_t)D;
                    const double* doi = dout + (t * Hq + h) * (int64_t)D;
                    double dot = 0.0, dP = 0.0;
                    for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
                    for (int d = 0; d < D; ++d) dP += doi[d] * vj[d];
                    double P = exp(scale * dot - lse_all[t * Hq + h]);
                    double dS = P * (dP - D_all[t * Hq + h]);
                    for (int d = 0; d < D; ++d) {
                        dkj[d] += scale * dS * qi[d];
                        dvj[d] += P * doi[d];
                    }
                }
            }
        }
    }
    free(need); free(lse_all); free(D_all);
    return err;
}

/* bf16-input wrappers: widen exactly, then run the fp64 definition. */
static double* widen(const uint16_t* src, int64_t n) {
    double* d = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (d) oracle_bf16_to_f64(src, d, n);
    return d;
}

static double* widen_f32(const float* src, int64_t n) {
    double* d = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (d)
        for (int64_t i = 0; i < n; ++i) d[i] = (double)src[i];
    return d;
}

int oracle_fwd_bf16(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                    const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sinks,
                    int window, double scale, double* out, double* lse, int nthreads) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !sinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v)) return ORACLE_ERR_ARG;
    double* qd = widen(q, (int64_t)T * Hq * D);
    double* kd = widen(k, (int64_t)T * Hkv * D);
    double* vd = widen(v, (int64_t)T * Hkv * D);
    double* sd = widen_f32(sinks, Hq);
    int rc = ORACLE_ERR_NOMEM;
    if (qd && kd && vd && sd)
        rc = oracle_fwd_f64(T, Hq, Hkv, D, B, cu_seqlens, qd, kd, vd, sd, window, scale, out, lse, nthreads);
    free(qd); free(kd); free(vd); free(sd);
    return rc;
}

int oracle_fwd_rows_bf16(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                         const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sinks,
                         int window, double scale, const int64_t* rows, int64_t nrows,
                         double* out_rows, double* lse_rows, int nthreads) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !sinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v)) return ORACLE_ERR_ARG;
    double* qd = widen(q, (int64_t)T * Hq * D);
    double* kd = widen(k, (int64_t)T * Hkv * D);
    double* vd = widen(v, (int64_t)T * Hkv * D);
    double* sd = widen_f32(sinks, Hq);
    int rc = ORACLE_ERR_NOMEM;
    if (qd && kd && vd && sd)
        rc = oracle_fwd_rows_f64(T, Hq, Hkv, D, B, cu_seqlens, qd, kd, vd, sd, window, scale, rows, nrows,
                                 out_rows, lse_rows, nthreads);
    free(qd); free(kd); free(vd); free(sd);
    return rc;
}

/* out_for_D_bf16: optional bf16 saved output used for D_i (NULL: the
 * oracle's own fp64 output). */
int oracle_bwd_bf16(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                    const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sinks,
                    int window, double scale, const uint16_t* out_for_D_bf16, const uint16_t* dout,
                    double* dq, double* dk, double* dv, double* dsinks, int nthreads) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !sinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v || !dout)) return ORACLE_ERR_ARG;
    double* qd = widen(q, (int64_t)T * Hq * D);
    double* kd = widen(k, (int64_t)T * Hkv * D);
    double* vd = widen(v, (int64_t)T * Hkv * D);
    double* dod = widen(dout, (int64_t)T * Hq * D);
    double* od = out_for_D_bf16 ? widen(out_for_D_bf16, (int64_t)T * Hq * D) : NULL;
    double* sd = widen_f32(sinks, Hq);
    int rc = ORACLE_ERR_NOMEM;
    if (qd && kd && vd && dod && sd && (od || !out_for_D_bf16))
        rc = oracle_bwd_f64(T, Hq, Hkv, D, B, cu_seqlens, qd, kd, vd, sd, window, scale, od, dod, dq, dk, dv,
                            dsinks, nthreads);
    free(qd); free(kd); free(vd); free(dod); free(od); free(sd);
    return rc;
}

int oracle_bwd_dsinks_bf16(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                           const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sinks,
                           int window, double scale, const uint16_t* out_for_D_bf16, const uint16_t* dout,
                           double* dsinks, int nthreads) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !sinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v || !dout)) return ORACLE_ERR_ARG;
    double* qd = widen(q, (int64_t)T * Hq * D);
    double* kd = widen(k, (int64_t)T * Hkv * D);
    double* vd = widen(v, (int64_t)T * Hkv * D);
    double* dod = widen(dout, (int64_t)T * Hq * D);
    double* od = out_for_D_bf16 ? widen(out_for_D_bf16, (int64_t)T * Hq * D) : NULL;
    double* sd = widen_f32(sinks, Hq);
    int rc = ORACLE_ERR_NOMEM;
    if (qd && kd && vd && dod && sd && (od || !out_for_D_bf16))
        rc = oracle_bwd_dsinks_f64(T, Hq, Hkv, D, B, cu_seqlens, qd, kd, vd, sd, window, scale, od, dod, dsinks,
                                   nthreads);
    free(qd); free(kd); free(vd); free(dod); free(od); free(sd);
    return rc;
}

int oracle_bwd_dq_rows_bf16(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                            const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sinks,
                            int window, double scale, const uint16_t* out_for_D_bf16, const uint16_t* dout,
                            const int64_t* rows, int64_t nrows, double* dq_rows, int nthreads) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !sinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v || !dout)) return ORACLE_ERR_ARG;
    double* qd = widen(q, (int64_t)T * Hq * D);
    double* kd = widen(k, (int64_t)T * Hkv * D);
    double* vd = widen(v, (int64_t)T * Hkv * D);
    double* dod = widen(dout, (int64_t)T * Hq * D);
    double* od = out_for_D_bf16 ? widen(out_for_D_bf16, (int64_t)T * Hq * D) : NULL;
    double* sd = widen_f32(sinks, Hq);
    int rc = ORACLE_ERR_NOMEM;
    if (qd && kd && vd && dod && sd && (od || !out_for_D_bf16))
        rc = oracle_bwd_dq_rows_f64(T, Hq, Hkv, D, B, cu_seqlens, qd, kd, vd, sd, window, scale, od, dod, rows,
                                    nrows, dq_rows, nthreads);
    free(qd); free(kd); free(vd); free(dod); free(od); free(sd);
    return rc;
}

int oracle_bwd_dkv_rows_bf16(int T, int Hq, int Hkv, int D, int B, const int32_t* cu_seqlens,
                             const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sinks,
                             int window, double scale, const uint16_t* out_for_D_bf16, const uint16_t* dout,
                             const int64_t* keys, int64_t nkeys, double* dk_rows, double* dv_rows, int nthreads) {
    if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !sinks) return ORACLE_ERR_ARG;
    if (T > 0 && (!q || !k || !v || !dout)) return ORACLE_ERR_ARG;
    double* qd = widen(q, (int64_t)T * Hq * D);
    double* kd = widen(k, (int64_t)T * Hkv * D);
    double* vd = widen(v, (int64_t)T * Hkv * D);
    double* dod = widen(dout, (int64_t)T * Hq * D);
    double* od = out_for_D_bf16 ? widen(out_for_D_bf16, (int64_t)T * Hq * D) : NULL;
    double* sd = widen_f32(sinks, Hq);
    int rc = ORACLE_ERR_NOMEM;
    if (qd && kd && vd && dod && sd && (od || !out_for_D_bf16))
        rc = oracle_bwd_dkv_rows_f64(T, Hq, Hkv, D, B, cu_seqlens, qd, kd, vd, sd, window, scale, od, dod, keys,
                                     nkeys, dk_rows, dv_rows, nthreads);
    free(qd); free(kd); free(vd); free(dod); free(od); free(sd);
    return rc;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * oracle/attn_ref.c -- plain f64 CPU causal attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle the CUDA kernels are checked
 * against. Only tests/, the smoke check and the bench's CPU-baseline leg may load
 * it; the product library never links or calls it, and it shares no code, header
 * or constant with the CUDA path.
 *
 * What it computes is the plain definition, row by row, with every score row
 * materialised in f64: no tiling, no online softmax, no fusion.
 *
 * Sources (Forge pages):
 *  - mask: key k is visible to query q iff  q - W < k <= q  (W = 0: no window).
 *    Forge ARCHITECTURES.md, "Vague 2" item 8 (sliding_window in the flash kernels
 *    and the reference); W = 0 is the sliding_window(0) default of the config
 *    schema (forge-studio RESEARCH.md, section 2).
 *  - softcap: s -> cap * tanh(s / cap) on the pre-softmax scores, cap = 0 off.
 *    ARCHITECTURES.md "Vague 2" item 9; src/nn/attention.h commit log, "Wave 2
 *    (attention kernels)": attn_softcap, whose backward differentiates through
 *    the tanh exactly.
 *  - GQA: n_heads % n_kv_heads == 0 (config schema validation, RESEARCH.md
 *    section 2). Reading: query head hq uses KV head hq / (Hq / Hkv), i.e. each
 *    KV head serves a contiguous group of query heads.
 *  - softmax (max, sum) per row: ARCHITECTURES.md "Vague 2" item 10 and
 *    "Vague 3" item 12 (the flash kernel keeps the per-row max).
 *  - Reading: the scale multiplies q.k before the cap: s = cap*tanh(scale*q.k/cap).
 *  - Reading: LSE is the natural-log log-sum-exp of the (capped) scores of a row.
 *  - attention sinks: a learned logit per head that joins the softmax
 *    denominator and has no value vector (a per-head bias in the softmax
 *    denominator: ARCHITECTURES.md family table, GPT-OSS row; "Vague 2" item 10,
 *    which seeds the online softmax's (max, sum) with it; SMALL_MODELS_RESEARCH.md
 *    section 2.4). Readings: one logit sigma_h per query head, shared by every
 *    batch entry and row, in the units of the scores the softmax sees (it is
 *    not capped); LSE includes it; its gradient is -sum_i P_i,sink Delta_i.
 *  - max logit: the per-head maximum attention logit that QK-Clip monitors
 *    (ARCHITECTURES.md "Vague 3" item 12; family table, Kimi K2 row). Reading:
 *    per (batch, query head), the maximum over the allowed (i, j) of the score
 *    the softmax sees (after scale and cap), the sink not included.
 *
 * Layouts: q, o, dO, dq are [B][Hq][T][D]; k, v, dk, dv are [B][Hkv][T][D];
 * lse and delta are [B][Hq][T]; all row-major, f64. The _ext functions take
 * the key head dim Dk (q, k, dq, dk) and the value head dim Dv (v, o, dO, dv)
 * separately: d_k != d_v is the decompressed form of multi-head latent
 * attention (ARCHITECTURES.md "Vague 3" item 13 and the family table's DeepSeek
 * V3 row: nope 128 + rope 64 = 192 for q.k, v 128), with the scale chosen by the
 * caller (1/sqrt(192) there).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* first key a query row may see */
static long first_key(long i, long window) {
    if (window > 0 && i - window + 1 > 0) return i - window + 1;
    return 0;
}

static double dot(const double *a, const double *b, int D) {
    double acc = 0.0;
#pragma omp simd reduction(+ : acc)
    for (int d = 0; d < D; d++) acc += a[d] * b[d];
    return acc;
}

/* scaled score before the cap (the argument of tanh when a cap is set) */
static double raw_score(const double *qi, const double *kj, int D, double scale) {
    return scale * dot(qi, kj, D);
}

/* the score the softmax sees */
static double capped(double s, double softcap) {
    return softcap > 0.0 ? softcap * tanh(s / softcap) : s;
}

/* derivative of the cap with respect to its argument: 1 - tanh^2(s/cap) */
static double cap_grad(double s, double softcap) {
    if (softcap <= 0.0) return 1.0;
    double t = tanh(s / softcap);
    return 1.0 - t * t;
}

/*
 * Rounding of an output value to the storage type of the call: 1 = f32
 * (round to nearest even), 2 = bf16 (to f32, then to the 8 significant bits of
 * bf16, round to nearest even on the f32 bit pattern), 0 = none.
 */
static double round_to(double x, int mode) {
    if (mode == 0) return x;
    float f = (float)x;
    if (mode == 1) return (double)f;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) != 0x7f800000u) {
        u += 0x7fffu + ((u >> 16) & 1u);
        u &= 0xffff0000u;
    }
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void oracle_round(const double *x, double *y, long n, int mode) {
    for (long i = 0; i < n; i++) y[i] = round_to(x[i], mode);
}

/*
 * Probabilities of one query row: p[j] for j in [lo, i], returns the LSE.
 * p[j] = exp(s_j - m) / (exp(sink - m) + sum_k exp(s_k - m)), m = the max of the
 * allowed s_k and the sink (sink = -inf: no sink; then exp(sink - m) = 0 and the
 * arithmetic is that of the plain softmax). *smax (may be NULL) receives the
 * max of the s_k alone.
 */
static double row_probs(const double *qi, const double *K, long i, long lo, int D,
                        double scale, double softcap, double sink, double *p, double *smax) {
    double m = -INFINITY;
    for (long j = lo; j <= i; j++) {
        p[j] = capped(raw_score(qi, K + j * D, D, scale), softcap);
        if (p[j] > m) m = p[j];
    }
    if (smax) *smax = m;
    if (sink > m) m = sink;
    double l = exp(sink - m);
    for (long j = lo; j <= i; j++) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    for (long j = lo; j <= i; j++) p[j] /= l;
    return m + log(l);
}

static double sink_of(const double *sink, int hq) { return sink ? sink[hq] : -INFINITY; }

/*
 * Forward: O_i = sum_j P_ij V_j, LSE_i = log (exp(sigma) + sum_j exp(s_ij)).
 * sink [Hq] may be NULL (no sink); max_logit [B][Hq] may be NULL.
 */
void oracle_attn_fwd_ext(const double *q, const double *k, const double *v, const double *sink,
                         double *o, double *lse, double *max_logit, int B, int Hq, int Hkv, int T,
                         int Dk, int Dv, double scale, int window, double softcap) {
    const int G = Hq / Hkv;
    double *rowmax = (double *)malloc(sizeof(double) * (size_t)B * Hq * T);
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
#pragma omp for collapse(3) schedule(dynamic, 8)
        for (int b = 0; b < B; b++)
            for (int hq = 0; hq < Hq; hq++)
                for (int i = 0; i < T; i++) {
                    const int hkv = hq / G;
                    const size_t qrow = ((size_t)(b * Hq + hq) * T + i);
                    const double *qi = q + qrow * Dk;
                    const double *K = k + (size_t)(b * Hkv + hkv) * T * Dk;
                    const double *V = v + (size_t)(b * Hkv + hkv) * T * Dv;
                    const long lo = first_key(i, window);
                    lse[qrow] = row_probs(qi, K, i, lo, Dk, scale, softcap, sink_of(sink, hq), p,
                                          rowmax + qrow);
                    double *oi = o + qrow * Dv;
                    for (int d = 0; d < Dv; d++) oi[d] = 0.0;
                    for (long j = lo; j <= i; j++)
                        for (int d = 0; d < Dv; d++) oi[d] += p[j] * V[j * Dv + d];
                }
        free(p);
    }
    if (max_logit)
        for (long bh = 0; bh < (long)B * Hq; bh++) {
            double m = -INFINITY;
            for (long i = 0; i < T; i++)
                if (rowmax[bh * T + i] > m) m = rowmax[bh * T + i];
            max_logit[bh] = m;
        }
    free(rowmax);
}

/* Forward without sink or max logit. */
void oracle_attn_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
                     int B, int Hq, int Hkv, int T, int D, double scale, int window,
                     double softcap) {
    oracle_attn_fwd_ext(q, k, v, NULL, o, lse, NULL, B, Hq, Hkv, T, D, D, scale, window, softcap);
}

/*
 * Backward of L(O) with upstream gradient dO:
 *   dP_ij  = dO_i . V_j
 *   Delta_i = sum_j P_ij dP_ij
 *   dS_ij  = P_ij (dP_ij - Delta_i) * (1 - tanh^2(S_ij / cap))   [cap factor only if cap > 0]
 *   dQ_i   = scale * sum_j dS_ij K_j
 *   dK_j   = scale * sum over the group's query heads and rows i of dS_ij Q_i
 *   dV_j   =         sum over the group's query heads and rows i of P_ij dO_i
 * Pass 1 walks query rows (P, Delta, dQ); pass 2 walks key rows (dK, dV), using
 * P_ij = exp(s_ij - LSE_i), which is the same softmax entry.
 * delta (may be NULL) receives Delta, lse_out (may be NULL) receives LSE.
 *
 * With a sink (sink [Hq] non-NULL) P and LSE include it, and dsink [Hq] (may be
 * NULL) receives d/d sigma_h = -sum over batches and rows of P_i,sink Delta_i,
 * P_i,sink = exp(sigma_h - LSE_i): the sink's column of the softmax Jacobian,
 * whose upstream dP is 0 (it has no value vector).
 *
 * o_round selects how Delta is formed. 0: Delta_i = sum_j P_ij dP_ij (the
 * definition). 1 or 2: Delta_i = sum_d dO_id * o_id with o_i = sum_j P_ij V_j
 * rounded to the storage type of the call (1 = f32, 2 = bf16): the backward's
 * first step takes rowsum(dO * O) of the O the forward returned, and in a bf16
 * call that O is bf16. With exact O both forms are equal (sum_j P_ij = 1).
 */
void oracle_attn_bwd_ext(const double *q, const double *k, const double *v, const double *dO,
                         const double *sink, double *dq, double *dk, double *dv, double *dsink,
                         double *delta, double *lse_out, int B, int Hq, int Hkv, int T, int Dk,
                         int Dv, double scale, int window, double softcap, int o_round) {
    const int G = Hq / Hkv;
    const size_t nrows = (size_t)B * Hq * T;
    double *lse = (double *)malloc(sizeof(double) * nrows);
    double *dlt = (double *)malloc(sizeof(double) * nrows);

    /* pass 1: query rows */
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
        double *dp = (double *)malloc(sizeof(double) * (size_t)T);
        double *oi = (double *)malloc(sizeof(double) * (size_t)Dv);
#pragma omp for collapse(3) schedule(dynamic, 8)
        for (int b = 0; b < B; b++)
            for (int hq = 0; hq < Hq; hq++)
                for (int i = 0; i < T; i++) {
                    const int hkv = hq / G;
                    const size_t qrow = ((size_t)(b * Hq + hq) * T + i);
                    const double *qi = q + qrow * Dk;
                    const double *doi = dO + qrow * Dv;
                    const double *K = k + (size_t)(b * Hkv + hkv) * T * Dk;
                    const double *V = v + (size_t)(b * Hkv + hkv) * T * Dv;
                    const long lo = first_key(i, window);
                    lse[qrow] = row_probs(qi, K, i, lo, Dk, scale, softcap, sink_of(sink, hq), p, NULL);
                    double dl = 0.0;
                    for (long j = lo; j <= i; j++) {
                        dp[j] = dot(doi, V + j * Dv, Dv);
                        dl += p[j] * dp[j];
                    }
                    if (o_round != 0) {
                        for (int d = 0; d < Dv; d++) oi[d] = 0.0;
                        for (long j = lo; j <= i; j++)
                            for (int d = 0; d < Dv; d++) oi[d] += p[j] * V[j * Dv + d];
                        dl = 0.0;
                        for (int d = 0; d < Dv; d++) dl += doi[d] * round_to(oi[d], o_round);
                    }
                    dlt[qrow] = dl;
                    double *dqi = dq + qrow * Dk;
                    for (int d = 0; d < Dk; d++) dqi[d] = 0.0;
                    for (long j = lo; j <= i; j++) {
                        const double s = raw_score(qi, K + j * Dk, Dk, scale);
                        const double ds = p[j] * (dp[j] - dl) * cap_grad(s, softcap);
                        for (int d = 0; d < Dk; d++) dqi[d] += scale * ds * K[j * Dk + d];
                    }
                }
        free(p);
        free(dp);
        free(oi);
    }

    /* pass 2: key rows, summed over the group's query heads */
#pragma omp parallel for collapse(3) schedule(dynamic, 8)
    for (int b = 0; b < B; b++)
        for (int hkv = 0; hkv < Hkv; hkv++)
            for (int j = 0; j < T; j++) {
                const double *K = k + (size_t)(b * Hkv + hkv) * T * Dk;
                const double *V = v + (size_t)(b * Hkv + hkv) * T * Dv;
                const double *kj = K + (size_t)j * Dk;
                const double *vj = V + (size_t)j * Dv;
                double *dkj = dk + ((size_t)(b * Hkv + hkv) * T + j) * Dk;
                double *dvj = dv + ((size_t)(b * Hkv + hkv) * T + j) * Dv;
                for (int d = 0; d < Dk; d++) dkj[d] = 0.0;
                for (int d = 0; d < Dv; d++) dvj[d] = 0.0;
                long last = T - 1;
                if (window > 0 && (long)j + window - 1 < last) last = (long)j + window - 1;
                for (int g = 0; g < G; g++) {
                    const int hq = hkv * G + g;
                    for (long i = j; i <= last; i++) {
                        const size_t qrow = ((size_t)(b * Hq + hq) * T + i);
                        const double *qi = q + qrow * Dk;
                        const double *doi = dO + qrow * Dv;
                        const double s = raw_score(qi, kj, Dk, scale);
                        const double pij = exp(capped(s, softcap) - lse[qrow]);
                        const double dpij = dot(doi, vj, Dv);
                        const double ds = pij * (dpij - dlt[qrow]) * cap_grad(s, softcap);
                        for (int d = 0; d < Dv; d++) dvj[d] += pij * doi[d];
                        for (int d = 0; d < Dk; d++) dkj[d] += scale * ds * qi[d];
                    }
                }
            }

    if (dsink) {
        for (int hq = 0; hq < Hq; hq++) {
            double acc = 0.0;
            if (sink)
                for (int b = 0; b < B; b++)
                    for (int i = 0; i < T; i++) {
                        const size_t qrow = ((size_t)(b * Hq + hq) * T + i);
                        acc -= exp(sink[hq] - lse[qrow]) * dlt[qrow];
                    }
            dsink[hq] = acc;
        }
    }
    if (delta) memcpy(delta, dlt, sizeof(double) * nrows);
    if (lse_out) memcpy(lse_out, lse, sizeof(double) * nrows);
    free(lse);
    free(dlt);
}

/* Backward without sink. */
void oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                     double *dq, double *dk, double *dv, double *delta, double *lse_out,
                     int B, int Hq, int Hkv, int T, int D, double scale, int window,
                     double softcap, int o_round) {
    oracle_attn_bwd_ext(q, k, v, dO, NULL, dq, dk, dv, NULL, delta, lse_out, B, Hq, Hkv, T, D, D,
                        scale, window, softcap, o_round);
}

/*
 * Decode: one new query per (b, hq) at position len_b - 1 attends the keys of a
 * KV cache (INFERENCE_RESEARCH.md section 2: cache pre-allocated to the maximum
 * length, [layer][head][seq][d] per layer, a dedicated one-query kernel).
 * q, o [B][Hq][D]; k, v [B][Hkv][Tmax][D]; lse [B][Hq]; seq_lens [B] (NULL: every
 * entry has T valid positions). Keys visible: [len - W, len - 1] clipped at 0
 * (W = 0: all len), the same mask as row len - 1 of the forward. sink as in the
 * forward (may be NULL).
 */
void oracle_attn_decode(const double *q, const double *k, const double *v, const double *sink,
                        const int *seq_lens, double *o, double *lse, int B, int Hq, int Hkv, int T,
                        int Tmax, int D, double scale, int window, double softcap) {
    const int G = Hq / Hkv;
    double *p = (double *)malloc(sizeof(double) * (size_t)Tmax);
    for (int b = 0; b < B; b++)
        for (int hq = 0; hq < Hq; hq++) {
            const int hkv = hq / G;
            const long len = seq_lens ? seq_lens[b] : T;
            const long i = len - 1;
            const size_t qrow = (size_t)(b * Hq + hq);
            const double *K = k + (size_t)(b * Hkv + hkv) * Tmax * D;
            const double *V = v + (size_t)(b * Hkv + hkv) * Tmax * D;
            const long lo = first_key(i, window);
            lse[qrow] = row_probs(q + qrow * D, K, i, lo, D, scale, softcap, sink_of(sink, hq), p, NULL);
            double *oi = o + qrow * D;
            for (int d = 0; d < D; d++) oi[d] = 0.0;
            for (long j = lo; j <= i; j++)
                for (int d = 0; d < D; d++) oi[d] += p[j] * V[j * D + d];
        }
    free(p);
}

/* Full probability matrix P [B][Hq][T][T] (zeros where masked); small sizes only. */
void oracle_attn_probs(const double *q, const double *k, double *P, int B, int Hq, int Hkv,
                       int T, int D, double scale, int window, double softcap) {
    const int G = Hq / Hkv;
    for (int b = 0; b < B; b++)
        for (int hq = 0; hq < Hq; hq++)
            for (int i = 0; i < T; i++) {
                const int hkv = hq / G;
                const size_t qrow = ((size_t)(b * Hq + hq) * T + i);
                double *pi = P + qrow * T;
                for (int j = 0; j < T; j++) pi[j] = 0.0;
                row_probs(q + qrow * D, k + (size_t)(b * Hkv + hkv) * T * D, i,
                          first_key(i, window), D, scale, softcap, -INFINITY, pi, NULL);
            }
}

/* Delta_i = sum_d dO_id O_id (the identity the backward's first step relies on). */
void oracle_rowdot(const double *o, const double *dO, double *delta, long rows, int D) {
    for (long r = 0; r < rows; r++) delta[r] = dot(o + r * D, dO + r * D, D);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the parallel loops use from now on (n >= 1), for timing the oracle on
 * one core; returns the count in force afterwards. No effect on the results. */
int oracle_set_num_threads(int n) {
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#endif
    return oracle_num_threads();
}

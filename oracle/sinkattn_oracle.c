/*
 * Float64 CPU oracle for grouped-query attention with a learnable per-head
 * sink logit.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call this file; the CUDA library never does,
 * and the two share no code.
 *
 * What it computes (page "Attention Sink, Learnable Sink and dsink",
 * notes.kuangjux.top, sections 1, 4, 7 and 8):
 *
 *   x_ijh = alpha * <Q_ih, K_j,g(h)>            for j in the visible set A_ih
 *   the sink is an extra softmax column with logit a_h and a zero value row;
 *   it is NOT scaled by alpha (section 7, second pitfall).
 *   M    = max(max_j x_ijh, a_h)
 *   den  = sum_j e^(x_ijh - M) + e^(a_h - M)
 *   Phat = e^(x - M) / den ;  p_sink = e^(a_h - M) / den
 *   O_ih = sum_j Phat_ij V_j,g(h)
 *   LSE_new = M + log(den)            (natural log; includes the sink)
 *   sink_s  = sum_j Phat_ij           (total mass on real tokens)
 *
 * The sink sits explicitly in the denominator here; nothing uses the
 * "plain attention, then scale by s" shortcut of section 4.
 *
 * Backward is the explicit Jacobian of the augmented softmax (independent of
 * the dsink closed form of section 7):
 *   dPhat_j = <dO_ih, V_j> (+ dss_ih, an optional upstream gradient of
 *             sink_s = sum_j Phat_j; page "Attention Sink and the native MoE
 *             in attention layers", section 5, trains through the gate)
 *   dPhat_sink = 0 (zero value row)
 *   mu      = sum_{j and sink} Phat dPhat          (equals Delta of section 7)
 *   dx_j    = Phat_j (dPhat_j - mu)
 *   da_h   += p_sink (0 - mu)
 *   dQ_ih  += alpha sum_j dx_j K_j ; dK_j += alpha dx_j Q_ih ; dV_j += Phat_j dO_ih
 *
 * Visible set (section 2: block selection, window, causality and sample
 * boundaries all restrict it), by brute force for every (i, j, h):
 *   same sequence; with sequence-local qi, kj:
 *   causal      => kj <= qi
 *   window > 0  => kj < n_sink  or  qi - kj < window
 *   block_indices != NULL => floor(kj / block_k) is listed in
 *       BI[g(h)][qblock(i)] where qblock numbers the sequence-local query
 *       blocks floor(qi / block_q) globally in sequence order.
 *   g(h) = floor(h / (Hq / Hkv)).
 *
 * Ring-buffer decode (StreamingLLM KV set: a fixed sink segment plus a
 * sliding window; page "Attention Sink / StreamingLLM" interview notes): a
 * token at absolute position p < n_sink sits in slot p, a token at
 * p >= n_sink sits in slot n_sink + (p - n_sink) mod window; with n tokens
 * appended the visible positions are [0, min(n_sink, n)) and
 * [max(n_sink, n - window), n).
 *
 * Empty visible set with no sink: O = 0, LSE = -inf, sink_s = 0, and the
 * backward gives zero gradients for that row.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int T_tot, Hq, Hkv, D;
    double scale;
    int causal, n_sink, window;
    const int32_t *cu_seqlens; /* [n_seq + 1] host; NULL => uniform seqlen */
    int n_seq, seqlen;
    const int32_t *block_indices; /* [Hkv, n_qblk_total, max_blocks] or NULL */
    int block_q, block_k, max_blocks;
} om_problem;

/* --- sequence bookkeeping ------------------------------------------------ */

static int seq_start(const om_problem *p, int s) {
    return p->cu_seqlens ? p->cu_seqlens[s] : s * p->seqlen;
}
static int seq_end(const om_problem *p, int s) {
    return p->cu_seqlens ? p->cu_seqlens[s + 1] : (s + 1) * p->seqlen;
}
static int seq_of(const om_problem *p, int i) {
    for (int s = 0; s < p->n_seq; ++s)
        if (i < seq_end(p, s)) return s;
    return -1;
}
/* first global query-block number of sequence s */
static int qblk_base(const om_problem *p, int s) {
    int b = 0;
    for (int t = 0; t < s; ++t) {
        int len = seq_end(p, t) - seq_start(p, t);
        b += (len + p->block_q - 1) / p->block_q;
    }
    return b;
}
static int n_qblk_total(const om_problem *p) { return qblk_base(p, p->n_seq); }

/* Is key j visible to query i for KV head g?  The plain predicate. */
static int visible(const om_problem *p, int i, int j, int g) {
    int s = seq_of(p, i);
    if (s < 0 || s != seq_of(p, j)) return 0;
    int st = seq_start(p, s);
    int qi = i - st, kj = j - st;
    if (p->causal && kj > qi) return 0;
    if (p->window > 0 && !(kj < p->n_sink || qi - kj < p->window)) return 0;
    if (p->block_indices) {
        int qb = qblk_base(p, s) + qi / p->block_q;
        int kb = kj / p->block_k;
        const int32_t *row =
            p->block_indices + ((size_t)g * n_qblk_total(p) + qb) * p->max_blocks;
        int found = 0;
        for (int t = 0; t < p->max_blocks; ++t)
            if (row[t] == kb) found = 1;
        if (!found) return 0;
    }
    return 1;
}

static double dot(const double *a, const double *b, int D) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

/* Per-row forward quantities. */
typedef struct {
    double M, den, lse, sink_s, p_sink;
    int n_vis;
} om_rowstat;

/* Forward for one (i, h): fills o_row[D] and the row statistics.  js/xs
 * (capacity: the sequence length) receive the visible keys and their scores
 * x_ij, in key order, so the backward can reuse them. */
static void row_forward(const om_problem *p, const double *q, const double *k,
                        const double *v, const double *sink, int i, int h,
                        double *o_row, om_rowstat *st, int *js, double *xs) {
    const int D = p->D, G = p->Hq / p->Hkv, g = h / G;
    const double *qrow = q + ((size_t)i * p->Hq + h) * D;
    int s = seq_of(p, i);
    int j0 = seq_start(p, s), j1 = seq_end(p, s);
    /* scores of the visible keys and the maximum over the augmented set */
    double M = -INFINITY;
    int n_vis = 0;
    for (int j = j0; j < j1; ++j) {
        if (!visible(p, i, j, g)) continue;
        double x = p->scale * dot(qrow, k + ((size_t)j * p->Hkv + g) * D, D);
        js[n_vis] = j;
        xs[n_vis] = x;
        if (x > M) M = x;
        ++n_vis;
    }
    if (sink && sink[h] > M) M = sink[h];
    for (int d = 0; d < D; ++d) o_row[d] = 0.0;
    st->n_vis = n_vis;
    if (M == -INFINITY) { /* nothing visible and no sink */
        st->M = -INFINITY; st->den = 0.0; st->lse = -INFINITY;
        st->sink_s = 0.0; st->p_sink = 0.0;
        return;
    }
    /* denominator including the sink column e^(a_h - M) */
    double den = 0.0;
    for (int t = 0; t < n_vis; ++t) den += exp(xs[t] - M);
    if (sink) den += exp(sink[h] - M);
    /* probabilities and output */
    double mass = 0.0;
    for (int t = 0; t < n_vis; ++t) {
        double P = exp(xs[t] - M) / den;
        mass += P;
        const double *vrow = v + ((size_t)js[t] * p->Hkv + g) * D;
        for (int d = 0; d < D; ++d) o_row[d] += P * vrow[d];
    }
    st->M = M;
    st->den = den;
    st->lse = M + log(den);
    st->sink_s = mass;
    st->p_sink = sink ? exp(sink[h] - M) / den : 0.0;
}

static int max_seq_len(int T_tot, const int32_t *cu, int n_seq, int seqlen) {
    if (!cu) return seqlen;
    int m = 0;
    for (int s = 0; s < n_seq; ++s)
        if (cu[s + 1] - cu[s] > m) m = cu[s + 1] - cu[s];
    (void)T_tot;
    return m;
}

static om_problem make_problem(int T_tot, int Hq, int Hkv, int D, double scale,
                               int causal, int n_sink, int window,
                               const int32_t *cu_seqlens, int n_seq, int seqlen,
                               const int32_t *block_indices, int block_q,
                               int block_k, int max_blocks) {
    om_problem p;
    p.T_tot = T_tot; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.scale = scale;
    p.causal = causal; p.n_sink = n_sink; p.window = window;
    p.cu_seqlens = cu_seqlens; p.n_seq = n_seq; p.seqlen = seqlen;
    p.block_indices = block_indices; p.block_q = block_q > 0 ? block_q : 64;
    p.block_k = block_k > 0 ? block_k : 64; p.max_blocks = max_blocks;
    return p;
}

#define OM_PROBLEM_ARGS                                                        \
    int T_tot, int Hq, int Hkv, int D, double scale, int causal, int n_sink,  \
        int window, const int32_t *cu_seqlens, int n_seq, int seqlen,          \
        const int32_t *block_indices, int block_q, int block_k, int max_blocks
#define OM_PROBLEM_PASS                                                        \
    T_tot, Hq, Hkv, D, scale, causal, n_sink, window, cu_seqlens, n_seq,       \
        seqlen, block_indices, block_q, block_k, max_blocks

/* Dense visibility of one KV head: vis[i * T_tot + j] = 1 if visible. */
int oracle_visible_dense(OM_PROBLEM_ARGS, int g, uint8_t *vis) {
    om_problem p = make_problem(OM_PROBLEM_PASS);
    for (int i = 0; i < T_tot; ++i)
        for (int j = 0; j < T_tot; ++j)
            vis[(size_t)i * T_tot + j] = (uint8_t)visible(&p, i, j, g);
    return 0;
}

/* Full forward: out [T,Hq,D], lse [T,Hq], sink_s [T,Hq]. sink may be NULL. */
int oracle_fwd(OM_PROBLEM_ARGS, const double *q, const double *k,
               const double *v, const double *sink, double *out, double *lse,
               double *sink_s) {
    om_problem p = make_problem(OM_PROBLEM_PASS);
    const int L = max_seq_len(T_tot, cu_seqlens, n_seq, seqlen);
#pragma omp parallel
    {
        int *js = (int *)malloc(sizeof(int) * (size_t)L);
        double *xs = (double *)malloc(sizeof(double) * (size_t)L);
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < (long)T_tot * Hq; ++r) {
            int i = (int)(r / Hq), h = (int)(r % Hq);
            om_rowstat st;
            row_forward(&p, q, k, v, sink, i, h, out + (size_t)r * D, &st, js, xs);
            lse[r] = st.lse;
            sink_s[r] = st.sink_s;
        }
        free(js); free(xs);
    }
    return 0;
}

/* Forward of selected rows only: rows[2*n] = (i, h). */
int oracle_fwd_rows(OM_PROBLEM_ARGS, const double *q, const double *k,
                    const double *v, const double *sink, int n_rows,
                    const int32_t *rows, double *out, double *lse,
                    double *sink_s) {
    om_problem p = make_problem(OM_PROBLEM_PASS);
    const int L = max_seq_len(T_tot, cu_seqlens, n_seq, seqlen);
#pragma omp parallel
    {
        int *js = (int *)malloc(sizeof(int) * (size_t)L);
        double *xs = (double *)malloc(sizeof(double) * (size_t)L);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n_rows; ++r) {
            om_rowstat st;
            row_forward(&p, q, k, v, sink, rows[2 * r], rows[2 * r + 1],
                        out + (size_t)r * D, &st, js, xs);
            lse[r] = st.lse;
            sink_s[r] = st.sink_s;
        }
        free(js); free(xs);
    }
    return 0;
}

/* Full backward: dq [T,Hq,D], dk/dv [T,Hkv,D], dsink [Hq] (if sink != NULL).
 * dout is the upstream gradient dL/dO; dss [T,Hq] (or NULL) that of sink_s.
 * Two plain phases:
 *   1. per row (i, h): forward statistics, mu = sum Phat dPhat, and dQ;
 *   2. per key (j, g): dK, dV summed over every (row, head of group g) that
 *      sees the key, with the row's Phat recomputed from its statistics. */
int oracle_bwd(OM_PROBLEM_ARGS, const double *q, const double *k,
               const double *v, const double *sink, const double *dout,
               const double *dss, double *dq, double *dk, double *dv, double *dsink) {
    om_problem p = make_problem(OM_PROBLEM_PASS);
    const int G = Hq / Hkv;
    const long R = (long)T_tot * Hq;
    const int L = max_seq_len(T_tot, cu_seqlens, n_seq, seqlen);
    om_rowstat *st = (om_rowstat *)malloc(sizeof(om_rowstat) * (size_t)R);
    double *mu = (double *)malloc(sizeof(double) * (size_t)R);
    if (!st || !mu) { free(st); free(mu); return 1; }

#pragma omp parallel
    {
        int *js = (int *)malloc(sizeof(int) * (size_t)L);
        double *xs = (double *)malloc(sizeof(double) * (size_t)L);
        double *o_row = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < R; ++r) {
            int i = (int)(r / Hq), h = (int)(r % Hq), g = h / G;
            row_forward(&p, q, k, v, sink, i, h, o_row, &st[r], js, xs);
            const double *dorow = dout + (size_t)r * D;
            double *dqrow = dq + (size_t)r * D;
            for (int d = 0; d < D; ++d) dqrow[d] = 0.0;
            mu[r] = 0.0;
            if (st[r].M == -INFINITY) continue;
            /* an upstream gradient of sink_s = sum_j Phat_j (the real-token
             * mass) adds dss to every real key's dPhat */
            const double gs = dss ? dss[r] : 0.0;
            /* mu = sum_j Phat_j dPhat_j + p_sink * 0 */
            double m = 0.0;
            for (int t = 0; t < st[r].n_vis; ++t) {
                double P = exp(xs[t] - st[r].M) / st[r].den;
                m += P * (dot(dorow, v + ((size_t)js[t] * Hkv + g) * D, D) + gs);
            }
            mu[r] = m;
            for (int t = 0; t < st[r].n_vis; ++t) {
                const double *krow = k + ((size_t)js[t] * Hkv + g) * D;
                double P = exp(xs[t] - st[r].M) / st[r].den;
                double dx = P * (dot(dorow, v + ((size_t)js[t] * Hkv + g) * D, D) + gs - m);
                for (int d = 0; d < D; ++d) dqrow[d] += scale * dx * krow[d];
            }
        }
        free(js); free(xs); free(o_row);
    }

#pragma omp parallel for schedule(dynamic, 4)
    for (long c = 0; c < (long)T_tot * Hkv; ++c) {
        int j = (int)(c / Hkv), g = (int)(c % Hkv);
        double *dkrow = dk + (size_t)c * D, *dvrow = dv + (size_t)c * D;
        for (int d = 0; d < D; ++d) { dkrow[d] = 0.0; dvrow[d] = 0.0; }
        int s = seq_of(&p, j);
        const double *krow = k + (size_t)c * D, *vrow = v + (size_t)c * D;
        for (int i = seq_start(&p, s); i < seq_end(&p, s); ++i) {
            if (!visible(&p, i, j, g)) continue;
            for (int h = g * G; h < (g + 1) * G; ++h) {
                long r = (long)i * Hq + h;
                if (st[r].M == -INFINITY) continue;
                const double *qrow = q + (size_t)r * D, *dorow = dout + (size_t)r * D;
                double x = scale * dot(qrow, krow, D);
                double P = exp(x - st[r].M) / st[r].den;
                double dx = P * (dot(dorow, vrow, D) + (dss ? dss[r] : 0.0) - mu[r]);
                for (int d = 0; d < D; ++d) {
                    dkrow[d] += scale * dx * qrow[d];
                    dvrow[d] += P * dorow[d];
                }
            }
        }
    }

    if (sink && dsink) {
        for (int h = 0; h < Hq; ++h) dsink[h] = 0.0;
        for (long r = 0; r < R; ++r) /* da_h += p_sink (0 - mu), all queries */
            dsink[r % Hq] += st[r].p_sink * (0.0 - mu[r]);
    }
    free(st); free(mu);
    return 0;
}

/* Backward on samples of a large problem: dQ of selected rows (i, h) and
 * dK / dV of selected keys (j, g), each from the same explicit Jacobian as
 * oracle_bwd.  A key's gradient needs the statistics (M, den, mu) of every
 * row that sees it, so phase 1 computes them for every row of the KV heads
 * the sampled keys belong to; phase 2 sums over those rows key by key. */
int oracle_bwd_sampled(OM_PROBLEM_ARGS, const double *q, const double *k,
                       const double *v, const double *sink, const double *dout,
                       int n_rows, const int32_t *rows, double *dq_rows,
                       int n_keys, const int32_t *keys, double *dk_keys,
                       double *dv_keys) {
    om_problem p = make_problem(OM_PROBLEM_PASS);
    const int G = Hq / Hkv;
    const int L = max_seq_len(T_tot, cu_seqlens, n_seq, seqlen);
    /* dQ rows */
#pragma omp parallel
    {
        int *js = (int *)malloc(sizeof(int) * (size_t)L);
        double *xs = (double *)malloc(sizeof(double) * (size_t)L);
        double *o_row = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n_rows; ++r) {
            int i = rows[2 * r], h = rows[2 * r + 1], g = h / G;
            om_rowstat st;
            row_forward(&p, q, k, v, sink, i, h, o_row, &st, js, xs);
            double *dqrow = dq_rows + (size_t)r * D;
            for (int d = 0; d < D; ++d) dqrow[d] = 0.0;
            if (st.M == -INFINITY) continue;
            const double *dorow = dout + ((size_t)i * Hq + h) * D;
            double m = 0.0;
            for (int t = 0; t < st.n_vis; ++t)
                m += exp(xs[t] - st.M) / st.den * dot(dorow, v + ((size_t)js[t] * Hkv + g) * D, D);
            for (int t = 0; t < st.n_vis; ++t) {
                const double *krow = k + ((size_t)js[t] * Hkv + g) * D;
                double P = exp(xs[t] - st.M) / st.den;
                double dx = P * (dot(dorow, v + ((size_t)js[t] * Hkv + g) * D, D) - m);
                for (int d = 0; d < D; ++d) dqrow[d] += scale * dx * krow[d];
            }
        }
        free(js); free(xs); free(o_row);
    }
    if (n_keys <= 0) return 0;
    /* phase 1: statistics of every row of the involved KV heads */
    const long long R = (long long)T_tot * Hq;
    om_rowstat *st = (om_rowstat *)malloc(sizeof(om_rowstat) * (size_t)R);
    double *mu = (double *)malloc(sizeof(double) * (size_t)R);
    uint8_t *need = (uint8_t *)calloc((size_t)Hkv, 1);
    if (!st || !mu || !need) { free(st); free(mu); free(need); return 1; }
    for (int c = 0; c < n_keys; ++c) need[keys[2 * c + 1]] = 1;
#pragma omp parallel
    {
        int *js = (int *)malloc(sizeof(int) * (size_t)L);
        double *xs = (double *)malloc(sizeof(double) * (size_t)L);
        double *o_row = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < R; ++r) {
            int i = (int)(r / Hq), h = (int)(r % Hq), g = h / G;
            mu[r] = 0.0;
            st[r].M = -INFINITY;
            if (!need[g]) continue;
            row_forward(&p, q, k, v, sink, i, h, o_row, &st[r], js, xs);
            if (st[r].M == -INFINITY) continue;
            const double *dorow = dout + (size_t)r * D;
            double m = 0.0;
            for (int t = 0; t < st[r].n_vis; ++t)
                m += exp(xs[t] - st[r].M) / st[r].den *
                     dot(dorow, v + ((size_t)js[t] * Hkv + g) * D, D);
            mu[r] = m;
        }
        free(js); free(xs); free(o_row);
    }
    /* phase 2: per sampled key */
#pragma omp parallel for schedule(dynamic, 1)
    for (int c = 0; c < n_keys; ++c) {
        int j = keys[2 * c], g = keys[2 * c + 1];
        double *dkrow = dk_keys + (size_t)c * D, *dvrow = dv_keys + (size_t)c * D;
        for (int d = 0; d < D; ++d) { dkrow[d] = 0.0; dvrow[d] = 0.0; }
        int s = seq_of(&p, j);
        const double *krow = k + ((size_t)j * Hkv + g) * D;
        const double *vrow = v + ((size_t)j * Hkv + g) * D;
        for (int i = seq_start(&p, s); i < seq_end(&p, s); ++i) {
            if (!visible(&p, i, j, g)) continue;
            for (int h = g * G; h < (g + 1) * G; ++h) {
                long r = (long)i * Hq + h;
                if (st[r].M == -INFINITY) continue;
                const double *qrow = q + (size_t)r * D, *dorow = dout + (size_t)r * D;
                double P = exp(scale * dot(qrow, krow, D) - st[r].M) / st[r].den;
                double dx = P * (dot(dorow, vrow, D) - mu[r]);
                for (int d = 0; d < D; ++d) {
                    dkrow[d] += scale * dx * qrow[d];
                    dvrow[d] += P * dorow[d];
                }
            }
        }
    }
    free(st); free(mu); free(need);
    return 0;
}

/* Ring-buffer decode.  q [B,Hq,D]; caches [B,S,Hkv,D] with S = n_sink+window;
 * cache_seqlens[b] = tokens ever appended (current token included). */
int oracle_decode(int B, int Hq, int Hkv, int D, double scale,
                  const double *q, const double *k_cache,
                  const double *v_cache, const int32_t *cache_seqlens,
                  int n_sink, int window, const double *sink, double *out,
                  double *lse, double *sink_s) {
    const int S = n_sink + window, G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < (long)B * Hq; ++r) {
        int b = (int)(r / Hq), h = (int)(r % Hq), g = h / G;
        long n = cache_seqlens[b];
        const double *qrow = q + (size_t)r * D;
        double *orow = out + (size_t)r * D;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        /* logical positions in time order: sink segment, then the window */
        long lo_win = n - window > n_sink ? n - window : n_sink;
        long n_pos = (n < n_sink ? n : n_sink) + (n > lo_win ? n - lo_win : 0);
        long *slot = (long *)malloc(sizeof(long) * (size_t)(n_pos > 0 ? n_pos : 1));
        long c = 0;
        for (long pos = 0; pos < n && pos < n_sink; ++pos) slot[c++] = pos;
        for (long pos = lo_win; pos < n; ++pos)
            slot[c++] = n_sink + (pos - n_sink) % window;
        double M = -INFINITY;
        for (long t = 0; t < c; ++t) {
            const double *krow = k_cache + (((size_t)b * S + slot[t]) * Hkv + g) * D;
            double x = scale * dot(qrow, krow, D);
            if (x > M) M = x;
        }
        if (sink && sink[h] > M) M = sink[h];
        if (M == -INFINITY) {
            lse[r] = -INFINITY; sink_s[r] = 0.0; free(slot); continue;
        }
        double den = 0.0;
        for (long t = 0; t < c; ++t) {
            const double *krow = k_cache + (((size_t)b * S + slot[t]) * Hkv + g) * D;
            den += exp(scale * dot(qrow, krow, D) - M);
        }
        if (sink) den += exp(sink[h] - M);
        double mass = 0.0;
        for (long t = 0; t < c; ++t) {
            const double *krow = k_cache + (((size_t)b * S + slot[t]) * Hkv + g) * D;
            const double *vrow = v_cache + (((size_t)b * S + slot[t]) * Hkv + g) * D;
            double P = exp(scale * dot(qrow, krow, D) - M) / den;
            mass += P;
            for (int d = 0; d < D; ++d) orow[d] += P * vrow[d];
        }
        lse[r] = M + log(den);
        sink_s[r] = mass;
        free(slot);
    }
    return 0;
}

/* Tile enumeration by brute force, for checking the GPU tile schedule.
 * A query tile is tile_q consecutive sequence-local tokens (the last one of a
 * sequence may be short); a key tile is tile_k consecutive sequence-local
 * keys.  For every (KV head g, query tile) in sequence order and every key
 * tile of the same sequence, state[...] = 0 if no pair (i, j) with i a valid
 * row of the query tile and j a valid key of the key tile is visible;
 * 1 if some but not all of the tile_q x tile_k positions are visible pairs
 * (positions past the end of the sequence count as not visible); 2 if all
 * are.  Output layout: state[g][qtile_global][ktile_local], with
 * ktile_local < max_ktiles (= ceil(max_seqlen / tile_k)).
 * Returns the number of query tiles. */
int oracle_tile_states(OM_PROBLEM_ARGS, int tile_q, int tile_k, int max_ktiles,
                       uint8_t *state) {
    om_problem p = make_problem(OM_PROBLEM_PASS);
    int nqt = 0;
    for (int s = 0; s < n_seq; ++s)
        nqt += (seq_end(&p, s) - seq_start(&p, s) + tile_q - 1) / tile_q;
    for (int g = 0; g < Hkv; ++g) {
        int qt = 0;
        for (int s = 0; s < n_seq; ++s) {
            int st = seq_start(&p, s), len = seq_end(&p, s) - st;
            for (int q0 = 0; q0 < len; q0 += tile_q, ++qt) {
                for (int kt = 0; kt < max_ktiles; ++kt) {
                    int k0 = kt * tile_k;
                    int any = 0, all = 1;
                    for (int a = 0; a < tile_q; ++a)
                        for (int b = 0; b < tile_k; ++b) {
                            int qi = q0 + a, kj = k0 + b;
                            int vis = (qi < len && kj < len)
                                          ? visible(&p, st + qi, st + kj, g) : 0;
                            if (vis) any = 1; else if (qi < len) all = 0;
                        }
                    /* rows past the sequence end are not part of the tile's
                       validity; keys past the end make the tile partial */
                    uint8_t v = any ? (all ? 2 : 1) : 0;
                    state[((size_t)g * nqt + qt) * max_ktiles + kt] = v;
                }
            }
        }
    }
    return nqt;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

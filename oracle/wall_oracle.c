/*
 * wall_oracle.c -- plain fp64 CPU oracle for Wall Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this file's library.  The
 * CUDA product path shares no code with it and never calls it.
 *
 * What it computes, and where the pages define it:
 *   - Wall score (Tilde blog "Wall Attention", section "Definition: Wall
 *     Attention"; wall-attention-release README, introduction):
 *         o_i = sum_j softmax_j( scale * sum_n F_ij,n q_i,n k_j,n ) v_j,
 *         F_ij,n = prod_{r=j+1..i} exp(g_r,n)        (causal, j <= i)
 *     with `g` read as the natural log of the per-channel gate, so g = 0
 *     is vanilla softmax attention (README introduction).
 *   - Optional arguments (README "Usage", optional arguments): a FoX-style
 *     scalar log-gate g_scalar [T,HQ] adding sum_{r=j+1..i} gs_r to the
 *     logit outside the scale (Tilde blog, FoX formula exp(q^T k + log F)),
 *     an attention-sink logit sink[h] with a zero value row, a sliding
 *     window (key visible iff 0 <= i-j < W), varlen packing via cu_seqlens,
 *     and GQA with query head h reading kv head h / (HQ/H).
 *   - Prefix form (Tilde blog, factorised form): P_t = sum_{u<=t} log g_u,
 *     F_ij = exp(L_i - L_j).  Implemented as the second, independent form.
 *   - Base-2 prefix P = cumsum(g) / ln 2 (README "Decode": the cumulative
 *     sum is taken with scale 1/ln 2).
 *   - Analytic backward: chain rule of the definition above.  The gate
 *     gradient is taken through the natural-log prefix L_t = sum_{u<=t} g_u:
 *     dL_i += c_ij and dL_j -= c_ij for every visible pair, with
 *     c_ij,n = scale * dS_ij * q_i,n k_j,n F_ij,n, then dg_u = sum_{t>=u} dL_t
 *     within the sequence.  (The blog's section on fast training prints only
 *     the key-side half, dP_j = -ln2 * K_j (.) dK_j.)
 *
 * Layout: every array is fp64, row-major, rows flattened over batch*time:
 * q [TT,HQ,K], k [TT,H,K], v [TT,H,V], g [TT,HQ,K], gs [TT,HQ], sink [HQ].
 * Sequences are given by cu [nseq+1] row offsets into the TT rows, so a
 * dense [B,T] batch is cu = {0, T, 2T, ..., BT}.  A "unit" is one
 * (sequence, query head) pair, u = seq * HQ + h; units are independent and
 * are spread over worker threads.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>

/* Deliberate-mistake switch used only by the tests that show the pins catch
 * plausible oracle bugs.  0 = the correct oracle. */
static int g_mutation = 0;
void wo_set_mutation(int m) { g_mutation = m; }
int wo_get_mutation(void) { return g_mutation; }

enum {
    MUT_NONE = 0,
    MUT_PRODUCT_RANGE = 1,   /* product over r = j..i instead of j+1..i   */
    MUT_DROP_KEY_DL = 2,     /* drop the key-side term of the gate grad    */
    MUT_SIGN_QUERY_DL = 3,   /* wrong sign on the query-side gate term     */
    MUT_GQA_MAP = 4,         /* kv head h % H instead of h / (HQ/H)        */
    MUT_DV_ROW = 5,          /* dv_j += p_ij dO_j instead of p_ij dO_i     */
    MUT_WINDOW = 6,          /* visible iff i-j <= W instead of i-j < W    */
    MUT_SINK_LSE = 7,        /* sink left out of the normaliser            */
    MUT_SCALE_BIAS = 8,      /* scale applied to the scalar-gate bias too  */
    MUT_PREFIX_BASE = 9,     /* base-2 prefix without the 1/ln2 factor     */
};

typedef struct {
    const double *q, *k, *v, *g, *gs, *sink, *dO;
    long TT;
    int H, HQ, K, V;
    double scale;
    long window;
    const long* cu;
    int nseq;
    int form;              /* 0: cumulative product, 1: prefix difference */
    const int* units;      /* NULL: all nseq*HQ units */
    int n_units;
    long row_lo, row_hi;   /* rows relative to sequence start; hi < 0 = all */
    long q_rows;           /* > 0: q holds only rows [row_lo, row_lo+q_rows) of
                              each sequence, as [nseq, q_rows, HQ, K] */
    /* forward outputs */
    double *o, *lse;
    /* backward outputs (per query head; dk/dv before the GQA reduction) */
    double *dq, *dkh, *dvh, *dg, *dgs, *dsink;
    atomic_int next;
    int backward;
} job_t;

/* Per-unit tables for one (sequence, query head): rows are relative to the
 * sequence start.  E = exp(g) for the product form; L (natural-log prefix)
 * and GS (prefix of the scalar gate) for the prefix form. */
typedef struct {
    int seq, h, kh;
    long s0, len;
    double *E, *L, *GS;
} unit_t;

static int kv_head(const job_t* J, int h) {
    int G = J->HQ / J->H;
    if (g_mutation == MUT_GQA_MAP) return h % J->H;
    return h / G;
}

static long first_visible(const job_t* J, long i) {
    if (J->window <= 0) return 0;
    long W = J->window;
    if (g_mutation == MUT_WINDOW) W += 1;
    long j0 = i - W + 1;
    return j0 < 0 ? 0 : j0;
}

static void unit_tables(const job_t* J, unit_t* U) {
    const int HQ = J->HQ, K = J->K, h = U->h;
    for (long t = 0; t < U->len; ++t) {
        const double* gt = J->g + ((U->s0 + t) * HQ + h) * K;
        for (int n = 0; n < K; ++n) U->E[t * K + n] = exp(gt[n]);
    }
    if (J->form == 1) {
        for (int n = 0; n < K; ++n) {
            double acc = 0.0;
            for (long t = 0; t < U->len; ++t) {
                acc += J->g[((U->s0 + t) * HQ + h) * K + n];
                U->L[t * K + n] = acc;
            }
        }
        double acc = 0.0;
        for (long t = 0; t < U->len; ++t) {
            if (J->gs) acc += J->gs[(U->s0 + t) * HQ + h];
            U->GS[t] = acc;
        }
    }
}

/* Logits of row i against keys j = i, i-1, ..., jmin, written to sc[i-j].
 * F is scratch of K doubles; Fmat (if not NULL) receives the per-channel
 * decay F_ij,n at Fmat[(i-j)*K + n]. */
static void row_logits(const job_t* J, const unit_t* U, long i, long jmin,
                       double* sc, double* F, double* Fmat) {
    const int K = J->K, HQ = J->HQ, H = J->H;
    const long qrow = J->q_rows > 0 ? (long)U->seq * J->q_rows + (i - J->row_lo) : U->s0 + i;
    const double* qi = J->q + (qrow * HQ + U->h) * K;
    double bias = 0.0;
    for (int n = 0; n < K; ++n) F[n] = 1.0;
    for (long j = i; j >= jmin; --j) {
        if (J->form == 0) {
            /* step the product from r = j+2..i to r = j+1..i */
            if (j < i) {
                const double* e = U->E + (j + 1) * K;
                for (int n = 0; n < K; ++n) F[n] *= e[n];
                if (J->gs) bias += J->gs[(U->s0 + j + 1) * HQ + U->h];
            }
        } else {
            const double* Li = U->L + i * K;
            const double* Lj = U->L + j * K;
            for (int n = 0; n < K; ++n) F[n] = exp(Li[n] - Lj[n]);
            if (J->gs) bias = U->GS[i] - U->GS[j];
        }
        const double* kj = J->k + ((U->s0 + j) * H + U->kh) * K;
        if (g_mutation == MUT_PRODUCT_RANGE) {
            const double* e = U->E + j * K;
            double dot = 0.0;
            for (int n = 0; n < K; ++n) dot += qi[n] * kj[n] * F[n] * e[n];
            if (Fmat) for (int n = 0; n < K; ++n) Fmat[(i - j) * K + n] = F[n] * e[n];
            sc[i - j] = J->scale * dot + bias;
            continue;
        }
        double dot = 0.0;
        for (int n = 0; n < K; ++n) dot += qi[n] * kj[n] * F[n];
        if (Fmat) memcpy(Fmat + (i - j) * K, F, sizeof(double) * K);
        double s = J->scale * dot;
        s += (g_mutation == MUT_SCALE_BIAS) ? J->scale * bias : bias;
        sc[i - j] = s;
    }
}

/* log-sum-exp of the row's logits plus the optional sink logit */
static double row_lse(const job_t* J, int h, const double* sc, long n) {
    double m = -INFINITY;
    for (long c = 0; c < n; ++c) m = sc[c] > m ? sc[c] : m;
    int with_sink = J->sink && g_mutation != MUT_SINK_LSE;
    if (with_sink && J->sink[h] > m) m = J->sink[h];
    double l = 0.0;
    for (long c = 0; c < n; ++c) l += exp(sc[c] - m);
    if (with_sink) l += exp(J->sink[h] - m);
    return m + log(l);
}

static void fwd_unit(job_t* J, const unit_t* U, double* sc, double* F) {
    const int HQ = J->HQ, H = J->H, V = J->V;
    long lo = J->row_lo < 0 ? 0 : J->row_lo;
    long hi = (J->row_hi < 0 || J->row_hi > U->len) ? U->len : J->row_hi;
    for (long i = lo; i < hi; ++i) {
        long jmin = first_visible(J, i);
        row_logits(J, U, i, jmin, sc, F, NULL);
        double lse = row_lse(J, U->h, sc, i - jmin + 1);
        double* oi = J->o + ((U->s0 + i) * HQ + U->h) * V;
        for (int c = 0; c < V; ++c) oi[c] = 0.0;
        for (long j = i; j >= jmin; --j) {
            double p = exp(sc[i - j] - lse);
            const double* vj = J->v + ((U->s0 + j) * H + U->kh) * V;
            for (int c = 0; c < V; ++c) oi[c] += p * vj[c];
        }
        J->lse[(U->s0 + i) * HQ + U->h] = lse;
    }
}

static void bwd_unit(job_t* J, const unit_t* U, double* sc, double* F, double* Fmat,
                     double* dL, double* dGSv, double* orow) {
    const int HQ = J->HQ, H = J->H, K = J->K, V = J->V, h = U->h;
    const long s0 = U->s0, len = U->len;
    memset(dL, 0, sizeof(double) * (len > 0 ? len : 1) * K);
    memset(dGSv, 0, sizeof(double) * (len > 0 ? len : 1));
    double dsink = 0.0;
    for (long i = 0; i < len; ++i) {
        const long ti = s0 + i;
        long jmin = first_visible(J, i);
        row_logits(J, U, i, jmin, sc, F, Fmat);
        double lse = row_lse(J, h, sc, i - jmin + 1);
        const double* dOi = J->dO + (ti * HQ + h) * V;
        /* o_i again, to form D_i = dO_i . o_i */
        for (int c = 0; c < V; ++c) orow[c] = 0.0;
        for (long j = i; j >= jmin; --j) {
            double p = exp(sc[i - j] - lse);
            const double* vj = J->v + ((s0 + j) * H + U->kh) * V;
            for (int c = 0; c < V; ++c) orow[c] += p * vj[c];
        }
        double D = 0.0;
        for (int c = 0; c < V; ++c) D += dOi[c] * orow[c];
        if (J->o) memcpy(J->o + (ti * HQ + h) * V, orow, sizeof(double) * V);
        if (J->lse) J->lse[ti * HQ + h] = lse;
        /* the sink logit has a zero value row: dS_sink = p_sink (0 - D_i) */
        if (J->sink) dsink -= exp(J->sink[h] - lse) * D;
        const double* qi = J->q + (ti * HQ + h) * K;
        double* dqi = J->dq + (ti * HQ + h) * K;
        for (long j = i; j >= jmin; --j) {
            const long tj = s0 + j;
            const double* kj = J->k + (tj * H + U->kh) * K;
            const double* vj = J->v + (tj * H + U->kh) * V;
            const double* Fj = Fmat + (i - j) * K;
            double p = exp(sc[i - j] - lse);
            double dp = 0.0;
            for (int c = 0; c < V; ++c) dp += dOi[c] * vj[c];
            double dS = p * (dp - D);
            double* dkj = J->dkh + (tj * HQ + h) * K;
            double* dvj = J->dvh + (tj * HQ + h) * V;
            const double* dOrow = (g_mutation == MUT_DV_ROW) ? J->dO + (tj * HQ + h) * V : dOi;
            for (int c = 0; c < V; ++c) dvj[c] += p * dOrow[c];
            for (int n = 0; n < K; ++n) {
                double cq = J->scale * dS * Fj[n];
                dqi[n] += cq * kj[n];
                dkj[n] += cq * qi[n];
                double c_ij = cq * qi[n] * kj[n];
                if (g_mutation == MUT_SIGN_QUERY_DL) dL[i * K + n] -= c_ij;
                else dL[i * K + n] += c_ij;
                if (g_mutation != MUT_DROP_KEY_DL) dL[j * K + n] -= c_ij;
            }
            /* scalar gate: the logit carries + GS_i - GS_j */
            double db = (g_mutation == MUT_SCALE_BIAS) ? J->scale * dS : dS;
            dGSv[i] += db;
            dGSv[j] -= db;
        }
    }
    /* reverse cumulative sums within the sequence: dg_u = sum_{t>=u} dL_t */
    for (int n = 0; n < K; ++n) {
        double acc = 0.0;
        for (long t = len - 1; t >= 0; --t) {
            acc += dL[t * K + n];
            J->dg[((s0 + t) * HQ + h) * K + n] = acc;
        }
    }
    if (J->dgs) {
        double acc = 0.0;
        for (long t = len - 1; t >= 0; --t) {
            acc += dGSv[t];
            J->dgs[(s0 + t) * HQ + h] = acc;
        }
    }
    if (J->dsink) J->dsink[(long)U->seq * HQ + h] = dsink;
}

static long max_len(const job_t* J) {
    long m = 1;
    for (int s = 0; s < J->nseq; ++s) {
        long l = J->cu[s + 1] - J->cu[s];
        if (l > m) m = l;
    }
    return m;
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    const long ml = max_len(J);
    const int K = J->K;
    unit_t U;
    U.E = (double*)malloc(sizeof(double) * ml * K);
    U.L = J->form == 1 ? (double*)malloc(sizeof(double) * ml * K) : NULL;
    U.GS = J->form == 1 ? (double*)malloc(sizeof(double) * ml) : NULL;
    double* sc = (double*)malloc(sizeof(double) * ml);
    double* F = (double*)malloc(sizeof(double) * K);
    double *Fmat = NULL, *dL = NULL, *dGSv = NULL, *orow = NULL;
    if (J->backward) {
        long wcap = (J->window > 0 && J->window + 1 < ml) ? J->window + 1 : ml;
        Fmat = (double*)malloc(sizeof(double) * wcap * K);
        dL = (double*)malloc(sizeof(double) * ml * K);
        dGSv = (double*)malloc(sizeof(double) * ml);
        orow = (double*)malloc(sizeof(double) * J->V);
    }
    const int total = J->units ? J->n_units : J->nseq * J->HQ;
    for (;;) {
        int idx = atomic_fetch_add(&J->next, 1);
        if (idx >= total) break;
        int u = J->units ? J->units[idx] : idx;
        U.seq = u / J->HQ;
        U.h = u % J->HQ;
        U.kh = kv_head(J, U.h);
        U.s0 = J->cu[U.seq];
        U.len = J->cu[U.seq + 1] - U.s0;
        unit_tables(J, &U);
        if (J->backward) bwd_unit(J, &U, sc, F, Fmat, dL, dGSv, orow);
        else fwd_unit(J, &U, sc, F);
    }
    free(U.E); free(U.L); free(U.GS);
    free(sc); free(F); free(Fmat); free(dL); free(dGSv); free(orow);
    return NULL;
}

static int run(job_t* J, int nthreads) {
    if (J->H <= 0 || J->HQ % J->H != 0) return 1;
    if (J->nseq < 0 || J->cu[0] != 0 || J->cu[J->nseq] != J->TT) return 1;
    for (int s = 0; s < J->nseq; ++s)
        if (J->cu[s + 1] < J->cu[s]) return 1;
    if (J->units)
        for (int x = 0; x < J->n_units; ++x)
            if (J->units[x] < 0 || J->units[x] >= J->nseq * J->HQ) return 1;
    atomic_store(&J->next, 0);
    if (nthreads < 1) nthreads = 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, J);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    return 0;
}

/* Forward: o [TT,HQ,V], lse [TT,HQ] (natural log).  Rows outside
 * [row_lo,row_hi) (relative to each sequence start) and units outside the
 * list are left untouched. */
int wo_forward(const double* q, const double* k, const double* v, const double* g,
               const double* gs, const double* sink, long TT, int H, int HQ, int K, int V,
               double scale, long window, const long* cu, int nseq, int form,
               const int* units, int n_units, long row_lo, long row_hi, long q_rows,
               double* o, double* lse, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.g = g; J.gs = gs; J.sink = sink;
    J.TT = TT; J.H = H; J.HQ = HQ; J.K = K; J.V = V;
    J.scale = scale; J.window = window; J.cu = cu; J.nseq = nseq; J.form = form;
    J.units = units; J.n_units = n_units; J.row_lo = row_lo; J.row_hi = row_hi;
    J.q_rows = q_rows;
    if (q_rows > 0 && (row_lo < 0 || row_hi < 0 || row_hi - row_lo > q_rows)) return 1;
    J.o = o; J.lse = lse;
    return run(&J, nthreads);
}

/* Backward of loss = sum(o * dO).  Outputs are per query head:
 * dq [TT,HQ,K], dkh [TT,HQ,K], dvh [TT,HQ,V] (before the GQA group sum),
 * dg [TT,HQ,K], dgs [TT,HQ] (NULL when gs is NULL), dsink [nseq,HQ] (NULL
 * when sink is NULL; one value per sequence, summed by the caller).
 * dq, dkh and dvh must be zero on entry.  o and lse (either may be NULL)
 * receive the forward. */
int wo_backward(const double* q, const double* k, const double* v, const double* g,
                const double* gs, const double* sink, const double* dO, long TT, int H,
                int HQ, int K, int V, double scale, long window, const long* cu, int nseq,
                int form, const int* units, int n_units, double* o, double* lse, double* dq,
                double* dkh, double* dvh, double* dg, double* dgs, double* dsink,
                int nthreads) {
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.g = g; J.gs = gs; J.sink = sink; J.dO = dO;
    J.TT = TT; J.H = H; J.HQ = HQ; J.K = K; J.V = V;
    J.scale = scale; J.window = window; J.cu = cu; J.nseq = nseq; J.form = form;
    J.units = units; J.n_units = n_units; J.row_lo = -1; J.row_hi = -1;
    J.o = o; J.lse = lse;
    J.dq = dq; J.dkh = dkh; J.dvh = dvh; J.dg = dg; J.dgs = dgs; J.dsink = dsink;
    J.backward = 1;
    return run(&J, nthreads);
}

/* Base-2 inclusive prefix P_t = carry + (sum_{u=s(t)..t} g_u) / ln 2 per
 * sequence; carry_in [nseq,HQ,K] (base-2 units) or NULL. */
int wo_prefix_log2(const double* g, long TT, int HQ, int K, const long* cu, int nseq,
                   const double* carry_in, double* P) {
    if (nseq < 0 || cu[0] != 0 || cu[nseq] != TT) return 1;
    const double inv_ln2 = (g_mutation == MUT_PREFIX_BASE) ? 1.0 : 1.0 / M_LN2;
    for (int s = 0; s < nseq; ++s)
        for (int h = 0; h < HQ; ++h)
            for (int n = 0; n < K; ++n) {
                double acc = 0.0;
                double c0 = carry_in ? carry_in[((long)s * HQ + h) * K + n] : 0.0;
                for (long t = cu[s]; t < cu[s + 1]; ++t) {
                    acc += g[(t * HQ + h) * K + n];
                    P[(t * HQ + h) * K + n] = c0 + acc * inv_ln2;
                }
            }
    return 0;
}

/*
 * lola_oracle.c -- CPU fp64 oracle for the LoLA hybrid-attention inference step.
 *
 * TEST INFRASTRUCTURE ONLY. This file defines what the GPU path must compute;
 * it is called by the tests, by __graft_entry__.smoke() and by the benchmark's
 * CPU-baseline leg, and by nothing else. It shares no code with the CUDA path.
 *
 * What it computes (LoLA: Low-Rank Linear Attention with Sparse Caching,
 * arXiv 2505.23666; gist.science technical summary, sections "Methodologie",
 * "Het Self-Recall Error (SRE) Mechanisme" and "Inferentiestrategie"):
 *
 *   Three memories per (batch, kv-head) stream: a sliding window of the most
 *   recent eta key/value pairs (full-rank softmax), a sparse global cache of at
 *   most lambda "hard to memorise" pairs (full-rank softmax), and the linear-
 *   attention recurrent state H (D x d) with normaliser s (D), holding every
 *   other pair folded in by outer products.
 *
 *   At each update interval [t0, t1):
 *     1. L = pairs leaving the window during the interval = { j : t0 <= j+eta < t1 }.
 *        Candidates Q = S (the sparse cache) united with L.
 *     2. Every candidate is scored against the state at t0 by the Self-Recall
 *        Error SRE(k,v|H,s) = || phi(k)^T H / (phi(k)^T s + eps) - v ||^2
 *        (the SRE equation of the "Self-Recall Error" section; eps added to the
 *        denominator). The ablations of the "Belangrijkste bijdragen" and
 *        "Ablaties" sections swap this score for the magnitude of attention
 *        weights or a softmax-approximation error, and the inference strategy
 *        mentions a FIFO structure; scorer 1 / 2 / 3 select those (this build's
 *        readings: the softmax weight of the candidate for the interval's first
 *        query, summed over the group's heads; the squared gap between that
 *        weight and the linear-attention weight phi(q).phi(k) normalised over the
 *        candidates, summed over heads; the token index, i.e. the most recent
 *        pairs stay).
 *     3. The min(lambda, |Q|) candidates of highest SRE stay in the cache
 *        (ties: lower token index stays); the rest, F, are folded.
 *     4. E = S n F is folded at the interval start: H' = H + sum phi(k) v^T,
 *        s' = s + sum phi(k).
 *     5. Each query p in [t0, t1) combines softmax over the kept cache and the
 *        window with the linear readout of (H', s') and of the folded leaving
 *        pairs that have left the window by p, under one shared normaliser.
 *     6. At t1: S <- kept set, H <- H' + sum over L n F.
 *   Feature map (the pages only call it a low-rank positive feature map; this
 *   build fixes it): phi(x) = [softmax(x W), softmax(-x W)], W is d x D/2.
 *   Softmax logits are q.k / sqrt(d).
 *
 * Interval boundaries are an input (a list of interval lengths), so the same
 * routine covers chunkwise prefill (length C) and decode (length C_dec).
 *
 * Inputs are float32 arrays whose values are exactly the workload dtype's values
 * (bf16 values widen exactly); all arithmetic is fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t B, Hq, Hkv, d, D, eta, lam;
    double eps;
    int32_t scorer; /* 0 SRE, 1 attention weight, 2 softmax-approximation error, 3 recency */
    int32_t w_per_head; /* 1: W holds one d x D/2 matrix per kv-head (the pages leave this open) */
} oracle_cfg;

/* phi(x) = [softmax(x W), softmax(-x W)]  (x: d, W: d x D/2 row-major, out: D) */
void oracle_phi(const double *x, const double *W, int d, int D, double *out)
{
    int Dh = D / 2;
    double *z = (double *)malloc(sizeof(double) * (size_t)Dh);
    for (int i = 0; i < Dh; ++i) {
        double acc = 0.0;
        for (int a = 0; a < d; ++a) acc += x[a] * W[(size_t)a * Dh + i];
        z[i] = acc;
    }
    /* softmax(z): shift by the max, exact in real arithmetic */
    double zmax = -INFINITY, zmin = INFINITY;
    for (int i = 0; i < Dh; ++i) {
        if (z[i] > zmax) zmax = z[i];
        if (z[i] < zmin) zmin = z[i];
    }
    double sp = 0.0, sn = 0.0;
    for (int i = 0; i < Dh; ++i) {
        out[i] = exp(z[i] - zmax);
        out[Dh + i] = exp(-z[i] + zmin);    /* softmax(-z), shifted by max(-z) = -zmin */
        sp += out[i];
        sn += out[Dh + i];
    }
    for (int i = 0; i < Dh; ++i) {
        out[i] /= sp;
        out[Dh + i] /= sn;
    }
    free(z);
}

/* SRE of one pair against (H, s): || phi^T H / (phi^T s + eps) - v ||^2.
 * With eps = 0 and phi^T s = 0 (empty state) the prediction is taken as 0. */
double oracle_sre(const double *phik, const double *v, const double *H, const double *s,
                  int d, int D, double eps)
{
    double den = eps;
    for (int i = 0; i < D; ++i) den += phik[i] * s[i];
    double num[1024];
    for (int c = 0; c < d; ++c) num[c] = 0.0;
    for (int i = 0; i < D; ++i)
        for (int c = 0; c < d; ++c) num[c] += phik[i] * H[(size_t)i * d + c];
    double err = 0.0;
    for (int c = 0; c < d; ++c) {
        double pred = (den != 0.0) ? num[c] / den : 0.0;
        double diff = pred - v[c];
        err += diff * diff;
    }
    return err;
}

typedef struct {
    double sre;
    int32_t tok;
} cand_t;

/* order: SRE descending, then token index ascending (lower index is kept) */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->sre > y->sre) return -1;
    if (x->sre < y->sre) return 1;
    return (x->tok > y->tok) - (x->tok < y->tok);
}

static int int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

typedef struct {
    const oracle_cfg *cfg;
    int T;
    const float *q, *k, *v; /* [B][T][H][d] */
    const double *W;        /* [d][D/2] */
    int n_int;
    const int32_t *int_len;
    const uint8_t *qmask; /* [T] or NULL: which query positions get outputs */
    const int32_t *out_row; /* [T] or NULL: output row of each position (NULL: row = position) */
    int n_out;            /* output rows per batch */
    double *out;          /* [B][n_out][Hq][d] */
    int32_t *kept;        /* [n_int][nstreams][lam] or NULL (sorted ascending, -1 pad) */
    int32_t *nkept;       /* [n_int][nstreams] or NULL */
    int32_t *nq;          /* [n_int][nstreams] or NULL */
    double *margin;       /* [n_int][nstreams] or NULL */
    int32_t *cand_tok;    /* [n_int][nstreams][cand_cap] or NULL */
    double *cand_sre;     /* same */
    int cand_cap;
    double *H_final;      /* [nstreams][D][d] or NULL */
    double *s_final;      /* [nstreams][D] or NULL */
    int next_stream;
    pthread_mutex_t mu;
    int status;
} job_t;

static void run_stream(job_t *J, int st)
{
    const oracle_cfg *cfg = J->cfg;
    const int B = cfg->B, Hq = cfg->Hq, Hkv = cfg->Hkv, d = cfg->d, D = cfg->D;
    const int eta = cfg->eta, lam = cfg->lam, T = J->T;
    const int g = Hq / Hkv;
    const int b = st / Hkv, hk = st % Hkv;
    const int nstreams = B * Hkv;
    const double eps = cfg->eps;
    const double scale = 1.0 / sqrt((double)d);
    /* the feature-map matrix of this stream's kv-head (its query heads share it) */
    const double *Wst = J->W + (cfg->w_per_head ? (size_t)hk * d * (D / 2) : 0);
    (void)B;

    /* per-stream copies of keys, values and phi(k) for every token */
    double *kd = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *vd = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *phik = (double *)malloc(sizeof(double) * (size_t)T * D);
    for (int t = 0; t < T; ++t) {
        size_t src = (((size_t)b * T + t) * Hkv + hk) * d;
        for (int c = 0; c < d; ++c) {
            kd[(size_t)t * d + c] = J->k[src + c];
            vd[(size_t)t * d + c] = J->v[src + c];
        }
        oracle_phi(kd + (size_t)t * d, Wst, d, D, phik + (size_t)t * D);
    }

    double *H = (double *)calloc((size_t)D * d, sizeof(double));
    double *s = (double *)calloc((size_t)D, sizeof(double));
    double *Hp = (double *)malloc(sizeof(double) * (size_t)D * d); /* H' */
    double *sp = (double *)malloc(sizeof(double) * (size_t)D);

    /* status per token: 0 = not yet resolved, 1 = in sparse cache S, 2 = folded */
    uint8_t *status = (uint8_t *)calloc((size_t)T, 1);
    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)(lam > 0 ? lam : 1));
    int nS = 0;
    int maxlen = 0;
    for (int i = 0; i < J->n_int; ++i)
        if (J->int_len[i] > maxlen) maxlen = J->int_len[i];
    cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(lam + maxlen + 1));
    uint8_t *keep = (uint8_t *)calloc((size_t)T, 1); /* kept flag for this interval */
    uint8_t *lfold = (uint8_t *)calloc((size_t)T, 1); /* j in L n F for this interval */
    double *phiq = (double *)malloc(sizeof(double) * (size_t)D);
    double *sc = (double *)malloc(sizeof(double) * (size_t)(lam + eta + maxlen + 1));
    double *sc2 = (double *)malloc(sizeof(double) * (size_t)(lam + maxlen + 1));
    int32_t *Aset = (int32_t *)malloc(sizeof(int32_t) * (size_t)(lam + eta + maxlen + 1));
    double *num = (double *)malloc(sizeof(double) * (size_t)d);
    double *lin = (double *)malloc(sizeof(double) * (size_t)d);

    int t0 = 0;
    for (int ci = 0; ci < J->n_int; ++ci) {
        const int t1 = t0 + J->int_len[ci];
        /* 1. candidates: S plus the pairs leaving the window in [t0, t1) */
        int Llo = t0 - eta, Lhi = t1 - eta; /* j in [Llo, Lhi) */
        if (Llo < 0) Llo = 0;
        if (Lhi < Llo) Lhi = Llo;
        int nQ = 0;
        for (int i = 0; i < nS; ++i) cand[nQ++].tok = S[i];
        for (int j = Llo; j < Lhi; ++j) cand[nQ++].tok = j;
        /* 2. score every candidate (the highest scores stay cached) */
        if (cfg->scorer == 0) {
            /* Self-Recall Error against the state at t0 */
            for (int c = 0; c < nQ; ++c) {
                const int j = cand[c].tok;
                cand[c].sre = oracle_sre(phik + (size_t)j * D, vd + (size_t)j * d, H, s, d, D, eps);
            }
        } else if (cfg->scorer == 3) {
            /* recency: the most recent pairs stay (a first-in first-out cache) */
            for (int c = 0; c < nQ; ++c) cand[c].sre = (double)cand[c].tok;
        } else {
            /* the interval's first query, every head of the group: a = softmax over the
               candidates of q.k / sqrt(d); scorer 1 keeps the largest sum over heads of a,
               scorer 2 the largest sum over heads of (a - b)^2, where b is the linear
               attention weight phi(q).phi(k) normalised over the candidates */
            for (int c = 0; c < nQ; ++c) cand[c].sre = 0.0;
            for (int r = 0; r < g; ++r) {
                const float *qsrc = J->q + (((size_t)b * T + t0) * Hq + hk * g + r) * d;
                double qv[1024];
                for (int c = 0; c < d; ++c) qv[c] = qsrc[c];
                double mx = -INFINITY, z = 0.0, u = 0.0;
                for (int c = 0; c < nQ; ++c) {
                    const double *kk = kd + (size_t)cand[c].tok * d;
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += qv[e] * kk[e];
                    sc[c] = dot * scale;
                    if (sc[c] > mx) mx = sc[c];
                }
                for (int c = 0; c < nQ; ++c) z += exp(sc[c] - mx);
                if (cfg->scorer == 2) {
                    oracle_phi(qv, Wst, d, D, phiq);
                    for (int c = 0; c < nQ; ++c) {
                        const double *pk = phik + (size_t)cand[c].tok * D;
                        double w = 0.0;
                        for (int e = 0; e < D; ++e) w += phiq[e] * pk[e];
                        sc2[c] = w;
                        u += w;
                    }
                }
                for (int c = 0; c < nQ; ++c) {
                    const double a = exp(sc[c] - mx) / z;
                    if (cfg->scorer == 1) {
                        cand[c].sre += a;
                    } else {
                        const double e2 = a - sc2[c] / u;
                        cand[c].sre += e2 * e2;
                    }
                }
            }
        }
        size_t logi = (size_t)ci * nstreams + st;
        if (J->cand_tok && J->cand_sre) {
            for (int i = 0; i < J->cand_cap; ++i) {
                J->cand_tok[logi * J->cand_cap + i] = (i < nQ) ? cand[i].tok : -1;
                J->cand_sre[logi * J->cand_cap + i] = (i < nQ) ? cand[i].sre : NAN;
            }
        }
        /* 3. keep the top min(lam, |Q|) by SRE (ties: lower index kept) */
        qsort(cand, (size_t)nQ, sizeof(cand_t), cand_cmp);
        int nK = nQ < lam ? nQ : lam;
        if (J->margin) {
            double m = INFINITY;
            if (nQ > lam && lam > 0) {
                double a = cand[lam - 1].sre, c = cand[lam].sre;
                m = (a > 0.0) ? (a - c) / a : 0.0;
            }
            J->margin[logi] = m;
        }
        if (J->nq) J->nq[logi] = nQ;
        for (int i = 0; i < nK; ++i) keep[cand[i].tok] = 1;

        /* 4. fold E = S n F at the interval start */
        memcpy(Hp, H, sizeof(double) * (size_t)D * d);
        memcpy(sp, s, sizeof(double) * (size_t)D);
        for (int i = 0; i < nS; ++i) {
            int j = S[i];
            if (keep[j]) continue;
            status[j] = 2;
            const double *ph = phik + (size_t)j * D, *vv = vd + (size_t)j * d;
            for (int r = 0; r < D; ++r) {
                for (int c = 0; c < d; ++c) Hp[(size_t)r * d + c] += ph[r] * vv[c];
                sp[r] += ph[r];
            }
        }
        for (int j = Llo; j < Lhi; ++j)
            if (!keep[j]) lfold[j] = 1;

        /* 5. outputs for the queries of the interval */
        for (int p = t0; p < t1 && p < T; ++p) {
            if (J->qmask && !J->qmask[p]) continue;
            /* softmax set A_p and linear band B_p do not depend on the head */
            int nA = 0;
            for (int i = 0; i < nS; ++i)
                if (keep[S[i]]) Aset[nA++] = S[i];
            int blo = t0 - eta < 0 ? 0 : t0 - eta;
            for (int j = blo; j <= p; ++j)
                if (!lfold[j] || j > p - eta) Aset[nA++] = j;
            for (int r = 0; r < g; ++r) {
                int hq = hk * g + r;
                const float *qsrc = J->q + (((size_t)b * T + p) * Hq + hq) * d;
                double qv[1024];
                for (int c = 0; c < d; ++c) qv[c] = qsrc[c];
                double mx = 0.0; /* shift m = max(0, max score) */
                for (int a = 0; a < nA; ++a) {
                    const double *kk = kd + (size_t)Aset[a] * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += qv[c] * kk[c];
                    sc[a] = dot * scale;
                    if (sc[a] > mx) mx = sc[a];
                }
                double den = 0.0;
                for (int c = 0; c < d; ++c) num[c] = 0.0;
                for (int a = 0; a < nA; ++a) {
                    double w = exp(sc[a] - mx);
                    den += w;
                    const double *vv = vd + (size_t)Aset[a] * d;
                    for (int c = 0; c < d; ++c) num[c] += w * vv[c];
                }
                /* linear terms: phi(q)^T H', phi(q)^T s', and the folded band */
                oracle_phi(qv, Wst, d, D, phiq);
                double lden = eps;
                for (int c = 0; c < d; ++c) lin[c] = 0.0;
                for (int rr = 0; rr < D; ++rr) {
                    lden += phiq[rr] * sp[rr];
                    for (int c = 0; c < d; ++c) lin[c] += phiq[rr] * Hp[(size_t)rr * d + c];
                }
                for (int j = blo; j <= p - eta; ++j) {
                    if (!lfold[j]) continue;
                    const double *ph = phik + (size_t)j * D, *vv = vd + (size_t)j * d;
                    double w = 0.0;
                    for (int rr = 0; rr < D; ++rr) w += phiq[rr] * ph[rr];
                    lden += w;
                    for (int c = 0; c < d; ++c) lin[c] += w * vv[c];
                }
                double em = exp(-mx);
                den += em * lden;
                const int orow = J->out_row ? J->out_row[p] : p;
                double *o = J->out + (((size_t)b * J->n_out + orow) * Hq + hq) * d;
                for (int c = 0; c < d; ++c) o[c] = (num[c] + em * lin[c]) / den;
            }
        }

        /* 6. close the interval: S <- kept set, H <- H' + sum over L n F */
        for (int r = 0; r < D * d; ++r) H[r] = Hp[r];
        for (int r = 0; r < D; ++r) s[r] = sp[r];
        for (int j = Llo; j < Lhi; ++j) {
            if (!lfold[j]) continue;
            status[j] = 2;
            const double *ph = phik + (size_t)j * D, *vv = vd + (size_t)j * d;
            for (int r = 0; r < D; ++r) {
                for (int c = 0; c < d; ++c) H[(size_t)r * d + c] += ph[r] * vv[c];
                s[r] += ph[r];
            }
        }
        int n = 0;
        for (int i = 0; i < nK; ++i) {
            S[n++] = cand[i].tok;
            status[cand[i].tok] = 1;
        }
        qsort(S, (size_t)n, sizeof(int32_t), int_cmp);
        nS = n;
        if (J->kept) {
            for (int i = 0; i < lam; ++i) J->kept[logi * lam + i] = (i < nS) ? S[i] : -1;
        }
        if (J->nkept) J->nkept[logi] = nS;
        for (int i = 0; i < nQ; ++i) keep[cand[i].tok] = 0;
        for (int j = Llo; j < Lhi; ++j) lfold[j] = 0;
        t0 = t1;
    }
    if (J->H_final) memcpy(J->H_final + (size_t)st * D * d, H, sizeof(double) * (size_t)D * d);
    if (J->s_final) memcpy(J->s_final + (size_t)st * D, s, sizeof(double) * (size_t)D);

    free(kd); free(vd); free(phik); free(H); free(s); free(Hp); free(sp);
    free(status); free(S); free(cand); free(keep); free(lfold); free(phiq);
    free(sc); free(sc2); free(Aset); free(num); free(lin);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int nstreams = J->cfg->B * J->cfg->Hkv;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int st = J->next_stream++;
        pthread_mutex_unlock(&J->mu);
        if (st >= nstreams) break;
        run_stream(J, st);
    }
    return NULL;
}

/*
 * Runs the recurrence for every (batch, kv-head) stream from an empty state.
 * Returns 0 on success, a negative number on an invalid argument.
 * Tokens [0, T) are split into n_int consecutive intervals of the given lengths;
 * they must cover [0, T), and the last may extend past T when the pairs it
 * scores (those leaving the window before its end) all exist. Every output
 * pointer except `out` may be NULL. With out_row, the output of position p goes
 * to row out_row[p] of an [B][n_out][Hq][d] array (for sampled long runs).
 */
int oracle_run(const oracle_cfg *cfg, int T, const float *q, const float *k, const float *v,
               const float *Wf, int n_int, const int32_t *int_len, const uint8_t *qmask,
               const int32_t *out_row, int n_out,
               double *out, int32_t *kept, int32_t *nkept, int32_t *nq, double *margin,
               int32_t *cand_tok, double *cand_sre, int cand_cap, double *H_final,
               double *s_final, int nthreads)
{
    if (!cfg || cfg->Hkv <= 0 || cfg->Hq % cfg->Hkv != 0 || cfg->d <= 0 || cfg->d > 1024 ||
        cfg->D <= 0 || cfg->D % 2 != 0 || cfg->eta < 0 || cfg->lam < 0 || T < 0)
        return -1;
    /* The intervals cover [0, T); the last one may run past T (a decode
     * interval that is still open), as long as every pair it scores exists. */
    long tot = 0;
    for (int i = 0; i < n_int; ++i) {
        if (int_len[i] <= 0) return -2;
        if (tot >= T && T > 0) return -3;
        tot += int_len[i];
        if (tot - cfg->eta > T) return -4;
    }
    if (tot < T) return -3;
    int Dh = cfg->D / 2;
    const int nW = cfg->w_per_head ? cfg->Hkv : 1;
    double *W = (double *)malloc(sizeof(double) * (size_t)nW * cfg->d * Dh);
    for (int i = 0; i < nW * cfg->d * Dh; ++i) W[i] = Wf[i];
    job_t J;
    memset(&J, 0, sizeof(J));
    J.cfg = cfg; J.T = T; J.q = q; J.k = k; J.v = v; J.W = W;
    J.n_int = n_int; J.int_len = int_len; J.qmask = qmask; J.out = out;
    J.out_row = out_row; J.n_out = out_row ? n_out : T;
    if (out_row) {
        /* every position that gets an output needs a row inside [0, n_out) */
        for (int p = 0; p < T; ++p)
            if ((!qmask || qmask[p]) && (out_row[p] < 0 || out_row[p] >= n_out)) {
                free(W);
                return -5;
            }
    }
    J.kept = kept; J.nkept = nkept; J.nq = nq; J.margin = margin;
    J.cand_tok = cand_tok; J.cand_sre = cand_sre; J.cand_cap = cand_cap;
    J.H_final = H_final; J.s_final = s_final;
    pthread_mutex_init(&J.mu, NULL);
    int nstreams = cfg->B * cfg->Hkv;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nstreams) nthreads = nstreams;
    if (nthreads == 1) {
        worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.mu);
    free(W);
    return 0;
}

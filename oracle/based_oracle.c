/*
 * based_oracle.c -- plain, slow, fp64 CPU oracle for the Based attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library and its
 * Python binding) may call, link or load this file.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg use it.  It shares no code,
 * header, constant or table with the CUDA path.
 *
 * Every routine is the textbook definition written out with loops, in double
 * precision, with no blocking, fusion or reordering beyond what the
 * definition itself states.  Parallelism is only across independent
 * (batch, head) sequences, one pthread per slice of them.
 *
 * Sources (the method this code restates):
 *  - "Базированная модель, часть 2" (botka_chronics blog post on Based),
 *    section "Что за линейное внимание?": softmax is replaced by the
 *    second-order Taylor expansion exp(qk) ~ 1 + qk + (qk)^2/2, realised as
 *    the feature map cat(1, x, vec(x x^T)/sqrt(2)) over the FULL outer
 *    product (both x_i x_j and x_j x_i appear), so d = 16 gives
 *    1 + 16 + 256 = 273 features.  Here the map is applied to x / d^(1/4)
 *    so that phi(q).phi(k) = 1 + q.k/sqrt(d) + (q.k)^2/(2d), the expansion
 *    of exp(q.k/sqrt(d)).
 *  - same post, paragraph on the state size: the recurrent form keeps a KV
 *    state (numerator) and a K state (denominator).
 *  - "based/train" README, training views: the "quadratic" view (masked
 *    phi(Q)phi(K)^T V), the "fla_parallel" chunked view and the "linear"
 *    causal-dot-product (recurrent) view compute the same function; all
 *    three are written out below so they can be checked against each other.
 *  - Based README (HazyResearch/based), introduction, item 1: exact softmax
 *    attention over a short sliding window (size 64) for local
 *    dependencies.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  feature order: index 0 = 1, 1..d = x_i/d^(1/4), 1+d+i*d+j = x_i x_j/sqrt(2d);
 *  eps is added to the denominator only; causality is inclusive (s <= t);
 *  the window holds the W keys t-W+1..t (the current token included) and the
 *  softmax temperature is 1/sqrt(d_head); a decode step first folds the new
 *  token into the state (or ring) and then reads out.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* feature map                                                               */
/* ------------------------------------------------------------------------ */

int oracle_num_features(int d) { return 1 + d + d * d; }

/* phi(x) for one d-vector; f has 1 + d + d*d entries. */
void oracle_phi(const double* x, int d, double* f) {
    const double lin_scale = 1.0 / sqrt(sqrt((double)d));        /* d^(-1/4)       */
    const double quad_scale = 1.0 / (sqrt(2.0) * sqrt((double)d)); /* 1/(sqrt2 sqrtd) */
    f[0] = 1.0;
    for (int i = 0; i < d; ++i) f[1 + i] = x[i] * lin_scale;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) f[1 + d + i * d + j] = x[i] * x[j] * quad_scale;
}

static double dot(const double* a, const double* b, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* ------------------------------------------------------------------------ */
/* a tiny parallel-for over independent sequences                           */
/* ------------------------------------------------------------------------ */

typedef void (*seq_fn)(void* ctx, int seq);
typedef struct { seq_fn fn; void* ctx; int begin, end; } slice_t;

static void* run_slice(void* p) {
    slice_t* s = (slice_t*)p;
    for (int i = s->begin; i < s->end; ++i) s->fn(s->ctx, i);
    return NULL;
}

static void parallel_for(int n, int nthreads, seq_fn fn, void* ctx) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n;
    if (nthreads <= 1) {
        for (int i = 0; i < n; ++i) fn(ctx, i);
        return;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    slice_t* sl = (slice_t*)malloc(sizeof(slice_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        sl[t].fn = fn;
        sl[t].ctx = ctx;
        sl[t].begin = (int)((long long)n * t / nthreads);
        sl[t].end = (int)((long long)n * (t + 1) / nthreads);
        pthread_create(&th[t], NULL, run_slice, &sl[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(sl);
}

/* ------------------------------------------------------------------------ */
/* causal linear attention                                                  */
/* layouts: q,k [n_seq, L, d]; v,y [n_seq, L, dv]; S [n_seq, F, dv]; z [n_seq, F]
 * ------------------------------------------------------------------------ */

typedef struct {
    const double *q, *k, *v, *S0, *z0;
    double *y, *S1, *z1;
    int L, d, dv;
    double eps;
    const int* bounds; /* chunked form: chunk starts, bounds[nchunks] == L */
    int nchunks;
} lin_ctx;

/* Recurrent ("linear" view): S += phi(k_t) v_t^T ; z += phi(k_t) ;
 * y_t = phi(q_t)^T S / (phi(q_t).z + eps), with the update before the read. */
static void lin_recurrent_seq(void* p, int n) {
    lin_ctx* c = (lin_ctx*)p;
    const int L = c->L, d = c->d, dv = c->dv, F = oracle_num_features(d);
    const double* q = c->q + (size_t)n * L * d;
    const double* k = c->k + (size_t)n * L * d;
    const double* v = c->v + (size_t)n * L * dv;
    double* y = c->y + (size_t)n * L * dv;
    double* S = (double*)calloc((size_t)F * dv, sizeof(double));
    double* z = (double*)calloc((size_t)F, sizeof(double));
    double* fq = (double*)malloc(sizeof(double) * (size_t)F);
    double* fk = (double*)malloc(sizeof(double) * (size_t)F);
    if (c->S0) memcpy(S, c->S0 + (size_t)n * F * dv, sizeof(double) * (size_t)F * dv);
    if (c->z0) memcpy(z, c->z0 + (size_t)n * F, sizeof(double) * (size_t)F);
    for (int t = 0; t < L; ++t) {
        oracle_phi(k + (size_t)t * d, d, fk);
        oracle_phi(q + (size_t)t * d, d, fq);
        const double* vt = v + (size_t)t * dv;
        for (int f = 0; f < F; ++f) {
            for (int j = 0; j < dv; ++j) S[(size_t)f * dv + j] += fk[f] * vt[j];
            z[f] += fk[f];
        }
        const double den = dot(fq, z, F) + c->eps;
        for (int j = 0; j < dv; ++j) {
            double num = 0.0;
            for (int f = 0; f < F; ++f) num += fq[f] * S[(size_t)f * dv + j];
            y[(size_t)t * dv + j] = num / den;
        }
    }
    if (c->S1) memcpy(c->S1 + (size_t)n * F * dv, S, sizeof(double) * (size_t)F * dv);
    if (c->z1) memcpy(c->z1 + (size_t)n * F, z, sizeof(double) * (size_t)F);
    free(S); free(z); free(fq); free(fk);
}

void oracle_linattn_recurrent(const double* q, const double* k, const double* v,
                              int n_seq, int L, int d, int dv, double eps,
                              const double* S0, const double* z0,
                              double* y, double* S1, double* z1, int nthreads) {
    lin_ctx c = {q, k, v, S0, z0, y, S1, z1, L, d, dv, eps, NULL, 0};
    parallel_for(n_seq, nthreads, lin_recurrent_seq, &c);
}

/* Quadratic ("quadratic" view): w_ts = phi(q_t).phi(k_s) for s <= t;
 * y_t = sum_s w_ts v_s / (sum_s w_ts + eps). */
static void lin_quadratic_seq(void* p, int n) {
    lin_ctx* c = (lin_ctx*)p;
    const int L = c->L, d = c->d, dv = c->dv, F = oracle_num_features(d);
    const double* q = c->q + (size_t)n * L * d;
    const double* k = c->k + (size_t)n * L * d;
    const double* v = c->v + (size_t)n * L * dv;
    double* y = c->y + (size_t)n * L * dv;
    double* fq = (double*)malloc(sizeof(double) * (size_t)F * L);
    double* fk = (double*)malloc(sizeof(double) * (size_t)F * L);
    double* num = (double*)malloc(sizeof(double) * (size_t)dv);
    for (int t = 0; t < L; ++t) {
        oracle_phi(q + (size_t)t * d, d, fq + (size_t)t * F);
        oracle_phi(k + (size_t)t * d, d, fk + (size_t)t * F);
    }
    for (int t = 0; t < L; ++t) {
        double den = 0.0;
        for (int j = 0; j < dv; ++j) num[j] = 0.0;
        for (int s = 0; s <= t; ++s) {
            const double w = dot(fq + (size_t)t * F, fk + (size_t)s * F, F);
            den += w;
            for (int j = 0; j < dv; ++j) num[j] += w * v[(size_t)s * dv + j];
        }
        for (int j = 0; j < dv; ++j) y[(size_t)t * dv + j] = num[j] / (den + c->eps);
    }
    free(fq); free(fk); free(num);
}

void oracle_linattn_quadratic(const double* q, const double* k, const double* v,
                              int n_seq, int L, int d, int dv, double eps,
                              double* y, int nthreads) {
    lin_ctx c = {q, k, v, NULL, NULL, y, NULL, NULL, L, d, dv, eps, NULL, 0};
    parallel_for(n_seq, nthreads, lin_quadratic_seq, &c);
}

/* Chunked ("fla_parallel" view) for an arbitrary partition of [0, L) into
 * chunks [bounds[c], bounds[c+1]): inside a chunk the quadratic masked form,
 * across chunks the state accumulated from all earlier chunks; the state is
 * advanced once per chunk, after its outputs. */
static void lin_chunked_seq(void* p, int n) {
    lin_ctx* c = (lin_ctx*)p;
    const int L = c->L, d = c->d, dv = c->dv, F = oracle_num_features(d);
    const double* q = c->q + (size_t)n * L * d;
    const double* k = c->k + (size_t)n * L * d;
    const double* v = c->v + (size_t)n * L * dv;
    double* y = c->y + (size_t)n * L * dv;
    double* S = (double*)calloc((size_t)F * dv, sizeof(double));
    double* z = (double*)calloc((size_t)F, sizeof(double));
    double* fq = (double*)malloc(sizeof(double) * (size_t)F * L);
    double* fk = (double*)malloc(sizeof(double) * (size_t)F * L);
    double* num = (double*)malloc(sizeof(double) * (size_t)dv);
    for (int t = 0; t < L; ++t) {
        oracle_phi(q + (size_t)t * d, d, fq + (size_t)t * F);
        oracle_phi(k + (size_t)t * d, d, fk + (size_t)t * F);
    }
    for (int ci = 0; ci < c->nchunks; ++ci) {
        const int a = c->bounds[ci], b = c->bounds[ci + 1];
        for (int t = a; t < b; ++t) {
            const double* fqt = fq + (size_t)t * F;
            /* inter-chunk part: everything before the chunk, via the state */
            double den = dot(fqt, z, F);
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int f = 0; f < F; ++f) acc += fqt[f] * S[(size_t)f * dv + j];
                num[j] = acc;
            }
            /* intra-chunk part: causal, s in [a, t] */
            for (int s = a; s <= t; ++s) {
                const double w = dot(fqt, fk + (size_t)s * F, F);
                den += w;
                for (int j = 0; j < dv; ++j) num[j] += w * v[(size_t)s * dv + j];
            }
            for (int j = 0; j < dv; ++j) y[(size_t)t * dv + j] = num[j] / (den + c->eps);
        }
        for (int s = a; s < b; ++s) {
            const double* fks = fk + (size_t)s * F;
            for (int f = 0; f < F; ++f) {
                for (int j = 0; j < dv; ++j) S[(size_t)f * dv + j] += fks[f] * v[(size_t)s * dv + j];
                z[f] += fks[f];
            }
        }
    }
    free(S); free(z); free(fq); free(fk); free(num);
}

/* Returns 0 on success, -1 if bounds is not a partition of [0, L). */
int oracle_linattn_chunked(const double* q, const double* k, const double* v,
                           int n_seq, int L, int d, int dv, double eps,
                           const int* bounds, int nchunks, double* y, int nthreads) {
    if (nchunks < 1 || bounds[0] != 0 || bounds[nchunks] != L) return -1;
    for (int i = 0; i < nchunks; ++i)
        if (bounds[i + 1] <= bounds[i]) return -1;
    lin_ctx c = {q, k, v, NULL, NULL, y, NULL, NULL, L, d, dv, eps, bounds, nchunks};
    parallel_for(n_seq, nthreads, lin_chunked_seq, &c);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* sliding-window softmax attention                                         */
/* layouts: q,k,v,y [n_seq, L, dh]                                          */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *q, *k, *v;
    double* y;
    int L, dh, W;
} win_ctx;

/* y_t = sum_{s=max(0,t-W+1)}^{t} softmax_s(q_t.k_s / sqrt(dh)) v_s,
 * the maximum subtracted before exponentiation. */
static void window_seq(void* p, int n) {
    win_ctx* c = (win_ctx*)p;
    const int L = c->L, dh = c->dh, W = c->W;
    const double* q = c->q + (size_t)n * L * dh;
    const double* k = c->k + (size_t)n * L * dh;
    const double* v = c->v + (size_t)n * L * dh;
    double* y = c->y + (size_t)n * L * dh;
    double* sc = (double*)malloc(sizeof(double) * (size_t)W);
    const double scale = 1.0 / sqrt((double)dh);
    for (int t = 0; t < L; ++t) {
        const int lo = t - W + 1 > 0 ? t - W + 1 : 0;
        double m = -INFINITY;
        for (int s = lo; s <= t; ++s) {
            sc[s - lo] = dot(q + (size_t)t * dh, k + (size_t)s * dh, dh) * scale;
            if (sc[s - lo] > m) m = sc[s - lo];
        }
        double den = 0.0;
        for (int s = lo; s <= t; ++s) {
            sc[s - lo] = exp(sc[s - lo] - m);
            den += sc[s - lo];
        }
        for (int j = 0; j < dh; ++j) {
            double acc = 0.0;
            for (int s = lo; s <= t; ++s) acc += sc[s - lo] * v[(size_t)s * dh + j];
            y[(size_t)t * dh + j] = acc / den;
        }
    }
    free(sc);
}

void oracle_window_attn(const double* q, const double* k, const double* v,
                        int n_seq, int L, int dh, int W, double* y, int nthreads) {
    win_ctx c = {q, k, v, y, L, dh, W};
    parallel_for(n_seq, nthreads, window_seq, &c);
}

/* ------------------------------------------------------------------------ */
/* decode: one new token per sequence                                       */
/* ------------------------------------------------------------------------ */

/* Linear part: S += phi(k) v^T ; z += phi(k) ; y = phi(q)^T S / (phi(q).z + eps).
 * q,k [n_seq, d]; v,y [n_seq, dv]; S [n_seq, F, dv] and z [n_seq, F] in place. */
void oracle_decode_linear(const double* q, const double* k, const double* v,
                          double* S, double* z, int n_seq, int d, int dv, double eps,
                          double* y) {
    const int F = oracle_num_features(d);
    double* fq = (double*)malloc(sizeof(double) * (size_t)F);
    double* fk = (double*)malloc(sizeof(double) * (size_t)F);
    for (int n = 0; n < n_seq; ++n) {
        double* Sn = S + (size_t)n * F * dv;
        double* zn = z + (size_t)n * F;
        const double* vn = v + (size_t)n * dv;
        oracle_phi(k + (size_t)n * d, d, fk);
        oracle_phi(q + (size_t)n * d, d, fq);
        for (int f = 0; f < F; ++f) {
            for (int j = 0; j < dv; ++j) Sn[(size_t)f * dv + j] += fk[f] * vn[j];
            zn[f] += fk[f];
        }
        const double den = dot(fq, zn, F) + eps;
        for (int j = 0; j < dv; ++j) {
            double num = 0.0;
            for (int f = 0; f < F; ++f) num += fq[f] * Sn[(size_t)f * dv + j];
            y[(size_t)n * dv + j] = num / den;
        }
    }
    free(fq); free(fk);
}

/* Window part: position pos (0-based, shared by all sequences) is written
 * into ring slot pos mod W, then softmax attention over the slots holding
 * positions max(0, pos-W+1)..pos.  q,k,v,y [n_seq, dh]; rings [n_seq, W, dh]. */
void oracle_decode_window(const double* q, const double* k, const double* v,
                          double* k_ring, double* v_ring, long long pos,
                          int n_seq, int dh, int W, double* y) {
    double* sc = (double*)malloc(sizeof(double) * (size_t)W);
    const double scale = 1.0 / sqrt((double)dh);
    const long long lo = pos - W + 1 > 0 ? pos - W + 1 : 0;
    for (int n = 0; n < n_seq; ++n) {
        double* kr = k_ring + (size_t)n * W * dh;
        double* vr = v_ring + (size_t)n * W * dh;
        const int slot = (int)(pos % W);
        for (int j = 0; j < dh; ++j) {
            kr[(size_t)slot * dh + j] = k[(size_t)n * dh + j];
            vr[(size_t)slot * dh + j] = v[(size_t)n * dh + j];
        }
        double m = -INFINITY;
        for (long long p = lo; p <= pos; ++p) {
            const int s = (int)(p % W);
            sc[p - lo] = dot(q + (size_t)n * dh, kr + (size_t)s * dh, dh) * scale;
            if (sc[p - lo] > m) m = sc[p - lo];
        }
        double den = 0.0;
        for (long long p = lo; p <= pos; ++p) {
            sc[p - lo] = exp(sc[p - lo] - m);
            den += sc[p - lo];
        }
        for (int j = 0; j < dh; ++j) {
            double acc = 0.0;
            for (long long p = lo; p <= pos; ++p) acc += sc[p - lo] * vr[(size_t)(p % W) * dh + j];
            y[(size_t)n * dh + j] = acc / den;
        }
    }
    free(sc);
}

/* ------------------------------------------------------------------------ */
/* projections of the layer input                                           */
/* layouts: x [B, L, Dm]; w [N, Dm] (one output feature per row)             */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *x, *w, *bias, *h;
    double* y;
    int L, Dm, H, D, K;
} proj_ctx;

/* Per-head projection ("Базированная модель, часть 2", the paragraph on the
 * size of the hidden state: the KV and K states are made smaller by
 * projections of the input).  For sequence b and head hh:
 *     y[b][hh][t][d] = sum_k x[b][t][k] * w[hh*D + d][k]
 * i.e. x W^T split into H heads of D features, heads before positions. */
static void proj_heads_seq(void* p, int bh) {
    const proj_ctx* c = (const proj_ctx*)p;
    const int b = bh / c->H, hh = bh % c->H;
    for (int t = 0; t < c->L; ++t)
        for (int d = 0; d < c->D; ++d) {
            const double* xr = c->x + ((size_t)b * c->L + t) * c->Dm;
            const double* wr = c->w + ((size_t)hh * c->D + d) * c->Dm;
            c->y[(((size_t)b * c->H + hh) * c->L + t) * c->D + d] = dot(xr, wr, c->Dm);
        }
}

void oracle_proj_heads(const double* x, const double* w, double* y, int B, int L, int Dm,
                       int H, int D, int nthreads) {
    proj_ctx c = {x, w, NULL, NULL, y, L, Dm, H, D, 0};
    parallel_for(B * H, nthreads, proj_heads_seq, &c);
}

/* BaseConv ("Базированная модель, часть 1", section "Кто виноват?": the block
 * y = linear(x) (.) conv(h, x), with (.) the elementwise product and h a
 * filter).  linear is a dense D x D map with a bias; conv is the causal
 * convolution of each channel with its own filter of K taps:
 *     y[b][t][c] = (sum_k x[b][t][k] w[c][k] + bias[c])
 *                * sum_{j=0}^{min(K-1, t)} h[c][j] x[b][t-j][c]. */
static void baseconv_seq(void* p, int bt) {
    const proj_ctx* c = (const proj_ctx*)p;
    const int D = c->D, t = bt % c->L;
    for (int ch = 0; ch < D; ++ch) {
        const double* xr = c->x + (size_t)bt * D;
        const double lin = dot(xr, c->w + (size_t)ch * D, D) + c->bias[ch];
        double conv = 0.0;
        for (int j = 0; j < c->K && j <= t; ++j)
            conv += c->h[(size_t)ch * c->K + j] * c->x[((size_t)bt - j) * D + ch];
        c->y[(size_t)bt * D + ch] = lin * conv;
    }
}

void oracle_baseconv(const double* x, const double* w, const double* bias, const double* h,
                     double* y, int B, int L, int D, int K, int nthreads) {
    proj_ctx c = {x, w, bias, h, y, L, D, 0, D, K};
    parallel_for(B * L, nthreads, baseconv_seq, &c);
}

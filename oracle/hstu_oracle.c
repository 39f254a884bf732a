/*
 * hstu_oracle.c -- plain float64 CPU oracle for HSTU pointwise-aggregated attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
 * Python binding) may include, link or call this file.  It exists so that the tests,
 * the smoke check and the CPU-baseline leg of the benchmark have an independent,
 * slow, obviously correct statement of what the GPU library must compute.  It shares
 * no code, header, table or constant with the CUDA sources.
 *
 * What it computes (sources):
 *   - HSTU replaces softmax with SiLU weighting, adds a relative attention bias and
 *     gates elementwise before the output projection: aitrends.kr summary, section
 *     "HSTU의 순차 모델링" (HSTU sequential modelling); news.bpdata.com, section "HSTU".
 *   - Inputs are jagged (variable-length) per-user sequences, and in serving the history
 *     K/V come from a paged GPU KV table while only new tokens are computed and appended:
 *     NVIDIA blog "Deploying an HSTU Generative Recommender with NVIDIA Dynamo-Triton",
 *     section "Why serving large sequential recommenders is hard" (서빙이 어려운 이유),
 *     and the closing section on benefits (이점).
 *   - The exact per-head formula this library implements (the 1/n_max scale, the
 *     target-aware causal mask, LayerNorm over the token's H*d vector, gate by U) is the
 *     library's specification, restated in include/hstu.h:
 *
 *       allowed(i,j)  = (j <= i and j < Hist) or (i >= Hist and j == i)
 *                       Hist = L - num_targets (history length of the user)
 *       s(i,j,h)      = sum_c q[i,h,c] k[j,h,c] + rab[h][bucket(i - j)]
 *       w(i,j,h)      = allowed ? s * sigmoid(s) / n_max : 0
 *       o[i,h,:]      = sum_j w(i,j,h) v[j,h,:]
 *       out[i,h,c]    = (o[i,h,c] - mean_i) / sqrt(var_i + eps) * u[i,h,c]
 *                       mean_i, var_i over all H*d entries of o[i,:,:] (biased variance)
 *
 *   - bucket(0) = 0; for delta >= 1:
 *       bucket(delta) = min(NB - 1, 1 + floor((NB - 1) * ln(delta) / ln(n_max)))
 *     (log-spaced; bucket 0 reserved for a token attending to itself).  The pages name
 *     a relative bias but not its bucketing; this is the plainest log-spaced reading.
 *
 * Everything is float64, evaluated in the order written above.  Inputs may be given as
 * fp32 or as raw bf16 bit patterns; they are widened exactly to double on read.
 *
 * Parity pins (tests/test_oracle_pins.py) tie this file to closed forms, library
 * routines and invariants; the readings above that the pages do not fix (bucket shape,
 * LayerNorm axis, eps, n_max) are "parity unpinned" as readings.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Widen one stored element to double.  bf16 is the top half of an IEEE fp32. */
static double ld(const void* base, int64_t idx, int elem_type)
{
    if (elem_type == ORACLE_BF16) {
        uint16_t h = ((const uint16_t*)base)[idx];
        uint32_t bits = ((uint32_t)h) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float*)base)[idx];
}

/* Log-spaced relative-position bucket (see the header comment). */
int oracle_bucket(int64_t delta, int64_t n_max, int32_t num_buckets)
{
    if (num_buckets <= 1 || delta <= 0 || n_max <= 1)
        return 0;
    double x = (double)(num_buckets - 1) * log((double)delta) / log((double)n_max);
    int64_t b = 1 + (int64_t)floor(x);
    if (b > num_buckets - 1)
        b = num_buckets - 1;
    return (int)b;
}

/* Fill table[0..n) with bucket(delta). */
void oracle_bucket_table(int64_t n, int64_t n_max, int32_t num_buckets, int32_t* table)
{
    for (int64_t delta = 0; delta < n; ++delta)
        table[delta] = oracle_bucket(delta, n_max, num_buckets);
}

static double sigmoid(double s) { return 1.0 / (1.0 + exp(-s)); }

/*
 * One query row i of a user whose L keys/values have been gathered, in logical order, into
 * dense float64 arrays K and V of shape [L][H][D].  q and u are the query's [H][D] rows in
 * float64.  Writes the gated LayerNorm output row (H*D values) to out_row.
 */
typedef struct {
    int32_t H, D, NB;
    int64_t n_max;
    double eps;
    const float* rab;          /* [H][NB] */
} common_args;

static void one_query(const common_args* a, int64_t i, int64_t L, int64_t hist,
                      const double* q, const double* u, const double* K, const double* V,
                      double* o, double* out_row)
{
    const int32_t H = a->H, D = a->D;
    const int64_t HD = (int64_t)H * D;
    const double inv_n = 1.0 / (double)a->n_max;
    for (int32_t h = 0; h < H; ++h) {
        double* oh = o + (int64_t)h * D;
        for (int32_t c = 0; c < D; ++c)
            oh[c] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            int allowed = (j <= i && j < hist) || (i >= hist && j == i);
            if (!allowed)
                continue;   /* masked pairs contribute nothing, not even 0 * v */
            const double* kj = K + j * HD + (int64_t)h * D;
            const double* vj = V + j * HD + (int64_t)h * D;
            double s = 0.0;
            for (int32_t c = 0; c < D; ++c)
                s += q[(int64_t)h * D + c] * kj[c];
            s += (double)a->rab[(int64_t)h * a->NB + oracle_bucket(i - j, a->n_max, a->NB)];
            double w = s * sigmoid(s) * inv_n;
            for (int32_t c = 0; c < D; ++c)
                oh[c] += w * vj[c];
        }
    }
    /* LayerNorm over the H*D vector (two passes, biased variance), then gate by u. */
    double mean = 0.0;
    for (int64_t e = 0; e < HD; ++e)
        mean += o[e];
    mean /= (double)HD;
    double var = 0.0;
    for (int64_t e = 0; e < HD; ++e)
        var += (o[e] - mean) * (o[e] - mean);
    var /= (double)HD;
    double rstd = 1.0 / sqrt(var + a->eps);
    for (int64_t e = 0; e < HD; ++e)
        out_row[e] = (o[e] - mean) * rstd * u[e];
}

/* Per-thread scratch: the gathered K/V of the user handled last. */
typedef struct {
    int64_t user, cap;
    double *K, *V, *q, *u, *o;
} scratch;

static void scratch_init(scratch* s, int64_t HD)
{
    s->user = -1;
    s->cap = 0;
    s->K = s->V = NULL;
    s->q = (double*)malloc(sizeof(double) * HD);
    s->u = (double*)malloc(sizeof(double) * HD);
    s->o = (double*)malloc(sizeof(double) * HD);
}

static void scratch_reserve(scratch* s, int64_t L, int64_t HD)
{
    if (L > s->cap) {
        free(s->K);
        free(s->V);
        s->cap = L;
        s->K = (double*)malloc(sizeof(double) * L * HD);
        s->V = (double*)malloc(sizeof(double) * L * HD);
    }
}

static void scratch_free(scratch* s)
{
    free(s->K); free(s->V); free(s->q); free(s->u); free(s->o);
}

static int64_t user_of_token(const int64_t* off, int32_t B, int64_t t)
{
    int32_t lo = 0, hi = B;   /* b with off[b] <= t < off[b+1]; empty users are skipped */
    while (hi - lo > 1) {
        int32_t mid = (lo + hi) / 2;
        if (off[mid] <= t)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

static int run_jobs(void* jobs, size_t job_size, int32_t n, void* (*fn)(void*))
{
    if (n <= 1) {
        fn(jobs);
        return 0;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * n);
    for (int32_t t = 0; t < n; ++t)
        pthread_create(&th[t], NULL, fn, (char*)jobs + (size_t)t * job_size);
    for (int32_t t = 0; t < n; ++t)
        pthread_join(th[t], NULL);
    free(th);
    return 0;
}

/* ------------------------------------------------------------------ jagged */

typedef struct {
    common_args a;
    int elem_type;
    int32_t B;
    const int64_t* seq_offsets;
    const int64_t* num_targets;
    const void *q, *k, *v, *u;
    const int64_t* rows;       /* token indices to compute (n_rows of them) */
    int64_t n_rows;
    double* out;               /* [n_rows][H][D] */
    double* o_out;             /* optional [n_rows][H][D] pre-LayerNorm o, or NULL */
    int32_t nthreads, tid;
} jagged_job;

static void* jagged_worker(void* p)
{
    jagged_job* J = (jagged_job*)p;
    const common_args* a = &J->a;
    const int64_t HD = (int64_t)a->H * a->D;
    scratch s;
    scratch_init(&s, HD);
    for (int64_t r = J->tid; r < J->n_rows; r += J->nthreads) {
        int64_t t = J->rows[r];
        int64_t b = user_of_token(J->seq_offsets, J->B, t);
        int64_t start = J->seq_offsets[b];
        int64_t L = J->seq_offsets[b + 1] - start;
        int64_t hist = L - J->num_targets[b];
        if (s.user != b) {
            scratch_reserve(&s, L, HD);
            for (int64_t e = 0; e < L * HD; ++e) {
                s.K[e] = ld(J->k, start * HD + e, J->elem_type);
                s.V[e] = ld(J->v, start * HD + e, J->elem_type);
            }
            s.user = b;
        }
        for (int64_t e = 0; e < HD; ++e) {
            s.q[e] = ld(J->q, t * HD + e, J->elem_type);
            s.u[e] = ld(J->u, t * HD + e, J->elem_type);
        }
        one_query(a, t - start, L, hist, s.q, s.u, s.K, s.V, s.o, J->out + r * HD);
        if (J->o_out)
            memcpy(J->o_out + r * HD, s.o, sizeof(double) * HD);
    }
    scratch_free(&s);
    return NULL;
}

/*
 * Jagged prefill: every token of every user is a query.  rows == NULL computes all
 * tokens (out is [T][H][D]); otherwise only the listed token indices, in that order.
 * o_out, when not NULL, receives the pre-LayerNorm o rows (same shape as out).
 * Returns 0, or -1 on inconsistent lengths (num_targets > length, offsets decreasing).
 */
int oracle_hstu_jagged(int32_t B, int32_t H, int32_t D, const int64_t* seq_offsets,
                       const int64_t* num_targets, const void* q, const void* k, const void* v,
                       const void* u, int32_t elem_type, const float* rab, int32_t num_buckets,
                       int64_t n_max, double eps, const int64_t* rows, int64_t n_rows,
                       double* out, double* o_out, int32_t nthreads)
{
    for (int32_t b = 0; b < B; ++b) {
        int64_t L = seq_offsets[b + 1] - seq_offsets[b];
        if (L < 0 || num_targets[b] < 0 || num_targets[b] > L)
            return -1;
    }
    int64_t T = seq_offsets[B];
    int64_t* all = NULL;
    if (rows == NULL) {
        all = (int64_t*)malloc(sizeof(int64_t) * (T > 0 ? T : 1));
        for (int64_t t = 0; t < T; ++t)
            all[t] = t;
        rows = all;
        n_rows = T;
    }
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= T) {
            free(all);
            return -1;
        }
    if (nthreads < 1)
        nthreads = 1;
    jagged_job* jobs = (jagged_job*)calloc((size_t)nthreads, sizeof(jagged_job));
    for (int32_t t = 0; t < nthreads; ++t) {
        jagged_job* J = &jobs[t];
        J->a.H = H; J->a.D = D; J->a.NB = num_buckets; J->a.n_max = n_max;
        J->a.eps = eps; J->a.rab = rab; J->elem_type = elem_type;
        J->B = B; J->seq_offsets = seq_offsets; J->num_targets = num_targets;
        J->q = q; J->k = k; J->v = v; J->u = u;
        J->rows = rows; J->n_rows = n_rows; J->out = out; J->o_out = o_out;
        J->nthreads = nthreads; J->tid = t;
    }
    run_jobs(jobs, sizeof(jagged_job), nthreads, jagged_worker);
    free(jobs);
    free(all);
    return 0;
}

/* ------------------------------------------------------------------ paged */

typedef struct {
    common_args a;
    int elem_type;
    int32_t B, P, num_pages, max_pages;
    const int32_t* page_table;     /* [B][max_pages] */
    const int64_t *cached_lens, *new_lens, *num_targets, *new_offsets;
    const void *k_pages, *v_pages; /* [num_pages][H][P][D] */
    const void *q_new, *k_new, *v_new, *u_new;   /* [total_new][H][D] */
    const int64_t* rows;           /* indices into the new-token array */
    int64_t n_rows;
    double* out;
    double* o_out;                 /* optional pre-LayerNorm o, or NULL */
    int32_t nthreads, tid;
    int err;
} paged_job;

static void* paged_worker(void* p)
{
    paged_job* J = (paged_job*)p;
    const common_args* a = &J->a;
    const int32_t H = a->H, D = a->D, P = J->P;
    const int64_t HD = (int64_t)H * D;
    scratch s;
    scratch_init(&s, HD);
    for (int64_t r = J->tid; r < J->n_rows; r += J->nthreads) {
        int64_t t = J->rows[r];
        int64_t b = user_of_token(J->new_offsets, J->B, t);
        int64_t C = J->cached_lens[b], N = J->new_lens[b];
        int64_t L = C + N, hist = L - J->num_targets[b];
        if (s.user != b) {
            /* Concatenate: cached prefix through the page table, then the new tokens. */
            scratch_reserve(&s, L, HD);
            for (int64_t j = 0; j < L; ++j) {
                for (int32_t h = 0; h < H; ++h) {
                    for (int32_t c = 0; c < D; ++c) {
                        int64_t dst = j * HD + (int64_t)h * D + c;
                        if (j < C) {
                            int32_t page = J->page_table[(int64_t)b * J->max_pages + j / P];
                            if (page < 0 || page >= J->num_pages) {
                                J->err = -2;
                                s.K[dst] = s.V[dst] = 0.0;
                                continue;
                            }
                            int64_t idx = (((int64_t)page * H + h) * P + j % P) * D + c;
                            s.K[dst] = ld(J->k_pages, idx, J->elem_type);
                            s.V[dst] = ld(J->v_pages, idx, J->elem_type);
                        } else {
                            int64_t idx = (J->new_offsets[b] + (j - C)) * HD + (int64_t)h * D + c;
                            s.K[dst] = ld(J->k_new, idx, J->elem_type);
                            s.V[dst] = ld(J->v_new, idx, J->elem_type);
                        }
                    }
                }
            }
            s.user = b;
        }
        for (int64_t e = 0; e < HD; ++e) {
            s.q[e] = ld(J->q_new, t * HD + e, J->elem_type);
            s.u[e] = ld(J->u_new, t * HD + e, J->elem_type);
        }
        /* The query's absolute position in the user's sequence. */
        int64_t i = C + (t - J->new_offsets[b]);
        one_query(a, i, L, hist, s.q, s.u, s.K, s.V, s.o, J->out + r * HD);
        if (J->o_out)
            memcpy(J->o_out + r * HD, s.o, sizeof(double) * HD);
    }
    scratch_free(&s);
    return NULL;
}

/*
 * Paged cache hit: queries are the new tokens only.  User b's keys are its cached_lens[b]
 * history tokens, read from the pages listed in page_table[b] in logical order, followed
 * by its new_lens[b] new tokens (rows new_offsets[b].. of k_new/v_new, with new_offsets
 * the exclusive prefix sum of new_lens).  Query row t of the new-token array has
 * absolute position cached_lens[b] + (t - new_offsets[b]).  The last num_targets[b] new
 * tokens are the candidates.  rows == NULL computes every new token.  o_out, when not
 * NULL, receives the pre-LayerNorm o rows.
 * Returns 0, -1 on inconsistent lengths, -2 if a page id is out of range.
 */
int oracle_hstu_paged(int32_t B, int32_t H, int32_t D, int32_t page_size, int32_t num_pages,
                      int32_t max_pages, const int32_t* page_table, const int64_t* cached_lens,
                      const int64_t* new_lens, const int64_t* num_targets, const void* k_pages,
                      const void* v_pages, const void* q_new, const void* k_new, const void* v_new,
                      const void* u_new, int32_t elem_type, const float* rab, int32_t num_buckets,
                      int64_t n_max, double eps, const int64_t* rows, int64_t n_rows, double* out,
                      double* o_out, int32_t nthreads)
{
    int64_t* new_offsets = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    new_offsets[0] = 0;
    for (int32_t b = 0; b < B; ++b) {
        if (cached_lens[b] < 0 || new_lens[b] < 0 || num_targets[b] < 0 ||
            num_targets[b] > new_lens[b] || cached_lens[b] > (int64_t)max_pages * page_size) {
            free(new_offsets);
            return -1;
        }
        new_offsets[b + 1] = new_offsets[b] + new_lens[b];
    }
    int64_t T = new_offsets[B];
    int64_t* all = NULL;
    if (rows == NULL) {
        all = (int64_t*)malloc(sizeof(int64_t) * (T > 0 ? T : 1));
        for (int64_t t = 0; t < T; ++t)
            all[t] = t;
        rows = all;
        n_rows = T;
    }
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= T) {
            free(all);
            free(new_offsets);
            return -1;
        }
    if (nthreads < 1)
        nthreads = 1;
    paged_job* jobs = (paged_job*)calloc((size_t)nthreads, sizeof(paged_job));
    for (int32_t t = 0; t < nthreads; ++t) {
        paged_job* J = &jobs[t];
        J->a.H = H; J->a.D = D; J->a.NB = num_buckets; J->a.n_max = n_max;
        J->a.eps = eps; J->a.rab = rab; J->elem_type = elem_type;
        J->B = B; J->P = page_size; J->num_pages = num_pages; J->max_pages = max_pages;
        J->page_table = page_table; J->cached_lens = cached_lens; J->new_lens = new_lens;
        J->num_targets = num_targets; J->new_offsets = new_offsets;
        J->k_pages = k_pages; J->v_pages = v_pages;
        J->q_new = q_new; J->k_new = k_new; J->v_new = v_new; J->u_new = u_new;
        J->rows = rows; J->n_rows = n_rows; J->out = out; J->o_out = o_out;
        J->nthreads = nthreads; J->tid = t;
    }
    run_jobs(jobs, sizeof(paged_job), nthreads, paged_worker);
    int err = 0;
    for (int32_t t = 0; t < nthreads; ++t)
        if (jobs[t].err)
            err = jobs[t].err;
    free(jobs);
    free(all);
    free(new_offsets);
    return err;
}

/* ------------------------------------------------------------------ append */

/*
 * kv_append: for user b and t < append_lens[b], token row new_offsets[b] + t of k_new and
 * v_new ([rows][H][D], elem_bytes per element) is copied to logical position
 * p = cached_lens[b] + t of the user's pages: page page_table[b][p / P], slot p % P, i.e.
 * element [page][h][slot][c] of k_pages / v_pages ([num_pages][H][P][D]).
 * A raw byte copy.  Tokens whose page id is out of range, or whose logical page index is
 * beyond max_pages, are skipped and counted; the count is returned negated (0 = clean).
 */
int64_t oracle_kv_append(int32_t B, int32_t H, int32_t D, int32_t page_size, int32_t num_pages,
                         int32_t max_pages, int32_t elem_bytes, void* k_pages, void* v_pages,
                         const int32_t* page_table, const void* k_new, const void* v_new,
                         const int64_t* cached_lens, const int64_t* new_offsets,
                         const int64_t* append_lens)
{
    int64_t bad = 0;
    const size_t row = (size_t)D * (size_t)elem_bytes;
    for (int32_t b = 0; b < B; ++b) {
        for (int64_t t = 0; t < append_lens[b]; ++t) {
            int64_t pos = cached_lens[b] + t;
            int64_t lp = pos / page_size;
            if (lp >= max_pages) {
                ++bad;
                continue;
            }
            int32_t page = page_table[(int64_t)b * max_pages + lp];
            if (page < 0 || page >= num_pages) {
                ++bad;
                continue;
            }
            int64_t slot = pos % page_size;
            int64_t src_tok = new_offsets[b] + t;
            for (int32_t h = 0; h < H; ++h) {
                size_t dst = ((((size_t)page * H + h) * page_size + slot) * D) * elem_bytes;
                size_t src = (((size_t)src_tok * H + h) * D) * elem_bytes;
                memcpy((char*)k_pages + dst, (const char*)k_new + src, row);
                memcpy((char*)v_pages + dst, (const char*)v_new + src, row);
            }
        }
    }
    return -bad;
}

/* ------------------------------------------------------------------ jagged backward */

/*
 * Gradients of the jagged forward above for a given upstream gradient dout = dL/d out
 * (the backward pass of the same definition, by the chain rule, in float64):
 *
 *   out  = xhat * u,  xhat = (o - mean) * rstd      (per token, over its H*D vector)
 *   du   = xhat * dout
 *   dy   = dout * u
 *   do   = rstd * (dy - mean(dy) - xhat * mean(dy * xhat))        (LayerNorm backward)
 *   for every allowed pair (i, j) of a user and head h:
 *     s    = q_i . k_j + rab[h][bucket(i - j)],  sig = sigmoid(s)
 *     w    = s * sig / n_max
 *     dw   = do_i . v_j
 *     ds   = dw * sig * (1 + s * (1 - sig)) / n_max             (d SiLU(s) / ds)
 *     dq_i += ds * k_j;  dk_j += ds * q_i;  dv_j += w * do_i;  drab[h][bucket(i - j)] += ds
 *
 * dq, dk, dv, du: [T][H][D] float64, drab: [H][NB] float64, all overwritten.  Pairs are taken
 * in the order written (users, heads, queries, keys); no blocking or reordering.
 * Returns 0, or -1 on inconsistent lengths.
 */
int oracle_hstu_jagged_bwd(int32_t B, int32_t H, int32_t D, const int64_t* seq_offsets,
                           const int64_t* num_targets, const void* q, const void* k, const void* v,
                           const void* u, const void* dout, int32_t elem_type, const float* rab,
                           int32_t num_buckets, int64_t n_max, double eps, double* dq, double* dk,
                           double* dv, double* du, double* drab)
{
    for (int32_t b = 0; b < B; ++b) {
        int64_t L = seq_offsets[b + 1] - seq_offsets[b];
        if (L < 0 || num_targets[b] < 0 || num_targets[b] > L)
            return -1;
    }
    const int64_t T = seq_offsets[B];
    const int64_t HD = (int64_t)H * D;
    const double inv_n = 1.0 / (double)n_max;
    memset(dq, 0, sizeof(double) * (size_t)(T * HD));
    memset(dk, 0, sizeof(double) * (size_t)(T * HD));
    memset(dv, 0, sizeof(double) * (size_t)(T * HD));
    memset(du, 0, sizeof(double) * (size_t)(T * HD));
    memset(drab, 0, sizeof(double) * (size_t)((int64_t)H * num_buckets));
    double* o = (double*)malloc(sizeof(double) * (size_t)(HD > 0 ? HD : 1));
    double* dO = (double*)malloc(sizeof(double) * (size_t)(T * HD > 0 ? T * HD : 1));
    for (int32_t b = 0; b < B; ++b) {
        const int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0;
        const int64_t hist = L - num_targets[b];
        /* forward o and the LayerNorm backward, token by token */
        for (int64_t i = 0; i < L; ++i) {
            for (int32_t h = 0; h < H; ++h)
                for (int32_t c = 0; c < D; ++c) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < L; ++j) {
                        int allowed = (j <= i && j < hist) || (i >= hist && j == i);
                        if (!allowed)
                            continue;
                        double s = 0.0;
                        for (int32_t e = 0; e < D; ++e)
                            s += ld(q, (s0 + i) * HD + (int64_t)h * D + e, elem_type) *
                                 ld(k, (s0 + j) * HD + (int64_t)h * D + e, elem_type);
                        s += (double)rab[(int64_t)h * num_buckets + oracle_bucket(i - j, n_max, num_buckets)];
                        acc += s * sigmoid(s) * inv_n * ld(v, (s0 + j) * HD + (int64_t)h * D + c, elem_type);
                    }
                    o[(int64_t)h * D + c] = acc;
                }
            double mean = 0.0;
            for (int64_t e = 0; e < HD; ++e)
                mean += o[e];
            mean /= (double)HD;
            double var = 0.0;
            for (int64_t e = 0; e < HD; ++e)
                var += (o[e] - mean) * (o[e] - mean);
            var /= (double)HD;
            const double rstd = 1.0 / sqrt(var + eps);
            double mdy = 0.0, mdyx = 0.0;
            for (int64_t e = 0; e < HD; ++e) {
                const int64_t idx = (s0 + i) * HD + e;
                const double xhat = (o[e] - mean) * rstd;
                const double g = ld(dout, idx, elem_type);
                du[idx] = xhat * g;
                const double dy = g * ld(u, idx, elem_type);
                mdy += dy;
                mdyx += dy * xhat;
            }
            mdy /= (double)HD;
            mdyx /= (double)HD;
            for (int64_t e = 0; e < HD; ++e) {
                const int64_t idx = (s0 + i) * HD + e;
                const double xhat = (o[e] - mean) * rstd;
                const double dy = ld(dout, idx, elem_type) * ld(u, idx, elem_type);
                dO[idx] = rstd * (dy - mdy - xhat * mdyx);
            }
        }
        /* attention backward over the allowed pairs */
        for (int32_t h = 0; h < H; ++h)
            for (int64_t i = 0; i < L; ++i)
                for (int64_t j = 0; j < L; ++j) {
                    int allowed = (j <= i && j < hist) || (i >= hist && j == i);
                    if (!allowed)
                        continue;
                    const int64_t qi = (s0 + i) * HD + (int64_t)h * D, kj = (s0 + j) * HD + (int64_t)h * D;
                    const int bk = oracle_bucket(i - j, n_max, num_buckets);
                    double s = 0.0, dw = 0.0;
                    for (int32_t e = 0; e < D; ++e) {
                        s += ld(q, qi + e, elem_type) * ld(k, kj + e, elem_type);
                        dw += dO[qi + e] * ld(v, kj + e, elem_type);
                    }
                    s += (double)rab[(int64_t)h * num_buckets + bk];
                    const double sig = sigmoid(s);
                    const double w = s * sig * inv_n;
                    const double ds = dw * sig * (1.0 + s * (1.0 - sig)) * inv_n;
                    for (int32_t e = 0; e < D; ++e) {
                        dq[qi + e] += ds * ld(k, kj + e, elem_type);
                        dk[kj + e] += ds * ld(q, qi + e, elem_type);
                        dv[kj + e] += w * dO[qi + e];
                    }
                    drab[(int64_t)h * num_buckets + bk] += ds;
                }
    }
    free(o);
    free(dO);
    return 0;
}

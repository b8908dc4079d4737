/*
 * kvc_oracle.c -- plain fp64 CPU oracle for attention-saliency KV-cache compaction.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this
 * file or the library built from it.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; the two meet only in the seeded input generator.
 *
 * What it computes, step by step, in the order the method is described:
 *
 *   score   The saliency of a cached token is the softmaxed attention it receives from the
 *           last `w` queries (the observation window).  SnapKV is the decoding-time
 *           compressor that scores this way (FastKV page, sec. 1 "Problemstellung", and
 *           StructKV page, "Probleemstelling"); FastKV's TSP layer selects tokens by such
 *           a saliency score (FastKV page, sec. 2A "Token-Selective Propagation").
 *           Window query i of head g sits at position t_i = N - w + i and sees keys
 *           j <= t_i (causal).  x_j = q.k_j / sqrt(D); p_j = exp(x_j - m) / l with
 *           m = max_j x_j and l = sum_j exp(x_j - m) over the visible keys.
 *   aggregate
 *           The per-KV-head score sums p over the window queries and over the G query
 *           heads that share the KV head (q head g reads KV head g / G).  For TSP and for
 *           StructKV the sum also runs over all heads; StructKV further sums over all
 *           layers up to the pivot (StructKV page, sec. 1 "Global In-Degree Centrality").
 *   pool    1-D max-pool of odd width P over the candidate range C = [S, N - w), edges
 *           clipped to C.
 *   select  The k_sel = budget - S - w largest pooled scores on C, ties to the lower
 *           index; kept = sinks [0, S)  U  selected  U  recent window [N - w, N), in
 *           ascending order.  Sinks and recent tokens are always kept (CentroidKV page,
 *           "Inferentie Pipeline", Preservation; FastKV page, sec. 2A: the selected
 *           tokens plus a window of the newest tokens are propagated).
 *   gather  Row r of the compact cache is the source row idx[r], byte for byte.
 *   pivot metrics
 *           StructKV watches attention entropy, sparsity and variance during the first
 *           pass to find the layer where attention settles (StructKV page, sec. 2
 *           "Dynamische Pivot Detectie"); the page gives no formulas.  Read here as: the
 *           Shannon entropy (nats) of each window query's attention row; the share of a
 *           score row's mass that the kept positions hold; the population variance of a
 *           score row over the candidates C.
 *   clustering and decode attention
 *           CentroidKV merges similar tokens into degree-weighted centroids instead of
 *           evicting them (Chunked Soft Matching, CentroidKV page, sec. 3-4) and attends to
 *           the centroids with the log of their degree added to the logits (sec. 4).
 *
 * Everything is done in double precision with plain loops; inputs arrive as raw fp32 or
 * bf16 bytes and are widened exactly.  Parallelism, where present, is only over
 * independent (layer, batch, KV head) units, and partial results are combined in a fixed
 * order so that the output does not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };
enum { OR_SCOPE_PER_KV_HEAD = 0, OR_SCOPE_ALL_HEADS = 1 };

/* Exact widening of one element to double. */
static double widen(const void *base, int dtype, size_t i)
{
    if (dtype == OR_F32) return (double)((const float *)base)[i];
    if (dtype == OR_F64) return ((const double *)base)[i];
    /* bf16: the upper half of an IEEE binary32 */
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------------------ */
/* score: one (layer, batch, KV head) unit                                               */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    int B, Hq, Hkv, N, D, w, L, dtype;
    const void *q, *k;
    double *unit_scores; /* [L*B*Hkv][N] */
    int next_unit, n_units;
    pthread_mutex_t lock;
} score_job;

/* s[j] = sum over the G heads of KV head h and the w window queries of p_{g,i,j}. */
static void score_unit(const score_job *J, int unit, double *row)
{
    const int N = J->N, D = J->D, w = J->w, G = J->Hq / J->Hkv;
    const int h = unit % J->Hkv;
    const int b = (unit / J->Hkv) % J->B;
    const int layer = unit / (J->Hkv * J->B);
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double *s = J->unit_scores + (size_t)unit * N;
    for (int j = 0; j < N; ++j) s[j] = 0.0;

    /* K rows of this unit start here (layout [L][B][Hkv][N][D]) */
    const size_t k_base = (((size_t)layer * J->B + b) * J->Hkv + h) * (size_t)N * D;
    for (int gg = 0; gg < G; ++gg) {
        const int g = h * G + gg;
        for (int i = 0; i < w; ++i) {
            /* query row (layout [L][B][Hq][w][D]) */
            const size_t q_base = ((((size_t)layer * J->B + b) * J->Hq + g) * w + i) * (size_t)D;
            const int t = N - w + i; /* position of this window query */
            double m = -INFINITY;
            for (int j = 0; j <= t; ++j) {
                double x = 0.0;
                for (int d = 0; d < D; ++d)
                    x += widen(J->q, J->dtype, q_base + d) * widen(J->k, J->dtype, k_base + (size_t)j * D + d);
                row[j] = x * inv_sqrt_d;
                if (row[j] > m) m = row[j];
            }
            double l = 0.0;
            for (int j = 0; j <= t; ++j) l += exp(row[j] - m);
            for (int j = 0; j <= t; ++j) s[j] += exp(row[j] - m) / l;
            /* keys j > t are masked: they receive nothing from this query */
        }
    }
}

static void *score_worker(void *arg)
{
    score_job *J = (score_job *)arg;
    double *row = (double *)malloc(sizeof(double) * (size_t)J->N);
    if (!row) return (void *)1;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        score_unit(J, u, row);
    }
    free(row);
    return NULL;
}

/*
 * oracle_score -- per-token saliency scores, summed over window queries and heads, and
 * over layers.
 *   q       [L, B, Hq, w, D]      fp32 / bf16 / fp64 (dtype)
 *   k       [L, B, Hkv, N, D]     same dtype
 *   scores  scope PER_KV_HEAD: [B, Hkv, N];  scope ALL_HEADS: [B, 1, N]   (fp64, written)
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_score(int B, int Hq, int Hkv, int N, int D, int w, int L, int scope,
                 const void *q, const void *k, int dtype, double *scores, int n_threads)
{
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || N < 1 || D < 1 || w < 1 || w > N || L < 1) return -1;
    if (scope != OR_SCOPE_PER_KV_HEAD && scope != OR_SCOPE_ALL_HEADS) return -1;
    score_job J;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.N = N; J.D = D; J.w = w; J.L = L; J.dtype = dtype;
    J.q = q; J.k = k;
    J.n_units = L * B * Hkv;
    J.next_unit = 0;
    J.unit_scores = (double *)malloc(sizeof(double) * (size_t)J.n_units * N);
    if (!J.unit_scores) return -1;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > J.n_units) n_threads = J.n_units;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int rc = 0;
    for (int t = 1; t < n_threads; ++t) pthread_create(&th[t], NULL, score_worker, &J);
    if (score_worker(&J)) rc = -1;
    for (int t = 1; t < n_threads; ++t) {
        void *r;
        pthread_join(th[t], &r);
        if (r) rc = -1;
    }
    free(th);
    pthread_mutex_destroy(&J.lock);

    /* fixed-order reduction: over layers, then (for ALL_HEADS) over KV heads */
    const int Hs = scope == OR_SCOPE_PER_KV_HEAD ? Hkv : 1;
    memset(scores, 0, sizeof(double) * (size_t)B * Hs * N);
    for (int layer = 0; layer < L; ++layer)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < Hkv; ++h) {
                const double *src = J.unit_scores + (((size_t)layer * B + b) * Hkv + h) * N;
                double *dst = scores + ((size_t)b * Hs + (Hs == 1 ? 0 : h)) * N;
                for (int j = 0; j < N; ++j) dst[j] += src[j];
            }
    free(J.unit_scores);
    return rc;
}

/*
 * oracle_accumulate -- acc[b, o, j] += sum over the Hi/Ho source heads i of group o of
 * src[b, i, j].  Group o holds source heads o*(Hi/Ho) ... (o+1)*(Hi/Ho)-1.
 */
int oracle_accumulate(double *acc, const double *src, int B, int Hi, int Ho, int N)
{
    if (B < 1 || Hi < 1 || Ho < 1 || Hi % Ho || N < 0) return -1;
    const int R = Hi / Ho;
    for (int b = 0; b < B; ++b)
        for (int o = 0; o < Ho; ++o)
            for (int r = 0; r < R; ++r) {
                const double *s = src + ((size_t)b * Hi + o * R + r) * N;
                double *a = acc + ((size_t)b * Ho + o) * N;
                for (int j = 0; j < N; ++j) a[j] += s[j];
            }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* pool                                                                                  */
/* ------------------------------------------------------------------------------------ */

/*
 * oracle_pool -- out[j] = max{ in[t] : lo <= t < hi, |t - j| <= (P-1)/2 } for lo <= j < hi;
 * out[j] = in[j] outside [lo, hi).  Rows of length N, B*H rows.  P must be odd and >= 1.
 */
int oracle_pool(const double *in, double *out, int B, int H, int N, int lo, int hi, int P)
{
    if (B < 1 || H < 1 || N < 0 || lo < 0 || hi > N || lo > hi || P < 1 || P % 2 == 0) return -1;
    const int r = (P - 1) / 2;
    for (size_t row = 0; row < (size_t)B * H; ++row) {
        const double *a = in + row * N;
        double *o = out + row * N;
        for (int j = 0; j < N; ++j) {
            if (j < lo || j >= hi) { o[j] = a[j]; continue; }
            int t0 = j - r < lo ? lo : j - r;
            int t1 = j + r > hi - 1 ? hi - 1 : j + r;
            double m = a[t0];
            for (int t = t0 + 1; t <= t1; ++t)
                if (a[t] > m) m = a[t];
            o[j] = m;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* select                                                                                */
/* ------------------------------------------------------------------------------------ */

typedef struct { double v; int j; } cand;

/* larger score first; equal scores: lower index first */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand *a = (const cand *)pa, *b = (const cand *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int int_cmp(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/*
 * oracle_select -- per row: sort the candidates C = [S, N - w) by (score desc, index asc),
 * keep the first budget - S - w, add the sinks [0, S) and the window [N - w, N), and write
 * the `budget` kept positions in ascending order to idx[row][0..budget).
 * Requires S >= 0, w >= 0, budget >= S + w + 1 and budget <= N.
 */
int oracle_select(const double *pooled, int B, int H, int N, int S, int w, int budget, int32_t *idx)
{
    if (B < 1 || H < 1 || S < 0 || w < 0 || budget < S + w + 1 || budget > N) return -1;
    const int n_c = N - w - S;
    const int k_sel = budget - S - w;
    cand *c = (cand *)malloc(sizeof(cand) * (size_t)(n_c > 0 ? n_c : 1));
    int *kept = (int *)malloc(sizeof(int) * (size_t)budget);
    if (!c || !kept) { free(c); free(kept); return -1; }
    for (size_t row = 0; row < (size_t)B * H; ++row) {
        const double *s = pooled + row * N;
        for (int t = 0; t < n_c; ++t) { c[t].v = s[S + t]; c[t].j = S + t; }
        qsort(c, (size_t)n_c, sizeof(cand), cand_cmp);
        int n = 0;
        for (int j = 0; j < S; ++j) kept[n++] = j;
        for (int t = 0; t < k_sel; ++t) kept[n++] = c[t].j;
        for (int j = N - w; j < N; ++j) kept[n++] = j;
        qsort(kept, (size_t)n, sizeof(int), int_cmp);
        for (int t = 0; t < budget; ++t) idx[row * budget + t] = kept[t];
    }
    free(c);
    free(kept);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* gather                                                                                */
/* ------------------------------------------------------------------------------------ */

/*
 * oracle_gather -- dst[b, h, r, :] = src[b, h, idx[b, h', r], :] with h' = h when
 * Hidx == Hsrc and h' = 0 when Hidx == 1.  Rows are `row_bytes` raw bytes.
 */
int oracle_gather(const void *src, int B, int Hsrc, int N, size_t row_bytes,
                  const int32_t *idx, int Hidx, int K, void *dst)
{
    if (B < 1 || Hsrc < 1 || N < 1 || K < 0 || (Hidx != 1 && Hidx != Hsrc)) return -1;
    const unsigned char *s = (const unsigned char *)src;
    unsigned char *d = (unsigned char *)dst;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hsrc; ++h)
            for (int r = 0; r < K; ++r) {
                int j = idx[((size_t)b * Hidx + (Hidx == 1 ? 0 : h)) * K + r];
                if (j < 0 || j >= N) return -1;
                memcpy(d + (((size_t)b * Hsrc + h) * K + r) * row_bytes,
                       s + (((size_t)b * Hsrc + h) * N + j) * row_bytes, row_bytes);
            }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* TSP row count                                                                         */
/* ------------------------------------------------------------------------------------ */

/*
 * oracle_tsp_count -- rows propagated by Token-Selective Propagation: floor(rate * N)
 * selected tokens (at most the N - S - w candidates) plus the S sinks and the w recent
 * tokens.  The TSP rate is its own knob, separate from the KV-retention budget (FastKV
 * page, sec. 2B "Entkoppelte KV-Cache-Reduktion").  Returns 0 when rate <= 0 or when
 * floor(rate * N) < 1 (no token would be selected).
 */
int oracle_tsp_count(int N, int w, int S, double rate)
{
    if (rate <= 0.0) return 0;
    long sel = (long)floor(rate * (double)N);
    long n_c = (long)N - w - S;
    if (sel > n_c) sel = n_c;
    if (sel < 1) return 0; /* nothing to select: not a valid TSP configuration */
    return (int)(sel + S + w);
}

/* ------------------------------------------------------------------------------------ */
/* pivot metrics                                                                         */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    int B, Hq, Hkv, N, D, w, dtype;
    const void *q, *k;
    const int32_t *rows;
    int n_rows, next;
    double *out;
    pthread_mutex_t lock;
} entropy_job;

/* H = -sum_j p_j ln p_j over the keys j <= t that flat query row r sees. */
static double row_entropy(const entropy_job *J, int r, double *x)
{
    const int N = J->N, D = J->D, w = J->w, G = J->Hq / J->Hkv;
    const int i = r % w;
    const int g = (r / w) % J->Hq;
    const int lb = r / (w * J->Hq); /* layer * B + b */
    const int h = g / G;
    const double scale = 1.0 / sqrt((double)J->D);
    const size_t q_base = (size_t)r * D;
    const size_t k_base = ((size_t)lb * J->Hkv + h) * (size_t)N * D;
    const int last = N - w + i; /* the row's position: keys 0..last are visible */
    double m = -INFINITY;
    for (int j = 0; j <= last; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += widen(J->q, J->dtype, q_base + d) * widen(J->k, J->dtype, k_base + (size_t)j * D + d);
        x[j] = acc * scale;
        if (x[j] > m) m = x[j];
    }
    double l = 0.0;
    for (int j = 0; j <= last; ++j) l += exp(x[j] - m);
    double H = 0.0;
    for (int j = 0; j <= last; ++j) {
        const double p = exp(x[j] - m) / l;
        if (p > 0.0) H -= p * log(p);
    }
    return H;
}

static void *entropy_worker(void *arg)
{
    entropy_job *J = (entropy_job *)arg;
    double *x = (double *)malloc(sizeof(double) * (size_t)J->N);
    if (!x) return (void *)1;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int n = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (n >= J->n_rows) break;
        J->out[n] = row_entropy(J, J->rows[n], x);
    }
    free(x);
    return NULL;
}

/*
 * oracle_entropy -- attention entropy (nats) of window query rows.
 *   q [L, B, Hq, w, D], k [L, B, Hkv, N, D] (dtype as in oracle_score); rows[n] is a flat
 *   query-row index ((layer * B + b) * Hq + g) * w + i; out[n] = -sum_j p_j ln p_j of that
 *   row's causal window softmax.
 */
int oracle_entropy(int B, int Hq, int Hkv, int N, int D, int w, int L, const void *q, const void *k,
                   int dtype, const int32_t *rows, int n_rows, double *out, int n_threads)
{
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || N < 1 || D < 1 || w < 1 || w > N || L < 1 || n_rows < 0)
        return -1;
    for (int n = 0; n < n_rows; ++n)
        if (rows[n] < 0 || rows[n] >= L * B * Hq * w) return -1;
    entropy_job J;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.N = N; J.D = D; J.w = w; J.dtype = dtype;
    J.q = q; J.k = k; J.rows = rows; J.n_rows = n_rows; J.next = 0; J.out = out;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_rows) n_threads = n_rows > 0 ? n_rows : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int rc = 0;
    for (int t = 1; t < n_threads; ++t) pthread_create(&th[t], NULL, entropy_worker, &J);
    if (entropy_worker(&J)) rc = -1;
    for (int t = 1; t < n_threads; ++t) {
        void *r;
        pthread_join(th[t], &r);
        if (r) rc = -1;
    }
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}

/*
 * oracle_row_stats -- per score row s (rows of length N):
 *   kept_mass[row] = sum of s over the row's `budget` positions in idx / sum_{j < N} s
 *                    (skipped when idx is NULL)
 *   cand_var[row]  = (1/n) sum_{j in C} (s_j - mean_C)^2 over the n = N - w - S candidates
 *                    C = [S, N - w), mean_C their mean (two passes)
 */
int oracle_row_stats(const double *scores, int rows, int N, int S, int w, const int32_t *idx, int budget,
                     double *kept_mass, double *cand_var)
{
    if (rows < 1 || N < 1 || S < 0 || w < 0 || S + w >= N || (idx && (budget < 1 || budget > N))) return -1;
    const int n_c = N - w - S;
    for (int row = 0; row < rows; ++row) {
        const double *s = scores + (size_t)row * N;
        if (idx) {
            double total = 0.0, kept = 0.0;
            for (int j = 0; j < N; ++j) total += s[j];
            for (int t = 0; t < budget; ++t) {
                const int j = idx[(size_t)row * budget + t];
                if (j < 0 || j >= N) return -1;
                kept += s[j];
            }
            kept_mass[row] = kept / total;
        }
        double mean = 0.0;
        for (int j = S; j < N - w; ++j) mean += s[j];
        mean /= n_c;
        double var = 0.0;
        for (int j = S; j < N - w; ++j) var += (s[j] - mean) * (s[j] - mean);
        cand_var[row] = var / n_c;
    }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Chunked Soft Matching (CentroidKV)                                                    */
/* ------------------------------------------------------------------------------------ */

/*
 * CentroidKV clusters KV states instead of evicting them (CentroidKV page, sec. 3 "Chunked
 * Soft Matching" and sec. 4 "Aggregatie"):
 *   chunks     the candidates C = [S, N - w) are cut into chunks of `chunk` tokens (sinks and
 *              the recent window stay as they are: sec. 2, Preservation);
 *   partition  inside a chunk, tokens alternate between set A (even offset) and set B (odd);
 *   matching   each A token's match is the B token of its chunk with the largest cosine
 *              similarity of the key states (ties: lower position; a zero key has
 *              similarity 0); an A token alone in its chunk has no match;
 *   merge      the matches are ranked by similarity and only the top fraction merges:
 *              m = min(floor(r * |C|), matchable A tokens) of them (ties: lower position);
 *   aggregate  a B token and the A tokens merged into it become their degree-weighted
 *              mean, K and V alike; degrees add (sec. 4: n_t counts the merged tokens).
 * The cache keeps every token except the merged A tokens, in position order.
 */

static double key_dot(const void *k, int dtype, size_t ra, size_t rb, int D)
{
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += widen(k, dtype, ra * D + d) * widen(k, dtype, rb * D + d);
    return s;
}

/* Rounds v to the element type (bf16: round to nearest even; f32: nearest) and stores it. */
static void store_elem(void *dst, int dtype, size_t i, double v)
{
    if (dtype == OR_F64) { ((double *)dst)[i] = v; return; }
    float f = (float)v;
    if (dtype == OR_F32) { ((float *)dst)[i] = f; return; }
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    if ((bits & 0x7F800000u) == 0x7F800000u && (bits & 0x007FFFFFu)) { /* NaN stays NaN */
        ((uint16_t *)dst)[i] = (uint16_t)((bits >> 16) | 0x40u);
        return;
    }
    /* v -> float may already round; redo from v in double for an exact bf16 RNE */
    double av = fabs(v);
    if (av == 0.0) { ((uint16_t *)dst)[i] = (uint16_t)(bits >> 16); return; }
    int e;
    frexp(av, &e);                                  /* av = f * 2^e, f in [0.5, 1) */
    double ulp = ldexp(1.0, (e < -125 ? -125 : e) - 8); /* bf16 spacing at av */
    double q = nearbyint(av / ulp) * ulp;           /* round half to even (default mode) */
    float qf = (float)(v < 0 ? -q : q);
    memcpy(&bits, &qf, sizeof bits);
    ((uint16_t *)dst)[i] = (uint16_t)(bits >> 16);
}

/* Merges m of a row's A tokens; see above.  Outputs per row: best[N] (match position or -1),
 * sim[N] (match similarity, -inf when there is none), merged[N] (0/1), and the kept rows. */
static int csm_row(const void *k, const void *v, int dtype, const int32_t *deg, int N, int D, int S, int w,
                   int chunk, int m, int32_t *best, double *sim, unsigned char *merged,
                   void *k_out, void *v_out, int32_t *deg_out, int32_t *pos_out)
{
    const int lo = S, hi = N - w;
    for (int j = 0; j < N; ++j) { best[j] = -1; sim[j] = -INFINITY; merged[j] = 0; }
    for (int c0 = lo; c0 < hi; c0 += chunk) {
        const int c1 = c0 + chunk < hi ? c0 + chunk : hi;
        for (int a = c0; a < c1; a += 2) {
            const double na = sqrt(key_dot(k, dtype, a, a, D));
            for (int b = c0 + 1; b < c1; b += 2) {
                const double nb = sqrt(key_dot(k, dtype, b, b, D));
                const double s = (na > 0.0 && nb > 0.0) ? key_dot(k, dtype, a, b, D) / (na * nb) : 0.0;
                if (best[a] < 0 || s > sim[a]) { best[a] = b; sim[a] = s; }
            }
        }
    }
    /* the m matches with the largest similarity, ties to the lower position */
    int n_a = 0;
    for (int j = lo; j < hi; ++j)
        if (best[j] >= 0) ++n_a;
    cand *c = (cand *)malloc(sizeof(cand) * (size_t)(n_a > 0 ? n_a : 1));
    if (!c) return -1;
    int t = 0;
    for (int j = lo; j < hi; ++j)
        if (best[j] >= 0) { c[t].v = sim[j]; c[t].j = j; ++t; }
    qsort(c, (size_t)n_a, sizeof(cand), cand_cmp);
    for (int q = 0; q < m && q < n_a; ++q) merged[c[q].j] = 1;
    free(c);
    /* kept rows in position order; a B token absorbs the A tokens merged into it */
    double *acc_k = (double *)malloc(sizeof(double) * (size_t)D), *acc_v = (double *)malloc(sizeof(double) * (size_t)D);
    if (!acc_k || !acc_v) { free(acc_k); free(acc_v); return -1; }
    int o = 0;
    for (int j = 0; j < N; ++j) {
        if (merged[j]) continue;
        long long n = deg[j];
        for (int d = 0; d < D; ++d) {
            acc_k[d] = (double)deg[j] * widen(k, dtype, (size_t)j * D + d);
            acc_v[d] = (double)deg[j] * widen(v, dtype, (size_t)j * D + d);
        }
        if (j >= lo && j < hi && (j - lo) % chunk % 2 == 1) {
            const int c0 = lo + (j - lo) / chunk * chunk;
            const int c1 = c0 + chunk < hi ? c0 + chunk : hi;
            for (int a = c0; a < c1; a += 2)
                if (merged[a] && best[a] == j) {
                    n += deg[a];
                    for (int d = 0; d < D; ++d) {
                        acc_k[d] += (double)deg[a] * widen(k, dtype, (size_t)a * D + d);
                        acc_v[d] += (double)deg[a] * widen(v, dtype, (size_t)a * D + d);
                    }
                }
        }
        for (int d = 0; d < D; ++d) {
            store_elem(k_out, dtype, (size_t)o * D + d, acc_k[d] / (double)n);
            store_elem(v_out, dtype, (size_t)o * D + d, acc_v[d] / (double)n);
        }
        deg_out[o] = (int32_t)n;
        pos_out[o] = j;
        ++o;
    }
    free(acc_k);
    free(acc_v);
    return o;
}

/*
 * oracle_csm_merges -- m = min(floor(r * |C|), matchable A tokens) for a row of N tokens.
 * An A token is matchable when its chunk holds a B token: every A token except one alone in
 * the last chunk.
 */
int oracle_csm_merges(int N, int S, int w, int chunk, double r)
{
    if (N < 1 || S < 0 || w < 0 || S + w > N || chunk < 2 || chunk % 2 || !(r >= 0.0 && r <= 0.5)) return -1;
    const int n_c = N - w - S;
    int n_a = 0;
    for (int c0 = 0; c0 < n_c; c0 += chunk) {
        const int len = c0 + chunk < n_c ? chunk : n_c - c0;
        if (len >= 2) n_a += (len + 1) / 2;
    }
    const long m = (long)floor(r * (double)n_c);
    return (int)(m < n_a ? m : n_a);
}

/*
 * oracle_csm -- one Chunked Soft Matching round over rows of [rows, N, D] K and V (dtype as
 * in oracle_score; fp64 arithmetic, outputs rounded to the same dtype) with degrees
 * deg[rows][N].  Outputs per row: best, sim, merged as in csm_row; k_out, v_out
 * [rows][N - m][D], deg_out and pos_out [rows][N - m].  Returns N - m, or -1 on bad
 * arguments.
 */
int oracle_csm(const void *k, const void *v, int dtype, const int32_t *deg, int rows, int N, int D, int S, int w,
               int chunk, double r, int32_t *best, double *sim, unsigned char *merged, void *k_out, void *v_out,
               int32_t *deg_out, int32_t *pos_out)
{
    const int m = oracle_csm_merges(N, S, w, chunk, r);
    if (m < 0 || rows < 1 || D < 1) return -1;
    const size_t esz = dtype == OR_F32 ? 4 : dtype == OR_F64 ? 8 : 2;
    const int n_out = N - m;
    for (int row = 0; row < rows; ++row) {
        const size_t in = (size_t)row * N, out = (size_t)row * n_out;
        const int o = csm_row((const char *)k + in * D * esz, (const char *)v + in * D * esz, dtype, deg + in, N, D,
                              S, w, chunk, m, best + in, sim + in, merged + in, (char *)k_out + out * D * esz,
                              (char *)v_out + out * D * esz, deg_out + out, pos_out + out);
        if (o != n_out) return -1;
    }
    return n_out;
}

/* The progressive schedule of the merge ratio over rounds (CentroidKV page, sec. 3):
 * r_j = r_init - j * delta, not below 0. */
double oracle_csm_ratio(double r_init, double delta, int round)
{
    const double r = r_init - (double)round * delta;
    return r > 0.0 ? r : 0.0;
}

/* ------------------------------------------------------------------------------------ */
/* Decode attention over a clustered cache (CentroidKV)                                  */
/* ------------------------------------------------------------------------------------ */

/*
 * oracle_centroid_attention -- attention of decode queries over a cache of centroids whose
 * degrees enter the softmax as a log term (CentroidKV page, sec. 4 "Aggregatie": the
 * cluster degree is added to the softmax as a log-term so that attention over a centroid
 * approximates attention over the tokens it replaced).  Read as: a centroid of degree n
 * weighs like n copies of itself, i.e. its logit gains ln n:
 *     x_t = q . k_t / sqrt(D) + ln n_t,   p = softmax_t(x),   out = sum_t p_t v_t
 * over all n cached rows (no mask: every cached row precedes the decode queries).
 * Layouts: q [B][Hq][nq][D], k and v [B][Hkv][n][D] (kv_dtype), deg [B][Hkv][n] or NULL
 * (all degrees 1: plain attention), out [B][Hq][nq][D] fp64.  Query head g reads KV head
 * g / (Hq / Hkv).  Returns 0, or -1 on bad arguments.
 */
int oracle_centroid_attention(const void *q, int q_dtype, const void *k, const void *v, int kv_dtype,
                              const int32_t *deg, int B, int Hq, int Hkv, int nq, int n, int D, double *out)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || nq < 1 || n < 1 || D < 1) return -1;
    const int G = Hq / Hkv;
    const double sqrt_d = sqrt((double)D);
    double *x = (double *)malloc(sizeof(double) * (size_t)n);
    if (!x) return -1;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hq; ++g) {
            const int kvh = g / G;
            const size_t kv_row0 = ((size_t)b * Hkv + kvh) * n;
            for (int i = 0; i < nq; ++i) {
                const size_t q0 = (((size_t)b * Hq + g) * nq + i) * D;
                double m = -INFINITY;
                for (int t = 0; t < n; ++t) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += widen(q, q_dtype, q0 + d) * widen(k, kv_dtype, (kv_row0 + t) * D + d);
                    x[t] = dot / sqrt_d + (deg ? log((double)deg[kv_row0 + t]) : 0.0);
                    if (x[t] > m) m = x[t];
                }
                double l = 0.0;
                for (int t = 0; t < n; ++t) l += exp(x[t] - m);
                double *o = out + q0;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int t = 0; t < n; ++t) {
                    const double p = exp(x[t] - m) / l;
                    for (int d = 0; d < D; ++d) o[d] += p * widen(v, kv_dtype, (kv_row0 + t) * D + d);
                }
            }
        }
    free(x);
    return 0;
}

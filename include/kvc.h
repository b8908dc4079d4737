/*
 * kvc.h -- C ABI of libkvc.so: attention-saliency KV-cache compaction on NVIDIA B200
 * (sm_100a).
 *
 * The library scores every cached token by the softmaxed attention of the last `window`
 * queries, sums the scores over the window, the GQA group and optionally over all heads
 * and layers, max-pools them, keeps a top-k budget per KV head plus the attention sinks
 * and the recent window, and gathers the kept K/V rows (or, for Token-Selective
 * Propagation, the kept hidden-state rows) into a compact cache.
 *
 * Sources of the operation (web summaries of the papers):
 *   - FastKV, sec. 1 "Problemstellung": SnapKV / StreamingLLM compress the KV cache after
 *     prefill (decoding-only eviction);
 *   - FastKV, sec. 2A "Token-Selective Propagation": a saliency score selects the tokens
 *     that are propagated, plus a window of the most recent tokens;
 *   - FastKV, sec. 2B "Entkoppelte KV-Cache-Reduktion": the TSP rate and the KV retention
 *     rate are separate knobs;
 *   - StructKV, sec. 1 "Global In-Degree Centrality": the cumulative score of a token is
 *     the sum of its attention scores over all layers up to the pivot;
 *   - CentroidKV, "Inferentie Pipeline" (Preservation): attention sinks and recent tokens
 *     are always kept;
 *   - CentroidKV, "Probleemstelling" (Eviction): tokens are evicted by attention score.
 * The pages do not write the score formula down; the definition used here is the
 * standard window-softmax one:
 *     x[g,i,j] = q[g,i] . k[j] / sqrt(D)                (query i of head g, key j)
 *     window query i sits at position N - window + i and sees keys j <= N - window + i
 *     p[g,i,j] = exp(x[g,i,j] - m[g,i]) / l[g,i]        (softmax over the visible keys)
 *     s[h,j]   = sum over heads g with g / G == h, and over i, of p[g,i,j]
 * with G = Hq / Hkv (contiguous head groups).  Candidates are C = [n_sink, N - window);
 * the pooled score of j in C is the max of s over {t in C : |t - j| <= (pool_kernel-1)/2};
 * k_sel = budget - n_sink - window candidates with the largest pooled score are kept,
 * equal scores going to the lower index; the kept list is sinks + selected + window in
 * ascending position order.
 *
 * Conventions for every entry point:
 *   Ownership  The caller owns every buffer.  The library allocates no device memory;
 *              scratch comes from the caller's workspace `ws` (size from
 *              kvc_workspace_size).  Pointers named "device" must be device (or managed)
 *              memory of the current device.
 *   Layout     All tensors are dense, row-major (C order), with the shapes given below.
 *   Asynchrony All work is enqueued on `stream` (a cudaStream_t; 0 = legacy default
 *              stream).  No call synchronises the host except kvc_poll_error.  Outputs are
 *              valid in stream order.
 *   Errors     Arguments are validated on the host before anything is enqueued; a call
 *              that returns anything but KVC_OK has enqueued nothing, except KVC_ERR_CUDA
 *              (a CUDA launch failed part way).  Device-side problems (a bounded wait that
 *              gave up, an index out of range in kvc_gather) never fault or hang the GPU:
 *              the kernel skips the work, records a flag, and kvc_poll_error reports it.
 *   Checks     The same sources also build as libkvc_checks.so (compile flag KVC_CHECKS=1):
 *              every kernel then tests the indices and coordinates it forms (score and
 *              index writes, gather rows, TMA tile coordinates, CSM owners and output
 *              slots, decode partial slots) against the extents of the buffers they
 *              address, plus the counts the selection must reach; a failed test skips the
 *              access and kvc_poll_error returns KVC_ERR_CHECK.  kvc_checks_enabled tells
 *              the two builds apart.  The regular build compiles the tests away.
 *   Threading  Calls are thread-safe; concurrent calls need distinct workspaces.
 *   Alignment  q, k, v, hidden and all outputs must be 16-byte aligned; ws 256-byte.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVC_API __attribute__((visibility("default")))
#else
#define KVC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvc_stream_t; /* identical to cudaStream_t */

typedef enum kvc_status {
    KVC_OK = 0,
    KVC_ERR_ARG = 1,         /* null pointer, non-positive or inconsistent shape          */
    KVC_ERR_UNSUPPORTED = 2, /* D != 128, unknown dtype/scope, G*window > 256             */
    KVC_ERR_BUDGET = 3,      /* budget < n_sink + window + 1, budget > N, empty TSP        */
    KVC_ERR_ALIGN = 4,       /* pointer or row size not 16-byte aligned (ws: 256-byte)     */
    KVC_ERR_WORKSPACE = 5,   /* ws_bytes smaller than kvc_workspace_size                  */
    KVC_ERR_CUDA = 6,        /* a CUDA runtime call failed                                */
    KVC_ERR_TIMEOUT = 7,     /* a device-side bounded wait gave up (reported by poll)      */
    KVC_ERR_INDEX = 8,       /* kvc_gather met an index outside [0, N) (reported by poll)  */
    KVC_ERR_CHECK = 9        /* a device-side range check failed: checks build only (poll)  */
} kvc_status;

enum { KVC_F32 = 0, KVC_BF16 = 1 };

enum {
    KVC_SCOPE_PER_KV_HEAD = 0, /* one score row per (batch, KV head)                    */
    KVC_SCOPE_ALL_HEADS = 1    /* one score row per batch element: summed over KV heads */
};

/* kvc_params.flags */
enum {
    KVC_FLAG_SIMT_SCORE = 1u << 0, /* score with the CUDA-core (FFMA) kernels even for bf16  */
    /* Test hook for failure detection: the tensor-core scoring kernel's cross-CTA wait
     * watches a flag that nothing sets, so it gives up after spin_limit polls; the scores
     * of the units involved come out as zeros and kvc_poll_error returns KVC_ERR_TIMEOUT.
     * Nothing faults or hangs.  Ignored by the CUDA-core path (it has no such wait). */
    KVC_FLAG_INJECT_WAIT_TIMEOUT = 1u << 1
};

/* Entries of kvc_params.stage_events: events recorded on the stream between the stages
 * of kvc_compress (index i is recorded before stage i; the last after the last stage). */
enum {
    KVC_STAGE_SCORE = 0,  /* window softmax + group/layer sums          */
    KVC_STAGE_SELECT = 1, /* head sums for TSP, pooling, top-k          */
    KVC_STAGE_GATHER = 2, /* compact K/V (and hidden-row) copies        */
    KVC_STAGE_COUNT = 3
};

typedef struct kvc_params {
    int32_t B;           /* batch (independent sequences)                                  */
    int32_t Hq;          /* query heads                                                    */
    int32_t Hkv;         /* KV heads; Hq % Hkv == 0, q head g reads KV head g / (Hq/Hkv)    */
    int32_t N;           /* cached tokens per sequence                                     */
    int32_t D;           /* head dimension; must be 128                                    */
    int32_t window;      /* observation-window queries w; 1 <= w < N                       */
    int32_t dtype;       /* KVC_F32 or KVC_BF16: q, K, V and hidden rows                    */
    int32_t n_sink;      /* attention sinks kept at positions [0, n_sink); >= 0             */
    int32_t pool_kernel; /* odd width of the 1-D max-pool; 1 disables pooling               */
    int32_t kv_budget;   /* kept KV rows per row of scores, INCLUDING sinks and window      */
    int32_t scope;       /* KVC_SCOPE_PER_KV_HEAD or KVC_SCOPE_ALL_HEADS                    */
    int32_t n_layers;    /* >= 1: q and k hold this many layers; scores are summed over them */
    float tsp_rate;      /* > 0: Token-Selective Propagation of floor(rate*N) tokens       */
    int32_t hidden_dim;  /* elements per hidden-state row (TSP only)                       */
    int64_t spin_limit;  /* iterations a device-side wait may spin; 0 = library default    */
    uint32_t flags;      /* KVC_FLAG_*                                                      */
    uint32_t reserved;   /* must be 0                                                      */
    void *const *stage_events; /* optional: KVC_STAGE_COUNT+1 cudaEvent_t (kvc_compress)  */
} kvc_params;

/*
 * kvc_workspace_size -- bytes of device workspace that kvc_score / kvc_compress need for
 * these parameters.  Host only; enqueues nothing.
 * Source: none on the pages (they describe no interface); the call exists because the
 * library allocates no device memory of its own.
 */
KVC_API kvc_status kvc_workspace_size(const kvc_params *p, size_t *bytes);

/*
 * kvc_score -- saliency scores (the definition above), summed over window queries, the
 * GQA group and the n_layers layers; for KVC_SCOPE_ALL_HEADS also over all KV heads.
 *   q       device, [n_layers, B, Hq, window, D]   dtype   (post-RoPE window queries)
 *   k       device, [n_layers, B, Hkv, N, D]       dtype   (post-RoPE keys)
 *   scores  device, [B, Hs, N] fp32, written; Hs = Hkv (PER_KV_HEAD) or 1 (ALL_HEADS).
 *           Every position gets its score, window keys included.
 *   ws      device workspace of >= kvc_workspace_size(p) bytes.
 * Sources: FastKV sec. 2A (saliency), StructKV sec. 1 (sum over layers).
 */
KVC_API kvc_status kvc_score(const kvc_params *p, const void *q, const void *k, float *scores,
                     void *ws, size_t ws_bytes, kvc_stream_t stream);

/*
 * kvc_accumulate -- acc[b, o, j] += sum_{r < Hi/Ho} src[b, o*(Hi/Ho) + r, j].
 *   acc  device [B, Ho, N] fp32, read and written;  src  device [B, Hi, N] fp32.
 *   Hi % Ho == 0.  The sum runs in a fixed order (deterministic).
 * Source: StructKV sec. 1 (cumulative sums over heads/layers); FastKV sec. 2A (TSP uses
 * one head-summed score per token).
 */
KVC_API kvc_status kvc_accumulate(float *acc, const float *src, int32_t B, int32_t Hi, int32_t Ho,
                          int32_t N, kvc_stream_t stream);

/*
 * kvc_pool -- 1-D max-pool over [lo, hi) with odd width `kernel`, edges clipped:
 *   out[r, j] = max{ in[r, t] : lo <= t < hi, |t - j| <= (kernel-1)/2 }  for lo <= j < hi,
 *   out[r, j] = in[r, j]                                                  otherwise.
 *   in, out  device [B, H, N] fp32 (distinct buffers).  0 <= lo <= hi <= N.
 * Source: no page describes pooling; the step (max-pool of the summed scores before the
 * top-k, clipped at the candidate range) is the target statement's, and it fixes no
 * more than that.
 */
KVC_API kvc_status kvc_pool(const float *in, float *out, int32_t B, int32_t H, int32_t N, int32_t lo,
                    int32_t hi, int32_t kernel, kvc_stream_t stream);

/*
 * kvc_topk_workspace_size -- device workspace of kvc_topk for B*H rows of length N
 * (currently always 0 bytes: the selection keeps its state in shared memory).
 * Source: none on the pages; the call keeps the workspace convention uniform.
 */
KVC_API kvc_status kvc_topk_workspace_size(int32_t B, int32_t H, int32_t N, size_t *bytes);

/*
 * kvc_topk -- per row of `pooled`: keep the k_sel = budget - n_sink - window largest values
 * among positions [n_sink, N - window) (equal values: lower position first), add the
 * positions [0, n_sink) and [N - window, N), and write the `budget` kept positions in
 * ascending order.  Values must not be NaN; -0.0 ranks equal to +0.0.
 *   pooled  device [B, H, N] fp32;   idx  device [B, H, budget] int32, written.
 *   Requires n_sink >= 0, window >= 0, n_sink + window + 1 <= budget <= N (else
 *   KVC_ERR_BUDGET).
 * Source: CentroidKV "Probleemstelling" (eviction by attention score) and "Inferentie
 * Pipeline" (sinks and recent tokens preserved); FastKV sec. 2A (recent window).
 */
KVC_API kvc_status kvc_topk(const float *pooled, int32_t B, int32_t H, int32_t N, int32_t n_sink,
                    int32_t window, int32_t budget, int32_t *idx, void *ws, size_t ws_bytes,
                    kvc_stream_t stream);

/*
 * kvc_gather -- dst[b, h, r, :] = src[b, h, idx[b, h', r], :] as raw bytes, with h' = h
 * when Hidx == Hsrc and h' = 0 when Hidx == 1 (one index list shared by all heads).
 *   src  device [B, Hsrc, N, row_bytes];  idx  device [B, Hidx, K] int32;
 *   dst  device [B, Hsrc, K, row_bytes], written.  row_bytes % 16 == 0.
 * An index outside [0, N) leaves its destination row zero-filled and makes the next
 * kvc_poll_error return KVC_ERR_INDEX.
 * Source: FastKV sec. 2B (KV entries kept per layer), sec. 2A (propagated rows).
 */
KVC_API kvc_status kvc_gather(const void *src, int32_t B, int32_t Hsrc, int32_t N, size_t row_bytes,
                      const int32_t *idx, int32_t Hidx, int32_t K, void *dst,
                      kvc_stream_t stream);

/*
 * kvc_compress -- the whole path: score -> (head/layer sums) -> pool -> top-k -> gather.
 *   q, k      as in kvc_score (all n_layers layers are scored).
 *   v         device [B, Hkv, N, D] dtype: the values of the LAST layer in k.
 *   k_out     device [B, Hkv, kv_budget, D], v_out likewise: rows of the last layer's K
 *             and of v at the kept positions.
 *   idx_out   device [B, Hs, kv_budget] int32 kept positions (Hs as in kvc_score; with
 *             KVC_SCOPE_ALL_HEADS one list is shared by all KV heads).
 *   TSP (tsp_rate > 0; otherwise hidden, hidden_out and tsp_idx_out must be NULL):
 *   hidden    device [B, N, hidden_dim] dtype;
 *   tsp_idx_out device [B, 1, kvc_tsp_count(N, window, n_sink, tsp_rate)] int32: kept
 *             positions of the head-summed (all KV heads) pooled scores;
 *   hidden_out device [B, kvc_tsp_count(...), hidden_dim]: the propagated rows.
 *   ws        device workspace of >= kvc_workspace_size(p) bytes.
 * Sources: all of the above.
 */
KVC_API kvc_status kvc_compress(const kvc_params *p, const void *q, const void *k, const void *v,
                        void *k_out, void *v_out, int32_t *idx_out, const void *hidden,
                        void *hidden_out, int32_t *tsp_idx_out, void *ws, size_t ws_bytes,
                        kvc_stream_t stream);

/*
 * kvc_score_entropy -- kvc_score plus the attention entropy of every window query row,
 * taken in the same pass.  StructKV watches attention entropy (with sparsity and variance,
 * see kvc_row_stats) during the first pass to find the layer where attention settles
 * (StructKV page, sec. 2 "Dynamische Pivot Detectie"); the page gives no formula, so the
 * entropy here is Shannon's, in nats, of each window query's causal softmax row:
 * H = -sum_j p_j ln p_j over the keys j <= N - window + i that query i sees.
 *   q, k, scores, ws  as in kvc_score (same results in `scores`).
 *   entropy  device, [n_layers, B, Hq, window] fp32 (4-byte aligned), written; row order as
 *            in q.
 * Cost: one extra multiply-add per logit and one more fp64 total per query row.
 */
KVC_API kvc_status kvc_score_entropy(const kvc_params *p, const void *q, const void *k, float *scores,
                                     float *entropy, void *workspace, size_t workspace_bytes,
                                     kvc_stream_t stream);

/*
 * kvc_row_stats -- the other two pivot-detection signals (StructKV page, sec. 2), per score
 * row: the share of the row's mass held by its kept positions (sparsity) and the population
 * variance of the row over the candidates C = [n_sink, N - window).
 *   scores     device, [rows, N] fp32 (e.g. kvc_score's [B, Hs, N] with rows = B * Hs).
 *   idx        device, [rows, budget] int32 kept positions (kvc_topk's output), or NULL to
 *              skip the kept mass.  An index outside [0, N) is left out of the sum and sets
 *              KVC_ERR_INDEX for kvc_poll_error.
 *   kept_mass  device, [rows] fp32: sum of s over idx / sum of s over [0, N) (unused when
 *              idx is NULL).
 *   cand_var   device, [rows] fp32: (1/n) sum over C of (s - mean_C)^2, n = |C|.
 * Requires n_sink + window < N and, with idx, 1 <= budget <= N.  fp64 sums in a fixed
 * order, so results are deterministic.
 */
KVC_API kvc_status kvc_row_stats(const float *scores, int32_t rows, int32_t N, int32_t n_sink, int32_t window,
                                 const int32_t *idx, int32_t budget, float *kept_mass, float *cand_var,
                                 kvc_stream_t stream);

/*
 * Chunked Soft Matching -- CentroidKV clusters KV states instead of evicting them (CentroidKV
 * page, sec. 3 "Chunked Soft Matching", sec. 4 "Aggregatie").  One round over rows (batch,
 * KV head) of N cached tokens with degrees n_t:
 *   - the candidates C = [n_sink, N - window) are cut into chunks of `chunk` tokens; sinks and
 *     the recent window stay as they are (sec. 2, Preservation);
 *   - in a chunk, the tokens at even offsets form set A and the odd ones set B; each A token
 *     is matched with the B token of its chunk whose key is the most cosine-similar (ties:
 *     lower position; a zero key has similarity 0); an A token alone in its chunk has no
 *     match;
 *   - the m = kvc_csm_merges(...) matches with the largest similarity merge (ties: lower
 *     position): a B token and the A tokens merged into it become their degree-weighted mean
 *     (keys and values alike, fp32 arithmetic rounded once to the element type) and their
 *     degrees add; every other kept row is copied bit for bit;
 *   - the output keeps every token except the merged A tokens, in position order.
 * The ratio r is at most 0.5 (at most half of the cache per round); CentroidKV lowers it
 * over rounds, see kvc_csm_ratio.
 */

/* kvc_csm_merges -- m = min(floor(ratio * |C|), matchable A tokens); -1 for invalid
 * arguments (chunk even in [2, 128], 0 <= ratio <= 0.5, n_sink + window <= N).  Host only. */
KVC_API int32_t kvc_csm_merges(int32_t N, int32_t n_sink, int32_t window, int32_t chunk, float ratio);

/* kvc_csm_ratio -- the progressive schedule of the merge ratio (CentroidKV page, sec. 3):
 * r_round = r_init - round * delta, not below 0.  Host only. */
KVC_API float kvc_csm_ratio(float r_init, float delta, int32_t round);

/* kvc_csm_workspace_size -- bytes of device workspace kvc_csm needs for B * H rows. */
KVC_API kvc_status kvc_csm_workspace_size(int32_t B, int32_t H, int32_t N, int32_t n_sink, int32_t window,
                                          int32_t chunk, float ratio, size_t *bytes);

/*
 * kvc_csm -- one Chunked Soft Matching round.
 *   k, v      device, rows (b, h) of N tokens at a stride of ld_in tokens: row (b, h) starts
 *             at (b * H + h) * ld_in * D elements; dtype KVC_F32 or KVC_BF16, D = 128,
 *             16-byte aligned.  ld_in = 0 means N (dense [B, H, N, D]).
 *   deg       device, same row layout, int32 degrees (>= 1), or NULL for all ones (a
 *             first round).
 *   pos       device, same row layout, int32 positions carried into pos_out, or NULL for
 *             the row index 0..N-1.
 *   k_out, v_out  device, rows of N - m tokens at a stride of ld_out tokens (0 means
 *             N - m), written; must not be k or v (a round is never in place).
 *   deg_out   device, [B, H] x ld_out int32 degrees of the kept tokens, written.
 *   pos_out   device, [B, H] x ld_out int32 positions of the kept tokens (pos[...] of the
 *             input row, or its index), in ascending input order.
 *   ws        device workspace of >= kvc_csm_workspace_size(...) bytes.
 * Errors: KVC_ERR_ARG (null pointers, in-place outputs, chunk/ratio/n_sink/window out of
 * range, ld_in < N, ld_out < N - m), KVC_ERR_UNSUPPORTED (dtype, D), KVC_ERR_ALIGN,
 * KVC_ERR_WORKSPACE.  A malformed selection inside the kernels (never for valid inputs)
 * sets KVC_ERR_INDEX in kvc_poll_error.
 */
KVC_API kvc_status kvc_csm(const void *k, const void *v, const int32_t *deg, const int32_t *pos, int32_t B,
                           int32_t H, int32_t N, int32_t ld_in, int32_t D, int32_t dtype, int32_t n_sink,
                           int32_t window, int32_t chunk, float ratio, void *k_out, void *v_out, int32_t *deg_out,
                           int32_t *pos_out, int32_t ld_out, void *workspace, size_t workspace_bytes,
                           kvc_stream_t stream);

/*
 * kvc_append -- appends t_new decode tokens to every (b, h) row of a cache (CentroidKV page,
 * sec. 2 Inferentie Pipeline, Decoding: the cache grows by one token per step between
 * clustering rounds).
 *   k_cache, v_cache  device, rows of capacity ld tokens holding n tokens; rows n .. n +
 *             t_new - 1 are written from k_new, v_new [B, H, t_new, D] (device).
 *   deg_cache, pos_cache  device int32 caches of the same row layout, or NULL; the new
 *             slots get degree 1 and positions pos0 .. pos0 + t_new - 1.
 * Errors: KVC_ERR_ARG (null pointers, n + t_new > ld), KVC_ERR_UNSUPPORTED (dtype, D),
 * KVC_ERR_ALIGN (16-byte).
 */
KVC_API kvc_status kvc_append(void *k_cache, void *v_cache, int32_t *deg_cache, int32_t *pos_cache, int32_t B,
                              int32_t H, int32_t ld, int32_t n, const void *k_new, const void *v_new,
                              int32_t t_new, int32_t pos0, int32_t D, int32_t dtype, kvc_stream_t stream);

/* kvc_decode_attention_workspace_size -- bytes of device workspace kvc_decode_attention
 * needs for these shapes (G * nq = Hq / Hkv * nq <= 8). */
KVC_API kvc_status kvc_decode_attention_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t nq, int32_t n,
                                                       size_t *bytes);

/*
 * kvc_decode_attention -- attention of decode queries over a clustered cache (CentroidKV
 * page, sec. 4 Aggregatie: the cluster degree enters the softmax as a log term, so that
 * a centroid of degree n weighs like n copies of itself):
 *     out[b, g, i, :] = sum_t softmax_t(q[b, g, i] . k[b, h, t] / sqrt(D) + ln deg[b, h, t]) v[b, h, t, :]
 * over the n cached rows t of KV head h = g / (Hq / Hkv); no mask.
 *   q         device, [B, Hq, nq, D] dtype (the cache's dtype), 16-byte aligned.
 *   k, v      device, rows (b, h) of capacity ld tokens (0 means n) holding n tokens.
 *   deg       device int32 degrees (>= 1) in the same row layout, or NULL (plain attention).
 *   out       device, [B, Hq, nq, D] fp32, written.
 *   ws        device workspace of >= kvc_decode_attention_workspace_size(...) bytes.
 * Errors: KVC_ERR_ARG (null pointers, Hq % Hkv, n < 1, ld < n), KVC_ERR_UNSUPPORTED
 * (Hq / Hkv * nq > 8, dtype, D), KVC_ERR_ALIGN, KVC_ERR_WORKSPACE.  A degree below 1 is
 * read as 1 and sets KVC_ERR_INDEX in kvc_poll_error.
 */
KVC_API kvc_status kvc_decode_attention(const void *q, const void *k, const void *v, const int32_t *deg, int32_t B,
                                        int32_t Hq, int32_t Hkv, int32_t nq, int32_t n, int32_t ld, int32_t D,
                                        int32_t dtype, float *out, void *workspace, size_t workspace_bytes,
                                        kvc_stream_t stream);

/*
 * Sequence sharding (one GPU per contiguous block of the sequence, for contexts beyond one
 * GPU's memory).  The exchange steps between the calls below are the caller's (collectives
 * of a few KiB): an all-gather of every shard's (m, l), a halo of (pool_kernel - 1) / 2
 * scores at each block edge for the pool, a sum of the radix-select histograms per digit,
 * and a count of the ties each shard holds.  Supported for the per-KV-head budget:
 * p->n_layers = 1 and p->scope = KVC_SCOPE_PER_KV_HEAD; p->N is the whole sequence's length.
 * Scoring runs on the CUDA cores.
 */

/* kvc_shard_workspace_size -- device workspace of kvc_shard_stats / kvc_shard_scores for a
 * block of n_local keys. */
KVC_API kvc_status kvc_shard_workspace_size(const kvc_params *p, int32_t n_local, size_t *bytes);

/*
 * kvc_shard_stats -- this block's part of each window row's softmax normaliser.
 *   q        device, [B, Hq, window, D] (all window queries; every shard holds them).
 *   k_local  device, [B, Hkv, n_local, D]: keys key_offset .. key_offset + n_local - 1.
 *   ml       device, [B * Hkv][G * window][2] fp32, written: a pair (m, l) with l * 2^m =
 *            the sum of 2^y over the block's keys that the row sees (y = q.k log2(e) /
 *            sqrt(D); window row i sits at position N - window + i); (-inf, 0) when it
 *            sees none.  The tensor-core path (bf16, G * window <= 128) writes 1 <= l < 2,
 *            the CUDA-core path m = the largest such y; both merge the same way.
 * Runs on the tensor cores when q and K are bf16 and G * window <= 128 (phase 1 of the
 * score kernel alone), otherwise (or with KVC_FLAG_SIMT_SCORE) on the CUDA cores.
 */
KVC_API kvc_status kvc_shard_stats(const kvc_params *p, const void *q, const void *k_local, int32_t n_local,
                                   int32_t key_offset, float *ml, void *workspace, size_t workspace_bytes,
                                   kvc_stream_t stream);

/*
 * kvc_shard_scores -- the block's saliency scores given every shard's (m, l).
 *   ml_all   device, [n_shards][B * Hkv][G * window][2]: the shards' kvc_shard_stats
 *            outputs in shard order; merged in that order into each row's log-sum-exp, so
 *            every shard uses the same value.
 *   scores   device, [B, Hkv, n_local] fp32, written.
 */
KVC_API kvc_status kvc_shard_scores(const kvc_params *p, const void *q, const void *k_local, int32_t n_local,
                                    int32_t key_offset, const float *ml_all, int32_t n_shards, float *scores,
                                    void *workspace, size_t workspace_bytes, kvc_stream_t stream);

/*
 * kvc_select_hist -- one digit of a radix select spread over shards: for each row of pooled
 * [rows, n] (fp32, device), hist[row][d] (device, [rows][1 << digit_bits] uint32, written)
 * counts the candidates j in [lo, hi) whose order key (a monotone map of the fp32 value to
 * uint32, -0.0 read as +0.0; larger value, larger key) has its top prefix_bits equal to
 * prefix[row]'s (device uint32 [rows]) and the next digit_bits equal to d.
 * 1 <= digit_bits <= 12, prefix_bits + digit_bits <= 32.
 */
KVC_API kvc_status kvc_select_hist(const float *pooled, int32_t rows, int32_t n, int32_t lo, int32_t hi,
                                   const uint32_t *prefix, int32_t prefix_bits, int32_t digit_bits, uint32_t *hist,
                                   kvc_stream_t stream);

/*
 * kvc_select_emit -- the shard's part of the selection once the threshold key is known:
 * for each row writes, in position order, pos_offset + j for the candidates j in [lo, hi)
 * whose key is above thr[row] and for the first ties[row] candidates whose key equals it
 * (ties go to the lower positions) into out[row][0 .. cap) (device int32), and the number
 * written into count[row].  More than cap sets KVC_ERR_INDEX in kvc_poll_error.  pos_offset
 * may be negative (a block's row can start with a halo) as long as pos_offset + lo >= 0.
 */
KVC_API kvc_status kvc_select_emit(const float *pooled, int32_t rows, int32_t n, int32_t lo, int32_t hi,
                                   const uint32_t *thr, const int32_t *ties, int32_t pos_offset, int32_t *out,
                                   int32_t cap, int32_t *count, kvc_stream_t stream);

/*
 * kvc_select_pick -- one digit of the distributed radix select, after the shards'
 * histograms of the digit have been summed: for each row, the bucket b (scanned from the
 * top) that holds the need[row]-th largest key; need[row] becomes the number of keys still
 * needed inside b, prefix[row] gets b in its next digit_bits bits below the top
 * prefix_bits, and eq_local[row] = hist_local[row][b] (this shard's keys in b).
 *   hist, hist_local  device uint32 [rows][1 << digit_bits]: summed over shards / this shard's
 *   need (int32), prefix (uint32), eq_local (int32): device [rows]; need and prefix read and
 *   written.  1 <= digit_bits <= 12, prefix_bits + digit_bits <= 32.
 * Source: none on the pages; the sequence-sharded variant's selection step (one radix digit
 * per exchange), the same ordering as kvc_topk (ties go to the lower positions).
 */
KVC_API kvc_status kvc_select_pick(const uint32_t *hist, const uint32_t *hist_local, int32_t rows,
                                   int32_t digit_bits, int32_t prefix_bits, int32_t *need, uint32_t *prefix,
                                   int32_t *eq_local, kvc_stream_t stream);

/*
 * kvc_select_ties -- this shard's share of the keys equal to the threshold: take[row] =
 * clamp(need[row] - sum over shards s < rank of eq_all[s][row], 0, eq_all[rank][row])
 * (the lower shards, i.e. the lower positions, take theirs first).
 *   eq_all  device int32 [n_shards][rows] (every shard's eq_local after the last digit);
 *   need, take  device int32 [rows].
 * Source: none on the pages; the tie rule of kvc_topk spread over shards.
 */
KVC_API kvc_status kvc_select_ties(const int32_t *eq_all, int32_t n_shards, int32_t rank, int32_t rows,
                                   const int32_t *need, int32_t *take, kvc_stream_t stream);

/*
 * kvc_select_kept -- the rows a shard keeps, in position order: the sinks [0, n_sink) that
 * lie in the shard, the shard's selected positions (kvc_select_emit's sel [rows][cap_sel]
 * and count_sel [rows]), the window keys [N - window, N) that lie in it.  Writes pos
 * [rows][cap] (global positions, -1 past the count), local_idx [rows][cap] (pos -
 * key_offset, 0 past the count; ready for kvc_gather) and count [rows] (all device int32).
 * More than cap rows sets KVC_ERR_INDEX in kvc_poll_error (cap = min(n_local, budget) is
 * always enough).
 * Source: CentroidKV "Inferentie Pipeline" and FastKV sec. 2A (sinks and recent tokens kept
 * beside the selection), spread over shards.
 */
KVC_API kvc_status kvc_select_kept(const int32_t *sel, const int32_t *count_sel, int32_t rows, int32_t cap_sel,
                                   int32_t N, int32_t n_sink, int32_t window, int32_t key_offset, int32_t n_local,
                                   int32_t cap, int32_t *pos, int32_t *local_idx, int32_t *count,
                                   kvc_stream_t stream);

/*
 * kvc_score_noalloc -- kvc_score for callers that cannot allocate device memory.  The
 * pages have no counterpart: it exists for engines that have already given all device
 * memory to their own pool, or plugin interfaces that forbid cudaMalloc/cudaFree during a
 * step, and so cannot pass a workspace.  Same arguments and results as kvc_score without
 * ws/ws_bytes; it always scores with the CUDA-core kernels and keeps their scratch in a
 * 4 MiB array compiled into the library, which every GPU that loads the library holds
 * until the process exits.
 *   Returns KVC_ERR_WORKSPACE when the scratch these parameters need exceeds 4 MiB; that
 *   check comes before the pointer checks.  With U = n_layers * B * Hkv, nq = (Hq / Hkv) *
 *   window, chunk = min(2048, max(32, 32 * ceil(ceil(N * U / 296) / 32))) and n_chunks =
 *   ceil(N / chunk), the scratch is r(U * n_chunks * nq * 8) + r(U * nq * 4) bytes, plus
 *   U * N * 4 bytes when several layers or all heads are summed (r() rounds up to a
 *   multiple of 256).
 *   The first call on each device looks up the array's address (with that device
 *   current); make it before any stream capture begins.  The address is kept for the life
 *   of the device's context: do not keep using the library across cudaDeviceReset or a
 *   reset of the primary context.  All calls on a device share the
 *   array: calls whose kernels may overlap on the GPU race and must be ordered by the
 *   caller.  It allocates nothing and clears nothing between calls (every scratch byte it
 *   reads is written earlier in the same call).
 */
KVC_API kvc_status kvc_score_noalloc(const kvc_params *p, const void *q, const void *k, float *scores,
                                     kvc_stream_t stream);

/*
 * kvc_tsp_count -- rows propagated by TSP: min(floor(tsp_rate * N), N - window - n_sink)
 * selected tokens plus n_sink + window; 0 when tsp_rate <= 0 or floor(tsp_rate*N) < 1.
 * Source: FastKV sec. 2B (the TSP rate sets how many tokens continue past the TSP layer).
 */
KVC_API int32_t kvc_tsp_count(int32_t N, int32_t window, int32_t n_sink, float tsp_rate);

/*
 * kvc_poll_error -- synchronises `stream`, then returns (and clears) the device-side
 * problems recorded since the last poll on this device, reporting the first of
 * KVC_ERR_TIMEOUT, KVC_ERR_INDEX, KVC_ERR_CHECK (checks build only) that is set, else KVC_OK.
 * KVC_ERR_CUDA if the synchronisation itself failed.
 */
KVC_API kvc_status kvc_poll_error(kvc_stream_t stream);

/*
 * kvc_checks_enabled -- 1 for the range-checking build (libkvc_checks.so, compiled with
 * KVC_CHECKS=1), 0 for the regular one.  Host only.
 */
KVC_API int32_t kvc_checks_enabled(void);

/*
 * kvc_launch_count -- number of CUDA kernels this library has launched in this process
 * (all devices, all threads), for diagnostics and benchmarks.  Host only.
 */
KVC_API uint64_t kvc_launch_count(void);

/* kvc_status_string -- static description of a status code (never NULL). */
KVC_API const char *kvc_status_string(kvc_status status);

/* kvc_version -- library version string, e.g. "kvc 0.1.0 sm_100a". */
KVC_API const char *kvc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */

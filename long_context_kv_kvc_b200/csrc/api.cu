// api.cu -- the C ABI of libkvc.so: argument validation, workspace layout and the
// launch sequence of each entry point.  See include/kvc.h for the contracts.
#include <algorithm>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "kvc_internal.cuh"

namespace kvc {

static __device__ unsigned int g_error_word;
static std::atomic<unsigned long long> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

unsigned int* device_error_word() {
    // one address per device; cudaGetSymbolAddress is cheap but not free
    static std::atomic<unsigned int*> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
    if (dev < 64) {
        unsigned int* c = cache[dev].load();
        if (c) return c;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    if (dev < 64) cache[dev].store((unsigned int*)p);
    return (unsigned int*)p;
}

}  // namespace kvc

using namespace kvc;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t esize(int dtype) { return dtype == KVC_F32 ? 4 : 2; }

// Workspace layout of one call.
struct Plan {
    int U = 0, nq = 0, Hs = 0, n_tsp = 0;
    bool units = false;  // unit scores need a reduction (several layers or all heads)
    bool use_tc = false;
    int n_chunks = 0, chunk = 0;
    size_t off_partial = 0, off_partial_t = 0, off_lse = 0, off_units = 0, off_scores = 0, off_pooled = 0;
    size_t off_tsp_scores = 0, off_tsp_pooled = 0, off_tc = 0, tc_bytes = 0, total = 0;
};

kvc_status check_params(const kvc_params* p) {
    if (!p) return KVC_ERR_ARG;
    if (p->reserved != 0) return KVC_ERR_ARG;
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->N < 1 || p->window < 1 || p->n_layers < 1)
        return KVC_ERR_ARG;
    if (p->Hq % p->Hkv) return KVC_ERR_ARG;
    if (p->D != kHeadDim) return KVC_ERR_UNSUPPORTED;
    if (p->dtype != KVC_F32 && p->dtype != KVC_BF16) return KVC_ERR_UNSUPPORTED;
    if (p->scope != KVC_SCOPE_PER_KV_HEAD && p->scope != KVC_SCOPE_ALL_HEADS) return KVC_ERR_UNSUPPORTED;
    if ((long long)(p->Hq / p->Hkv) * p->window > 256) return KVC_ERR_UNSUPPORTED;
    if (p->n_sink < 0 || p->window >= p->N) return KVC_ERR_ARG;
    if (p->pool_kernel < 1 || p->pool_kernel % 2 == 0) return KVC_ERR_ARG;
    if (!(p->tsp_rate >= 0.f) || p->spin_limit < 0) return KVC_ERR_ARG;
    // every unit's K block must be addressable with 64-bit offsets and N fits int32
    if ((long long)p->n_layers * p->B * p->Hkv > (1LL << 30)) return KVC_ERR_ARG;
    return KVC_OK;
}

kvc_status check_budget(int N, int S, int w, int budget) {
    if ((long long)S + w + 1 > budget || budget > N) return KVC_ERR_BUDGET;
    return KVC_OK;
}

ScoreJob make_job(const kvc_params* p, const void* q, const void* k) {
    ScoreJob j{};
    j.q = q;
    j.k = k;
    j.dtype = p->dtype;
    j.U = p->n_layers * p->B * p->Hkv;
    j.N = p->N;
    j.window = p->window;
    j.G = p->Hq / p->Hkv;
    j.nq = j.G * p->window;
    j.spin_limit = p->spin_limit > 0 ? p->spin_limit : (1LL << 22);
    j.inject_timeout = (p->flags & KVC_FLAG_INJECT_WAIT_TIMEOUT) ? 1 : 0;
    return j;
}

// Fills `pl` for kvc_score (compress = false) or kvc_compress (compress = true).
void make_plan(const kvc_params* p, bool compress, Plan* pl) {
    Plan P;
    const ScoreJob job = make_job(p, nullptr, nullptr);
    P.U = job.U;
    P.nq = job.nq;
    P.Hs = p->scope == KVC_SCOPE_PER_KV_HEAD ? p->Hkv : 1;
    P.units = p->n_layers > 1 || p->scope == KVC_SCOPE_ALL_HEADS;
    P.use_tc = !(p->flags & KVC_FLAG_SIMT_SCORE) && tc_score_supported(job);
    P.n_tsp = kvc_tsp_count(p->N, p->window, p->n_sink, p->tsp_rate);
    size_t off = 0;
    if (P.use_tc) {
        P.tc_bytes = tc_score_workspace(P.U, p->N, P.nq);
        P.off_tc = off;
        off = align_up(off + P.tc_bytes);
    } else {
        const size_t pb = simt_score_workspace(P.U, p->N, P.nq, &P.n_chunks, &P.chunk);
        P.off_partial = off;
        off = align_up(off + pb);
        P.off_partial_t = off;  // the entropy's third statistic, half the size of (m, l)
        off = align_up(off + pb / 2);
    }
    P.off_lse = off;
    off = align_up(off + (size_t)P.U * P.nq * sizeof(float));
    const size_t row = (size_t)p->N * sizeof(float);
    if (P.units) {
        P.off_units = off;
        off = align_up(off + (size_t)P.U * row);
    }
    if (compress) {
        P.off_scores = off;
        off = align_up(off + (size_t)p->B * P.Hs * row);
        P.off_pooled = off;
        off = align_up(off + (size_t)p->B * P.Hs * row);
        if (p->tsp_rate > 0.f) {
            P.off_tsp_scores = off;
            off = align_up(off + (size_t)p->B * row);
            P.off_tsp_pooled = off;
            off = align_up(off + (size_t)p->B * row);
        }
    }
    P.total = off;
    *pl = P;
}

// Runs the scoring stage: unit scores (and their reduction) into `scores` [B, Hs, N].
kvc_status run_score(const kvc_params* p, const Plan& P, const void* q, const void* k, float* scores,
                     char* ws, cudaStream_t s, float* entropy = nullptr) {
    ScoreJob job = make_job(p, q, k);
    job.entropy = entropy;
    job.unit_scores = P.units ? (float*)(ws + P.off_units) : scores;
    job.lse = (float*)(ws + P.off_lse);
    job.err = device_error_word();
    if (!job.err) return KVC_ERR_CUDA;
    cudaError_t e;
    if (P.use_tc) {
        job.tc_ws = ws + P.off_tc;
        job.tc_ws_bytes = P.tc_bytes;
        e = tc_score(job, s);
    } else {
        job.partial = (float2*)(ws + P.off_partial);
        job.partial_t = (float*)(ws + P.off_partial_t);
        job.n_chunks = P.n_chunks;
        job.chunk = P.chunk;
        e = simt_score(job, s);
    }
    if (e != cudaSuccess) return KVC_ERR_CUDA;
    if (P.units) {
        e = reduce_units(job.unit_scores, p->n_layers, p->B, p->Hkv, p->N,
                         p->scope == KVC_SCOPE_ALL_HEADS, scores, s);
        if (e != cudaSuccess) return KVC_ERR_CUDA;
    }
    return KVC_OK;
}

kvc_status record_stage(const kvc_params* p, int i, cudaStream_t s) {
    if (!p->stage_events || !p->stage_events[i]) return KVC_OK;
    return cudaEventRecord((cudaEvent_t)p->stage_events[i], s) == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

#define KVC_TRY(x)                         \
    do {                                   \
        kvc_status st_ = (x);              \
        if (st_ != KVC_OK) return st_;     \
    } while (0)
#define KVC_CUDA(x)                                      \
    do {                                                 \
        if ((x) != cudaSuccess) return KVC_ERR_CUDA;     \
    } while (0)

}  // namespace

extern "C" {

kvc_status kvc_workspace_size(const kvc_params* p, size_t* bytes) {
    if (!bytes) return KVC_ERR_ARG;
    KVC_TRY(check_params(p));
    Plan P;
    make_plan(p, true, &P);
    *bytes = P.total;
    return KVC_OK;
}

kvc_status kvc_score(const kvc_params* p, const void* q, const void* k, float* scores, void* ws,
                     size_t ws_bytes, kvc_stream_t stream) {
    KVC_TRY(check_params(p));
    if (!q || !k || !scores || !ws) return KVC_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(scores) || ((uintptr_t)ws & (kAlign - 1)))
        return KVC_ERR_ALIGN;
    Plan P;
    make_plan(p, false, &P);
    if (ws_bytes < P.total) return KVC_ERR_WORKSPACE;
    return run_score(p, P, q, k, scores, (char*)ws, (cudaStream_t)stream);
}

kvc_status kvc_score_entropy(const kvc_params* p, const void* q, const void* k, float* scores, float* entropy,
                             void* ws, size_t ws_bytes, kvc_stream_t stream) {
    KVC_TRY(check_params(p));
    if (!q || !k || !scores || !entropy || !ws) return KVC_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(scores) || ((uintptr_t)entropy & 3u) ||
        ((uintptr_t)ws & (kAlign - 1)))
        return KVC_ERR_ALIGN;
    Plan P;
    make_plan(p, false, &P);
    if (ws_bytes < P.total) return KVC_ERR_WORKSPACE;
    return run_score(p, P, q, k, scores, (char*)ws, (cudaStream_t)stream, entropy);
}

kvc_status kvc_row_stats(const float* scores, int32_t rows, int32_t N, int32_t n_sink, int32_t window,
                         const int32_t* idx, int32_t budget, float* kept_mass, float* cand_var,
                         kvc_stream_t stream) {
    if (!scores || !cand_var || rows < 1 || N < 1 || n_sink < 0 || window < 0) return KVC_ERR_ARG;
    if ((long long)n_sink + window >= N) return KVC_ERR_ARG;
    if (idx && (!kept_mass || budget < 1 || budget > N)) return KVC_ERR_ARG;
    unsigned* err = device_error_word();
    if (!err) return KVC_ERR_CUDA;
    KVC_CUDA(kvc::row_stats(scores, rows, N, n_sink, window, idx, idx ? budget : 0, kept_mass, cand_var, err,
                            (cudaStream_t)stream));
    return KVC_OK;
}

namespace {
kvc_status check_csm(int32_t N, int32_t D, int32_t n_sink, int32_t window, int32_t chunk, float ratio) {
    if (N < 1 || n_sink < 0 || window < 0 || (long long)n_sink + window > N) return KVC_ERR_ARG;
    if (chunk < 2 || chunk > 128 || chunk % 2 || !(ratio >= 0.f && ratio <= 0.5f)) return KVC_ERR_ARG;
    if (D != kHeadDim) return KVC_ERR_UNSUPPORTED;
    return KVC_OK;
}
}  // namespace

int32_t kvc_csm_merges(int32_t N, int32_t n_sink, int32_t window, int32_t chunk, float ratio) {
    if (check_csm(N, kHeadDim, n_sink, window, chunk, ratio) != KVC_OK) return -1;
    return kvc::csm_merges(N, n_sink, window, chunk, ratio);
}

float kvc_csm_ratio(float r_init, float delta, int32_t round) {
    const float r = r_init - (float)round * delta;
    return r > 0.f ? r : 0.f;
}

kvc_status kvc_csm_workspace_size(int32_t B, int32_t H, int32_t N, int32_t n_sink, int32_t window, int32_t chunk,
                                  float ratio, size_t* bytes) {
    if (!bytes || B < 1 || H < 1) return KVC_ERR_ARG;
    KVC_TRY(check_csm(N, kHeadDim, n_sink, window, chunk, ratio));
    *bytes = kvc::csm_workspace(B * H, N, kvc::csm_merges(N, n_sink, window, chunk, ratio));
    return KVC_OK;
}

kvc_status kvc_csm(const void* k, const void* v, const int32_t* deg, const int32_t* pos, int32_t B, int32_t H,
                   int32_t N, int32_t ld_in, int32_t D, int32_t dtype, int32_t n_sink, int32_t window, int32_t chunk,
                   float ratio, void* k_out, void* v_out, int32_t* deg_out, int32_t* pos_out, int32_t ld_out,
                   void* ws, size_t ws_bytes, kvc_stream_t stream) {
    if (!k || !v || !k_out || !v_out || !deg_out || !pos_out || !ws || B < 1 || H < 1) return KVC_ERR_ARG;
    if (k_out == k || v_out == v || k_out == v || v_out == k) return KVC_ERR_ARG;  // no in-place round
    if (dtype != KVC_F32 && dtype != KVC_BF16) return KVC_ERR_UNSUPPORTED;
    KVC_TRY(check_csm(N, D, n_sink, window, chunk, ratio));
    const int m = kvc::csm_merges(N, n_sink, window, chunk, ratio);
    if (ld_in == 0) ld_in = N;
    if (ld_out == 0) ld_out = N - m;
    if (ld_in < N || ld_out < N - m) return KVC_ERR_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_out) || !aligned16(v_out) || ((uintptr_t)ws & (kAlign - 1)))
        return KVC_ERR_ALIGN;
    if ((long long)B * H * std::max(ld_in, N) > (1LL << 31) - 1) return KVC_ERR_ARG;
    if (ws_bytes < kvc::csm_workspace(B * H, N, m)) return KVC_ERR_WORKSPACE;
    KVC_CUDA(kvc::csm(k, v, dtype, deg, pos, B * H, N, ld_in, n_sink, window, chunk, m, k_out, v_out, deg_out,
                      pos_out, ld_out, ws, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_append(void* k_cache, void* v_cache, int32_t* deg_cache, int32_t* pos_cache, int32_t B, int32_t H,
                      int32_t ld, int32_t n, const void* k_new, const void* v_new, int32_t t_new, int32_t pos0,
                      int32_t D, int32_t dtype, kvc_stream_t stream) {
    if (!k_cache || !v_cache || !k_new || !v_new || B < 1 || H < 1 || n < 0 || t_new < 0) return KVC_ERR_ARG;
    if ((long long)n + t_new > ld || (long long)B * H * ld > (1LL << 31) - 1) return KVC_ERR_ARG;
    if (dtype != KVC_F32 && dtype != KVC_BF16) return KVC_ERR_UNSUPPORTED;
    if (D != kHeadDim) return KVC_ERR_UNSUPPORTED;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new)) return KVC_ERR_ALIGN;
    KVC_CUDA(kvc::append_rows(k_cache, v_cache, deg_cache, pos_cache, dtype, B * H, ld, n, k_new, v_new, t_new, pos0,
                              (cudaStream_t)stream));
    return KVC_OK;
}

namespace {
kvc_status check_decode(int32_t B, int32_t Hq, int32_t Hkv, int32_t nq, int32_t n) {
    if (B < 1 || Hq < 1 || Hkv < 1 || nq < 1 || n < 1 || Hq % Hkv) return KVC_ERR_ARG;
    if (!kvc::decode_rows_supported(Hq / Hkv * nq)) return KVC_ERR_UNSUPPORTED;
    return KVC_OK;
}
}  // namespace

kvc_status kvc_decode_attention_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t nq, int32_t n,
                                               size_t* bytes) {
    if (!bytes) return KVC_ERR_ARG;
    KVC_TRY(check_decode(B, Hq, Hkv, nq, n));
    *bytes = kvc::decode_workspace(B * Hkv, Hq / Hkv * nq, n);
    return KVC_OK;
}

kvc_status kvc_decode_attention(const void* q, const void* k, const void* v, const int32_t* deg, int32_t B,
                                int32_t Hq, int32_t Hkv, int32_t nq, int32_t n, int32_t ld, int32_t D, int32_t dtype,
                                float* out, void* ws, size_t ws_bytes, kvc_stream_t stream) {
    if (!q || !k || !v || !out || !ws) return KVC_ERR_ARG;
    KVC_TRY(check_decode(B, Hq, Hkv, nq, n));
    if (ld == 0) ld = n;
    if (ld < n || (long long)B * Hkv * ld > (1LL << 31) - 1) return KVC_ERR_ARG;
    if (dtype != KVC_F32 && dtype != KVC_BF16) return KVC_ERR_UNSUPPORTED;
    if (D != kHeadDim) return KVC_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || ((uintptr_t)ws & (kAlign - 1)))
        return KVC_ERR_ALIGN;
    const int U = B * Hkv, Rv = Hq / Hkv * nq;
    if (ws_bytes < kvc::decode_workspace(U, Rv, n)) return KVC_ERR_WORKSPACE;
    KVC_CUDA(kvc::decode_attention(q, k, v, deg, dtype, U, Rv, n, ld, out, ws, (cudaStream_t)stream));
    return KVC_OK;
}

namespace {
// sequence sharding supports the per-KV-head budget (one layer, per-KV-head scope); the block
// of keys [key_offset, key_offset + n_local) lies inside the sequence of p->N keys
kvc_status check_shard(const kvc_params* p, int32_t n_local, int32_t key_offset) {
    KVC_TRY(check_params(p));
    if (p->n_layers != 1 || p->scope != KVC_SCOPE_PER_KV_HEAD) return KVC_ERR_UNSUPPORTED;
    if (n_local < 1 || key_offset < 0 || (long long)key_offset + n_local > p->N) return KVC_ERR_ARG;
    return KVC_OK;
}

// The block's scoring runs on the tensor cores (bf16, G * window <= 128, unless the caller
// asks for the CUDA-core path) or on the CUDA cores; the workspace is that path's.
struct ShardPlan {
    bool use_tc;
    int n_chunks, chunk;
    size_t off_partial, off_lse, total;
};

ShardPlan shard_plan(const kvc_params* p, int n_local) {
    ShardPlan P{};
    ScoreJob job = make_job(p, nullptr, nullptr);
    job.N = n_local;
    P.use_tc = !(p->flags & KVC_FLAG_SIMT_SCORE) && tc_score_supported(job);
    if (P.use_tc) {
        P.total = align_up(tc_score_workspace(job.U, n_local, job.nq));
        return P;
    }
    const size_t pb = simt_score_workspace(job.U, n_local, job.nq, &P.n_chunks, &P.chunk);
    P.off_partial = 0;
    P.off_lse = align_up(pb);
    P.total = align_up(P.off_lse + (size_t)job.U * job.nq * sizeof(float));
    return P;
}

ScoreJob shard_job(const kvc_params* p, const ShardPlan& P, const void* q, const void* k, int n_local, int key_offset,
                   char* ws) {
    ScoreJob job = make_job(p, q, k);
    job.N = n_local;
    job.key_off = key_offset;
    job.n_total = p->N;
    job.err = device_error_word();
    if (P.use_tc) {
        job.tc_ws = ws;
        job.tc_ws_bytes = P.total;
        return job;
    }
    job.partial = (float2*)(ws + P.off_partial);
    job.lse = (float*)(ws + P.off_lse);
    job.n_chunks = P.n_chunks;
    job.chunk = P.chunk;
    return job;
}
}  // namespace

kvc_status kvc_shard_workspace_size(const kvc_params* p, int32_t n_local, size_t* bytes) {
    if (!bytes) return KVC_ERR_ARG;
    KVC_TRY(check_shard(p, n_local, 0));
    *bytes = shard_plan(p, n_local).total;
    return KVC_OK;
}

kvc_status kvc_shard_stats(const kvc_params* p, const void* q, const void* k_local, int32_t n_local,
                           int32_t key_offset, float* ml, void* ws, size_t ws_bytes, kvc_stream_t stream) {
    KVC_TRY(check_shard(p, n_local, key_offset));
    if (!q || !k_local || !ml || !ws) return KVC_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_local) || ((uintptr_t)ml & 7u) || ((uintptr_t)ws & (kAlign - 1)))
        return KVC_ERR_ALIGN;
    const ShardPlan P = shard_plan(p, n_local);
    if (ws_bytes < P.total) return KVC_ERR_WORKSPACE;
    const ScoreJob job = shard_job(p, P, q, k_local, n_local, key_offset, (char*)ws);
    if (!job.err) return KVC_ERR_CUDA;
    if (P.use_tc) {
        KVC_CUDA(kvc::tc_shard_stats(job, (float2*)ml, (cudaStream_t)stream));
    } else {
        KVC_CUDA(kvc::simt_shard_stats(job, (float2*)ml, (cudaStream_t)stream));
    }
    return KVC_OK;
}

kvc_status kvc_shard_scores(const kvc_params* p, const void* q, const void* k_local, int32_t n_local,
                            int32_t key_offset, const float* ml_all, int32_t n_shards, float* scores, void* ws,
                            size_t ws_bytes, kvc_stream_t stream) {
    KVC_TRY(check_shard(p, n_local, key_offset));
    if (!q || !k_local || !ml_all || !scores || !ws || n_shards < 1) return KVC_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_local) || ((uintptr_t)ml_all & 7u) || ((uintptr_t)scores & 3u) ||
        ((uintptr_t)ws & (kAlign - 1)))
        return KVC_ERR_ALIGN;
    const ShardPlan P = shard_plan(p, n_local);
    if (ws_bytes < P.total) return KVC_ERR_WORKSPACE;
    ScoreJob job = shard_job(p, P, q, k_local, n_local, key_offset, (char*)ws);
    job.unit_scores = scores;
    if (!job.err) return KVC_ERR_CUDA;
    if (P.use_tc) {
        KVC_CUDA(kvc::tc_shard_scores(job, (const float2*)ml_all, n_shards, (cudaStream_t)stream));
    } else {
        KVC_CUDA(kvc::simt_shard_scores(job, (const float2*)ml_all, n_shards, (cudaStream_t)stream));
    }
    return KVC_OK;
}

kvc_status kvc_select_hist(const float* pooled, int32_t rows, int32_t n, int32_t lo, int32_t hi,
                           const uint32_t* prefix, int32_t prefix_bits, int32_t digit_bits, uint32_t* hist,
                           kvc_stream_t stream) {
    if (!pooled || !prefix || !hist || rows < 1 || n < 1) return KVC_ERR_ARG;
    if (lo < 0 || hi > n || lo > hi || digit_bits < 1 || digit_bits > 12 || prefix_bits < 0 ||
        prefix_bits + digit_bits > 32)
        return KVC_ERR_ARG;
    KVC_CUDA(kvc::select_hist(pooled, rows, n, lo, hi, prefix, prefix_bits, digit_bits, hist, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_select_emit(const float* pooled, int32_t rows, int32_t n, int32_t lo, int32_t hi, const uint32_t* thr,
                           const int32_t* ties, int32_t pos_offset, int32_t* out, int32_t cap, int32_t* count,
                           kvc_stream_t stream) {
    if (!pooled || !thr || !ties || !out || !count || rows < 1 || n < 1 || cap < 0) return KVC_ERR_ARG;
    if (lo < 0 || hi > n || lo > hi || (long long)pos_offset + hi > (1LL << 31) - 1 ||
        (hi > lo && (long long)pos_offset + lo < 0))
        return KVC_ERR_ARG;
    KVC_CUDA(kvc::select_emit(pooled, rows, n, lo, hi, thr, ties, pos_offset, out, cap, count, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_select_pick(const uint32_t* hist, const uint32_t* hist_local, int32_t rows, int32_t digit_bits,
                           int32_t prefix_bits, int32_t* need, uint32_t* prefix, int32_t* eq_local,
                           kvc_stream_t stream) {
    if (!hist || !hist_local || !need || !prefix || !eq_local || rows < 1) return KVC_ERR_ARG;
    if (digit_bits < 1 || digit_bits > 12 || prefix_bits < 0 || prefix_bits + digit_bits > 32) return KVC_ERR_ARG;
    KVC_CUDA(kvc::select_pick(hist, hist_local, rows, digit_bits, prefix_bits, need, prefix, eq_local,
                              (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_select_ties(const int32_t* eq_all, int32_t n_shards, int32_t rank, int32_t rows, const int32_t* need,
                           int32_t* take, kvc_stream_t stream) {
    if (!eq_all || !need || !take || rows < 1 || n_shards < 1 || rank < 0 || rank >= n_shards) return KVC_ERR_ARG;
    KVC_CUDA(kvc::select_ties(eq_all, n_shards, rank, rows, need, take, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_select_kept(const int32_t* sel, const int32_t* count_sel, int32_t rows, int32_t cap_sel, int32_t N,
                           int32_t n_sink, int32_t window, int32_t key_offset, int32_t n_local, int32_t cap,
                           int32_t* pos, int32_t* local_idx, int32_t* count, kvc_stream_t stream) {
    if (!sel || !count_sel || !pos || !local_idx || !count || rows < 1 || cap_sel < 1 || cap < 1) return KVC_ERR_ARG;
    if (N < 1 || n_sink < 0 || window < 0 || key_offset < 0 || n_local < 1 || (long long)key_offset + n_local > N)
        return KVC_ERR_ARG;
    unsigned* err = device_error_word();
    if (!err) return KVC_ERR_CUDA;
    KVC_CUDA(kvc::select_kept(sel, count_sel, rows, cap_sel, N, n_sink, window, key_offset, n_local, cap, pos,
                              local_idx, count, err, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_accumulate(float* acc, const float* src, int32_t B, int32_t Hi, int32_t Ho, int32_t N,
                          kvc_stream_t stream) {
    if (!acc || !src || B < 1 || Hi < 1 || Ho < 1 || N < 0 || Hi % Ho) return KVC_ERR_ARG;
    KVC_CUDA(kvc::accumulate(acc, src, B, Hi, Ho, N, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_pool(const float* in, float* out, int32_t B, int32_t H, int32_t N, int32_t lo,
                    int32_t hi, int32_t kernel, kvc_stream_t stream) {
    if (!in || !out || in == out || B < 1 || H < 1 || N < 0) return KVC_ERR_ARG;
    if (lo < 0 || hi > N || lo > hi || kernel < 1 || kernel % 2 == 0) return KVC_ERR_ARG;
    KVC_CUDA(kvc::pool(in, out, B * H, N, lo, hi, kernel, (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_topk_workspace_size(int32_t B, int32_t H, int32_t N, size_t* bytes) {
    if (!bytes || B < 1 || H < 1 || N < 1) return KVC_ERR_ARG;
    *bytes = 0;
    return KVC_OK;
}

kvc_status kvc_topk(const float* pooled, int32_t B, int32_t H, int32_t N, int32_t n_sink,
                    int32_t window, int32_t budget, int32_t* idx, void* ws, size_t ws_bytes,
                    kvc_stream_t stream) {
    (void)ws;
    (void)ws_bytes;
    if (!pooled || !idx || B < 1 || H < 1 || N < 1 || n_sink < 0 || window < 0) return KVC_ERR_ARG;
    KVC_TRY(check_budget(N, n_sink, window, budget));
    if (kvc::topk_fused_fits(N, n_sink, window)) {
        KVC_CUDA(kvc::topk_fused(pooled, B * H, N, n_sink, window, budget, 1, idx, (cudaStream_t)stream));
    } else {
        KVC_CUDA(kvc::topk(pooled, B * H, N, n_sink, window, budget, idx, (cudaStream_t)stream));
    }
    return KVC_OK;
}

kvc_status kvc_gather(const void* src, int32_t B, int32_t Hsrc, int32_t N, size_t row_bytes,
                      const int32_t* idx, int32_t Hidx, int32_t K, void* dst, kvc_stream_t stream) {
    if (!src || !idx || !dst || B < 1 || Hsrc < 1 || N < 1 || K < 0 || row_bytes == 0) return KVC_ERR_ARG;
    if (Hidx != 1 && Hidx != Hsrc) return KVC_ERR_ARG;
    if (row_bytes % 16 || !aligned16(src) || !aligned16(dst)) return KVC_ERR_ALIGN;
    unsigned* err = device_error_word();
    if (!err) return KVC_ERR_CUDA;
    KVC_CUDA(kvc::gather(src, dst, nullptr, nullptr, B, Hsrc, N, row_bytes, idx, Hidx, K, err,
                         (cudaStream_t)stream));
    return KVC_OK;
}

kvc_status kvc_compress(const kvc_params* p, const void* q, const void* k, const void* v, void* k_out,
                        void* v_out, int32_t* idx_out, const void* hidden, void* hidden_out,
                        int32_t* tsp_idx_out, void* ws, size_t ws_bytes, kvc_stream_t stream) {
    KVC_TRY(check_params(p));
    if (!q || !k || !v || !k_out || !v_out || !idx_out || !ws) return KVC_ERR_ARG;
    const bool tsp = p->tsp_rate > 0.f;
    if (tsp) {
        if (!hidden || !hidden_out || !tsp_idx_out || p->hidden_dim < 1) return KVC_ERR_ARG;
    } else if (hidden || hidden_out || tsp_idx_out) {
        return KVC_ERR_ARG;
    }
    KVC_TRY(check_budget(p->N, p->n_sink, p->window, p->kv_budget));
    Plan P;
    make_plan(p, true, &P);
    if (tsp && P.n_tsp == 0) return KVC_ERR_BUDGET;
    const void* ptrs[] = {q, k, v, k_out, v_out, idx_out, hidden, hidden_out, tsp_idx_out};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KVC_ERR_ALIGN;
    if ((uintptr_t)ws & (kAlign - 1)) return KVC_ERR_ALIGN;
    if (tsp && ((size_t)p->hidden_dim * esize(p->dtype)) % 16) return KVC_ERR_ALIGN;
    if (ws_bytes < P.total) return KVC_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return KVC_ERR_CUDA;

    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)ws;
    const int N = p->N, S = p->n_sink, win = p->window, B = p->B, Hkv = p->Hkv;
    float* scores = (float*)(w + P.off_scores);
    float* pooled = (float*)(w + P.off_pooled);

    KVC_TRY(record_stage(p, KVC_STAGE_SCORE, s));
    KVC_TRY(run_score(p, P, q, k, scores, w, s));

    KVC_TRY(record_stage(p, KVC_STAGE_SELECT, s));
    const bool fused = kvc::topk_fused_fits(N, S, win);
    if (fused) {
        KVC_CUDA(kvc::topk_fused(scores, B * P.Hs, N, S, win, p->kv_budget, p->pool_kernel, idx_out, s));
    } else {
        KVC_CUDA(kvc::pool(scores, pooled, B * P.Hs, N, S, N - win, p->pool_kernel, s));
        KVC_CUDA(kvc::topk(pooled, B * P.Hs, N, S, win, p->kv_budget, idx_out, s));
    }
    if (tsp) {
        float* tsp_scores = (float*)(w + P.off_tsp_scores);
        float* tsp_pooled = (float*)(w + P.off_tsp_pooled);
        const float* src = scores;
        if (P.Hs > 1) {
            KVC_CUDA(cudaMemsetAsync(tsp_scores, 0, (size_t)B * N * sizeof(float), s));
            KVC_CUDA(kvc::accumulate(tsp_scores, scores, B, P.Hs, 1, N, s));
            src = tsp_scores;
        }
        if (fused) {
            KVC_CUDA(kvc::topk_fused(src, B, N, S, win, P.n_tsp, p->pool_kernel, tsp_idx_out, s));
        } else {
            KVC_CUDA(kvc::pool(src, tsp_pooled, B, N, S, N - win, p->pool_kernel, s));
            KVC_CUDA(kvc::topk(tsp_pooled, B, N, S, win, P.n_tsp, tsp_idx_out, s));
        }
    }

    KVC_TRY(record_stage(p, KVC_STAGE_GATHER, s));
    const size_t row = (size_t)p->D * esize(p->dtype);
    const char* k_last = (const char*)k + (size_t)(p->n_layers - 1) * B * Hkv * N * row;
    KVC_CUDA(kvc::gather(k_last, k_out, v, v_out, B, Hkv, N, row, idx_out, P.Hs, p->kv_budget, err, s));
    if (tsp) {
        KVC_CUDA(kvc::gather(hidden, hidden_out, nullptr, nullptr, B, 1, N,
                             (size_t)p->hidden_dim * esize(p->dtype), tsp_idx_out, 1, P.n_tsp, err, s));
    }
    KVC_TRY(record_stage(p, KVC_STAGE_COUNT, s));
    return KVC_OK;
}

int32_t kvc_tsp_count(int32_t N, int32_t window, int32_t n_sink, float tsp_rate) {
    if (!(tsp_rate > 0.f) || N < 1) return 0;
    long long sel = (long long)floor((double)tsp_rate * (double)N);
    const long long n_c = (long long)N - window - n_sink;
    if (sel > n_c) sel = n_c;
    if (sel < 1) return 0;
    return (int32_t)(sel + n_sink + window);
}

kvc_status kvc_poll_error(kvc_stream_t stream) {
    unsigned* err = device_error_word();
    if (!err) return KVC_ERR_CUDA;
    unsigned h = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KVC_ERR_CUDA;
    if (cudaMemcpy(&h, err, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return KVC_ERR_CUDA;
    if (h) {
        const unsigned zero = 0;
        if (cudaMemcpy(err, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return KVC_ERR_CUDA;
    }
    if (h & kErrTimeout) return KVC_ERR_TIMEOUT;
    if (h & kErrIndex) return KVC_ERR_INDEX;
    if (h & kErrCheck) return KVC_ERR_CHECK;
    return KVC_OK;
}

int32_t kvc_checks_enabled(void) { return kChecks ? 1 : 0; }

const char* kvc_status_string(kvc_status st) {
    switch (st) {
        case KVC_OK: return "ok";
        case KVC_ERR_ARG: return "invalid argument (null pointer or bad shape)";
        case KVC_ERR_UNSUPPORTED: return "unsupported configuration (head dim, dtype, scope or window size)";
        case KVC_ERR_BUDGET: return "budget out of range (needs n_sink + window + 1 <= budget <= N)";
        case KVC_ERR_ALIGN: return "misaligned pointer or row size (16 bytes; workspace 256 bytes)";
        case KVC_ERR_WORKSPACE: return "workspace too small";
        case KVC_ERR_CUDA: return "CUDA runtime error";
        case KVC_ERR_TIMEOUT: return "a device-side bounded wait gave up";
        case KVC_ERR_INDEX: return "gather index out of range";
        case KVC_ERR_CHECK: return "a device-side range check failed (checks build)";
    }
    return "unknown status";
}

uint64_t kvc_launch_count(void) { return (uint64_t)g_launches.load(std::memory_order_relaxed); }

const char* kvc_version(void) { return "kvc 0.1.0 sm_100a"; }

}  // extern "C"

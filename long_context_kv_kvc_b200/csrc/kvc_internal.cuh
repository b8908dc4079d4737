// kvc_internal.cuh -- declarations shared by the translation units of libkvc.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvc.h"

namespace kvc {

constexpr int kHeadDim = 128;  // D: the only head dimension the kernels are built for

// bits of the per-device error word (see kvc_poll_error)
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrIndex = 2u;
constexpr unsigned kErrCheck = 4u;  // a device-side range check failed (checks build only)

// Device-side range checks.  Built with -DKVC_CHECKS=1 (libkvc_checks.so), every kernel tests
// the indices and coordinates it forms against the extents of the buffers they address; a
// failed test sets kErrCheck in the error word and the access is skipped.  In the regular
// build dcheck is the constant true and the tests compile away.
#if defined(KVC_CHECKS) && KVC_CHECKS
constexpr bool kChecks = true;
#else
constexpr bool kChecks = false;
#endif

__device__ __forceinline__ bool dcheck(unsigned* err, bool ok) {
    if constexpr (kChecks) {
        if (!ok) {
            if (err) atomicOr(err, kErrCheck);
            return false;
        }
    }
    return true;
}

// index i in [0, n)
__device__ __forceinline__ bool dcheck_idx(unsigned* err, long long i, long long n) {
    return dcheck(err, i >= 0 && i < n);
}

// counts kernel launches issued by the library (kvc_launch_count)
void count_launches(int n);

// per-device error word, set by kernels with atomicOr, read and cleared by kvc_poll_error
unsigned int* device_error_word();

// log2(e) / sqrt(128): logits are taken to base 2 so that exp becomes exp2
constexpr float kLog2eOverSqrtD = 0.12751743082459868f;

// One scoring job: every (layer, batch, KV head) "unit" u = (layer*B + b)*Hkv + h.
// Unit u reads the G*window query rows starting at q + u*G*window*D (heads h*G..h*G+G-1
// are adjacent) and the N key rows starting at k + u*N*D.
struct ScoreJob {
    const void* q;
    const void* k;
    int dtype;
    int U;        // units = n_layers * B * Hkv
    int N;        // keys per unit in k
    int key_off;  // sequence sharding: position of k's first key in the whole sequence
    int n_total;  // sequence sharding: keys of the whole sequence (0: N)
    int window;
    int G;
    int nq;       // G * window query rows per unit
    float* unit_scores;  // [U][N] fp32 output (sum over the unit's query rows)
    float* entropy;      // [U][nq] attention entropy per window row (nats), or null
    // workspace
    float2* partial;     // SIMT: [U][n_chunks][nq] (m, l) partial softmax stats
    float* partial_t;    // SIMT with entropy: [U][n_chunks][nq] sum 2^(y - m) (y - m)
    float* lse;          // [U][nq] log2-sum-exp per query row
    int n_chunks;
    int chunk;
    // tensor-core path
    void* tc_ws;
    size_t tc_ws_bytes;
    unsigned* err;
    long long spin_limit;
    int inject_timeout;  // test hook: the cross-CTA wait watches a flag nothing sets
};

// CUDA-core (FFMA) scoring, fp32 or bf16 inputs
size_t simt_score_workspace(int U, int N, int nq, int* n_chunks, int* chunk);
cudaError_t simt_score(const ScoreJob& job, cudaStream_t s);
// sequence sharding: this block of keys' (m, l) per (unit, window row); then the scores of the
// block's keys given every shard's (m, l) [W][U * nq] (merged into job.lse in shard order)
cudaError_t simt_shard_stats(const ScoreJob& job, float2* ml, cudaStream_t s);
cudaError_t simt_shard_scores(const ScoreJob& job, const float2* ml_all, int W, cudaStream_t s);

// tensor-core scoring (bf16, tcgen05 + TMA); returns false if the shape is not supported
bool tc_score_supported(const ScoreJob& job);
size_t tc_score_workspace(int U, int N, int nq);
cudaError_t tc_score(const ScoreJob& job, cudaStream_t s);
// sequence sharding on the tensor cores: this block's (m, l) per (unit, row) (phase 1 only),
// then the block's scores given every shard's (m, l) [W][U * nq] (phase 2 only)
cudaError_t tc_shard_stats(const ScoreJob& job, float2* ml, cudaStream_t s);
cudaError_t tc_shard_scores(const ScoreJob& job, const float2* ml_all, int W, cudaStream_t s);

// sums of unit scores over layers (and KV heads for the all-heads scope)
cudaError_t reduce_units(const float* unit_scores, int L, int B, int Hkv, int N, int all_heads,
                         float* out, cudaStream_t s);
cudaError_t accumulate(float* acc, const float* src, int B, int Hi, int Ho, int N, cudaStream_t s);
cudaError_t pool(const float* in, float* out, int rows, int N, int lo, int hi, int kernel,
                 cudaStream_t s);
cudaError_t topk(const float* pooled, int rows, int N, int n_sink, int window, int budget,
                 int32_t* idx, cudaStream_t s);
// pool (odd width `kernel` over [n_sink, N - window)) and top-k in one launch, one 8-CTA
// cluster per row; for rows whose candidates fit the clusters' shared memory
bool topk_fused_fits(int N, int n_sink, int window);
// distributed radix select over a sharded score row (select.cu)
cudaError_t select_hist(const float* pooled, int rows, int n, int lo, int hi, const uint32_t* prefix, int prefix_bits,
                        int digit_bits, uint32_t* hist, cudaStream_t s);
cudaError_t select_emit(const float* pooled, int rows, int n, int lo, int hi, const uint32_t* thr, const int32_t* ties,
                        int pos_offset, int32_t* out, int cap, int32_t* count, cudaStream_t s);
cudaError_t select_pick(const uint32_t* hist, const uint32_t* hist_local, int rows, int digit_bits, int prefix_bits,
                        int32_t* need, uint32_t* prefix, int32_t* eq_local, cudaStream_t s);
cudaError_t select_ties(const int32_t* eq_all, int W, int rank, int rows, const int32_t* need, int32_t* take,
                        cudaStream_t s);
cudaError_t select_kept(const int32_t* sel, const int32_t* cnt, int rows, int cap_sel, int N, int S, int w,
                        int key_off, int n_local, int cap, int32_t* pos, int32_t* local, int32_t* count,
                        unsigned* err, cudaStream_t s);
cudaError_t topk_fused(const float* scores, int rows, int N, int n_sink, int window, int budget, int kernel,
                       int32_t* idx, cudaStream_t s);
// two gathers of the same shape in one launch (src1/dst1 may be null)
cudaError_t gather(const void* src0, void* dst0, const void* src1, void* dst1, int B, int Hsrc,
                   int N, size_t row_bytes, const int32_t* idx, int Hidx, int K, unsigned* err,
                   cudaStream_t s);

// per score row: share of mass at the kept positions (when idx is not null) and population
// variance over the candidates [S, N - w)
cudaError_t row_stats(const float* scores, int rows, int N, int S, int w, const int32_t* idx, int budget,
                      float* kept_mass, float* cand_var, unsigned* err, cudaStream_t s);

// CentroidKV Chunked Soft Matching (csm.cu): merges m = csm_merges(...) A tokens per row
int csm_merges(int N, int S, int w, int chunk, float ratio);
size_t csm_workspace(int rows, int N, int m);
cudaError_t csm(const void* k, const void* v, int dtype, const int32_t* deg, const int32_t* pos, int rows, int N,
                long long ld_in, int S, int w, int chunk, int m, void* k_out, void* v_out, int32_t* deg_out,
                int32_t* pos_out, long long ld_out, void* ws, cudaStream_t s);

// decode attention over a (clustered) cache (decode.cu): U = B * Hkv units of Rv = G * nq
// query rows each, n cached rows at a row stride of ld tokens; out [U * Rv][128] fp32
bool decode_rows_supported(int rows_per_kv_head);
size_t decode_workspace(int U, int Rv, int n);
cudaError_t decode_attention(const void* q, const void* k, const void* v, const int32_t* deg, int dtype, int U,
                             int Rv, int n, long long ld, float* out, void* ws, cudaStream_t s);
// appends t_new rows per unit to caches of row stride ld holding n rows (decode.cu)
cudaError_t append_rows(void* k_cache, void* v_cache, int32_t* deg_cache, int32_t* pos_cache, int dtype, int U,
                        long long ld, int n, const void* k_new, const void* v_new, int t_new, int pos0, cudaStream_t s);

}  // namespace kvc

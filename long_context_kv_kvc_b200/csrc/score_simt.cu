// score_simt.cu -- window-softmax saliency scores on the CUDA cores (FFMA, fp32 accumulate).
//
// This is the scoring path for fp32 inputs (where tensor-core TF32 would lose the 1e-3
// score tolerance) and the reference path on the GPU for bf16 inputs.  It runs in three
// launches per call:
//   1. stats:   per (unit, key chunk, query row) the partial base-2 softmax statistics
//               (m, l) = (max y, sum 2^(y - m)) over the visible keys of the chunk,
//               y = q.k * log2(e)/sqrt(D);
//   2. combine: per (unit, query row) lse = M + log2(sum_c l_c 2^(m_c - M)), fixed order;
//   3. scores:  per key j, s_j = sum over query rows r of 2^(y_rj - lse_r), masked for keys
//               after the row's position (causal window).
// With an entropy output the statistics carry t = sum 2^(y - m) (y - m) as well, and the
// combine step writes each row's attention entropy ln2 (log2 l - t / l) in nats (StructKV
// page, sec. 2: attention entropy is one of the signals watched for the pivot layer).
// The definition is the plain window softmax: the FastKV page (sec. 2A) selects tokens by
// a saliency score, and the SnapKV scoring it names uses the softmaxed attention of the
// observation window; all sums run in a fixed order so results are deterministic.
#include <math.h>

#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr int D = kHeadDim;
constexpr int kThreads = 256;
constexpr int kQB = 32;        // query rows per block pass
constexpr int kKT = 32;        // keys per shared-memory tile
constexpr int kKPT = kKT / 8;  // keys per thread (8 threads share a query row)
constexpr int kChunkMax = 2048;

__device__ __forceinline__ float load_elem(const float* p, size_t i) { return __ldg(p + i); }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}

// Copies `rows` rows of D elements starting at `src` (rows beyond `valid` are zero) into
// a padded fp32 shared array.
template <typename T>
__device__ __forceinline__ void stage_rows(float (*dst)[D + 1], const T* src, int rows, int valid) {
    for (int e = threadIdx.x; e < rows * D; e += kThreads) {
        const int r = e / D, d = e % D;
        dst[r][d] = r < valid ? load_elem(src, (size_t)r * D + d) : 0.f;
    }
}

__device__ __forceinline__ void merge_stats(float& m, float& l, float m2, float l2) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;
    l = (m == -INFINITY ? 0.f : l * exp2f(m - M)) + (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - M));
    m = M;
}

// The same merge for (m, l, t) with t = sum 2^(y - m) (y - m): moving the reference from m
// to M scales the sums by 2^(m - M) and shifts each y - m by m - M.  l is formed by the very
// expression of merge_stats, so the entropy pass leaves the statistics (and the scores)
// bit-identical.
__device__ __forceinline__ void merge_stats3(float& m, float& l, float& t, float m2, float l2, float t2) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;
    float T = 0.f;
    if (m != -INFINITY) T += exp2f(m - M) * (t + (m - M) * l);
    if (m2 != -INFINITY) T += exp2f(m2 - M) * (t2 + (m2 - M) * l2);
    l = (m == -INFINITY ? 0.f : l * exp2f(m - M)) + (m2 == -INFINITY ? 0.f : l2 * exp2f(m2 - M));
    m = M;
    t = T;
}

template <typename T, bool ENT>
__global__ void __launch_bounds__(kThreads)
stats_kernel(const T* __restrict__ q, const T* __restrict__ k, int N, int key_off, int n_total, int w, int nq,
             int chunk, int n_chunks, float2* __restrict__ partial, float* __restrict__ partial_t, unsigned* err) {
    __shared__ float Qs[kQB][D + 1];
    __shared__ float Ks[kKT][D + 1];
    const int u = blockIdx.y, c = blockIdx.x;
    const int j0 = c * chunk, j1 = min(N, j0 + chunk);
    // the chunk is a non-empty slice of the unit's keys and a column of the partials
    if (!dcheck(err, j0 < j1 && c < n_chunks)) return;
    const T* qu = q + (size_t)u * nq * D;
    const T* ku = k + (size_t)u * N * D;
    const int tid = threadIdx.x, qi = tid >> 3, kj = tid & 7;

    for (int qb = 0; qb < nq; qb += kQB) {
        __syncthreads();
        stage_rows(Qs, qu + (size_t)qb * D, kQB, nq - qb);
        const int r = qb + qi;
        // position of window query r, in this block of keys (which starts at key_off of n_total)
        const int t_r = r < nq ? n_total - w + r % w - key_off : -1;
        float m = -INFINITY, l = 0.f, tt = 0.f;
        for (int jt = j0; jt < j1; jt += kKT) {
            __syncthreads();
            stage_rows(Ks, ku + (size_t)jt * D, kKT, j1 - jt);
            __syncthreads();
            float acc[kKPT];
#pragma unroll
            for (int t = 0; t < kKPT; ++t) acc[t] = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) {
                const float qv = Qs[qi][d];
#pragma unroll
                for (int t = 0; t < kKPT; ++t) acc[t] = fmaf(qv, Ks[kj + 8 * t][d], acc[t]);
            }
#pragma unroll
            for (int t = 0; t < kKPT; ++t) {
                const int j = jt + kj + 8 * t;
                if (j < j1 && j <= t_r) {
                    const float y = acc[t] * kLog2eOverSqrtD;
                    if (y > m) {
                        if (m == -INFINITY) {
                            l = 1.f;
                            tt = 0.f;
                        } else {
                            const float f = exp2f(m - y);
                            if (ENT) tt = f * (tt + (m - y) * l);
                            l = l * f + 1.f;
                        }
                        m = y;
                    } else {
                        const float e = exp2f(y - m);
                        l += e;
                        if (ENT) tt = fmaf(e, y - m, tt);
                    }
                }
            }
        }
        // combine the 8 threads that share query row r (adjacent lanes)
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
            if (ENT) {
                const float t2 = __shfl_xor_sync(0xffffffffu, tt, off);
                merge_stats3(m, l, tt, m2, l2, t2);
            } else {
                merge_stats(m, l, m2, l2);
            }
        }
        if (kj == 0 && r < nq) {
            partial[((size_t)u * n_chunks + c) * nq + r] = make_float2(m, l);
            if (ENT) partial_t[((size_t)u * n_chunks + c) * nq + r] = tt;
        }
    }
}

// lse per row; with `entropy`, also each row's attention entropy in nats: with the chunks'
// (m, l, t) moved to the common reference M, E[y] = M + T / L and lse = M + log2 L, so
// -sum p ln p = ln2 (lse - E[y]) = ln2 (log2 L - T / L).
__global__ void combine_kernel(const float2* __restrict__ partial, const float* __restrict__ partial_t,
                               int n_chunks, int nq, float* __restrict__ lse, float* __restrict__ entropy) {
    const int u = blockIdx.x;
    for (int r = threadIdx.x; r < nq; r += blockDim.x) {
        const float2* p = partial + (size_t)u * n_chunks * nq + r;
        float M = -INFINITY;
        for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, p[(size_t)c * nq].x);
        float S = 0.f, T = 0.f;
        for (int c = 0; c < n_chunks; ++c) {
            const float2 v = p[(size_t)c * nq];
            if (v.x != -INFINITY) {
                const float f = exp2f(v.x - M);
                S += v.y * f;
                if (entropy) T += f * (partial_t[((size_t)u * n_chunks + c) * nq + r] + (v.x - M) * v.y);
            }
        }
        lse[(size_t)u * nq + r] = M + log2f(S);
        if (entropy) entropy[(size_t)u * nq + r] = 0.69314718055994531f * (log2f(S) - T / S);
    }
}

// Sequence sharding: this block's (m, l) per (unit, row), the chunk partials merged in
// chunk order (M = -inf, l = 0 when the block holds no key the row sees).
__global__ void shard_ml_kernel(const float2* __restrict__ partial, int n_chunks, int nq, float2* __restrict__ ml) {
    const int u = blockIdx.x;
    for (int r = threadIdx.x; r < nq; r += blockDim.x) {
        const float2* p = partial + (size_t)u * n_chunks * nq + r;
        float M = -INFINITY;
        for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, p[(size_t)c * nq].x);
        float S = 0.f;
        if (M != -INFINITY)
            for (int c = 0; c < n_chunks; ++c) {
                const float2 v = p[(size_t)c * nq];
                if (v.x != -INFINITY) S += v.y * exp2f(v.x - M);
            }
        ml[(size_t)u * nq + r] = make_float2(M, S);
    }
}

// lse per row from every shard's (m, l), merged in shard order (so every shard computes the
// same value): ml_all [W][rows].
__global__ void shard_lse_kernel(const float2* __restrict__ ml_all, int W, int rows, float* __restrict__ lse) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += gridDim.x * blockDim.x) {
        float M = -INFINITY;
        for (int w = 0; w < W; ++w) M = fmaxf(M, ml_all[(size_t)w * rows + i].x);
        float S = 0.f;
        for (int w = 0; w < W; ++w) {
            const float2 v = ml_all[(size_t)w * rows + i];
            if (v.x != -INFINITY) S += v.y * exp2f(v.x - M);
        }
        lse[i] = M + log2f(S);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
scores_kernel(const T* __restrict__ q, const T* __restrict__ k, int N, int key_off, int n_total, int w, int nq,
              int chunk, const float* __restrict__ lse, float* __restrict__ out, unsigned* err) {
    __shared__ float Qs[kQB][D + 1];
    __shared__ float Ks[kKT][D + 1];
    __shared__ float Ls[kQB];
    __shared__ float red[kThreads / 32][kKT];
    __shared__ float sacc[kChunkMax];
    const int u = blockIdx.y, c = blockIdx.x;
    const int j0 = c * chunk, j1 = min(N, j0 + chunk);
    const T* qu = q + (size_t)u * nq * D;
    const T* ku = k + (size_t)u * N * D;
    const int tid = threadIdx.x, qi = tid >> 3, kj = tid & 7, warp = tid >> 5, lane = tid & 31;
    // the chunk's sums fit the shared accumulator
    if (!dcheck(err, j0 < j1 && j1 - j0 <= kChunkMax)) return;

    for (int j = tid; j < j1 - j0; j += kThreads) sacc[j] = 0.f;
    for (int qb = 0; qb < nq; qb += kQB) {
        __syncthreads();
        stage_rows(Qs, qu + (size_t)qb * D, kQB, nq - qb);
        if (tid < kQB) Ls[tid] = qb + tid < nq ? lse[(size_t)u * nq + qb + tid] : INFINITY;
        const int r = qb + qi;
        const int t_r = r < nq ? n_total - w + r % w - key_off : -1;
        for (int jt = j0; jt < j1; jt += kKT) {
            __syncthreads();
            stage_rows(Ks, ku + (size_t)jt * D, kKT, j1 - jt);
            __syncthreads();
            float acc[kKPT];
#pragma unroll
            for (int t = 0; t < kKPT; ++t) acc[t] = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) {
                const float qv = Qs[qi][d];
#pragma unroll
                for (int t = 0; t < kKPT; ++t) acc[t] = fmaf(qv, Ks[kj + 8 * t][d], acc[t]);
            }
            const float L = Ls[qi];
            float p[kKPT];
#pragma unroll
            for (int t = 0; t < kKPT; ++t) {
                const int j = jt + kj + 8 * t;
                p[t] = (j < j1 && j <= t_r) ? exp2f(fmaf(acc[t], kLog2eOverSqrtD, -L)) : 0.f;
                // sum over the 4 query rows of this warp (lanes with equal kj)
                p[t] += __shfl_xor_sync(0xffffffffu, p[t], 8);
                p[t] += __shfl_xor_sync(0xffffffffu, p[t], 16);
            }
            if (lane < 8) {
#pragma unroll
                for (int t = 0; t < kKPT; ++t) red[warp][kj + 8 * t] = p[t];
            }
            __syncthreads();
            if (tid < kKT && jt + tid < j1) {
                float s = 0.f;
#pragma unroll
                for (int wi = 0; wi < kThreads / 32; ++wi) s += red[wi][tid];
                sacc[jt - j0 + tid] += s;
            }
        }
    }
    __syncthreads();
    for (int j = j0 + tid; j < j1; j += kThreads) out[(size_t)u * N + j] = sacc[j - j0];
}

}  // namespace

// partial (m, l) per (unit, chunk, row); the entropy's t per (unit, chunk, row) is a separate
// array of half that size (ScoreJob::partial_t)
size_t simt_score_workspace(int U, int N, int nq, int* n_chunks_out, int* chunk_out) {
    // enough CTAs to fill the GPU about twice, chunks of at most kChunkMax keys
    long long target = 148LL * 2;
    long long chunk = ((long long)N * U + target - 1) / target;
    chunk = ((chunk + kKT - 1) / kKT) * kKT;
    if (chunk < kKT) chunk = kKT;
    if (chunk > kChunkMax) chunk = kChunkMax;
    const int n_chunks = (int)((N + chunk - 1) / chunk);
    if (n_chunks_out) *n_chunks_out = n_chunks;
    if (chunk_out) *chunk_out = (int)chunk;
    return (size_t)U * n_chunks * nq * sizeof(float2);
}

namespace {

cudaError_t launch_stats(const ScoreJob& j, cudaStream_t s) {
    dim3 grid(j.n_chunks, j.U);
    const int n_total = j.n_total > 0 ? j.n_total : j.N;
    float* partial_t = j.partial_t;
    const bool ent = j.entropy != nullptr;
    if (j.dtype == KVC_F32) {
        if (ent)
            stats_kernel<float, true><<<grid, kThreads, 0, s>>>((const float*)j.q, (const float*)j.k, j.N, j.key_off,
                                                                 n_total, j.window, j.nq, j.chunk, j.n_chunks,
                                                                 j.partial, partial_t, j.err);
        else
            stats_kernel<float, false><<<grid, kThreads, 0, s>>>((const float*)j.q, (const float*)j.k, j.N,
                                                                  j.key_off, n_total, j.window, j.nq, j.chunk,
                                                                  j.n_chunks, j.partial, partial_t, j.err);
    } else {
        if (ent)
            stats_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, s>>>(
                (const __nv_bfloat16*)j.q, (const __nv_bfloat16*)j.k, j.N, j.key_off, n_total, j.window, j.nq,
                j.chunk, j.n_chunks, j.partial, partial_t, j.err);
        else
            stats_kernel<__nv_bfloat16, false><<<grid, kThreads, 0, s>>>(
                (const __nv_bfloat16*)j.q, (const __nv_bfloat16*)j.k, j.N, j.key_off, n_total, j.window, j.nq,
                j.chunk, j.n_chunks, j.partial, partial_t, j.err);
    }
    return cudaGetLastError();
}

cudaError_t launch_scores(const ScoreJob& j, cudaStream_t s) {
    dim3 grid(j.n_chunks, j.U);
    const int n_total = j.n_total > 0 ? j.n_total : j.N;
    if (j.dtype == KVC_F32) {
        scores_kernel<float><<<grid, kThreads, 0, s>>>((const float*)j.q, (const float*)j.k, j.N, j.key_off, n_total,
                                                        j.window, j.nq, j.chunk, j.lse, j.unit_scores, j.err);
    } else {
        scores_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
            (const __nv_bfloat16*)j.q, (const __nv_bfloat16*)j.k, j.N, j.key_off, n_total, j.window, j.nq, j.chunk,
            j.lse, j.unit_scores, j.err);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t simt_score(const ScoreJob& j, cudaStream_t s) {
    count_launches(3);
    cudaError_t e = launch_stats(j, s);
    if (e != cudaSuccess) return e;
    combine_kernel<<<j.U, 128, 0, s>>>(j.partial, j.partial_t, j.n_chunks, j.nq, j.lse, j.entropy);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_scores(j, s);
}

cudaError_t simt_shard_stats(const ScoreJob& j, float2* ml, cudaStream_t s) {
    count_launches(2);
    cudaError_t e = launch_stats(j, s);
    if (e != cudaSuccess) return e;
    shard_ml_kernel<<<j.U, 128, 0, s>>>(j.partial, j.n_chunks, j.nq, ml);
    return cudaGetLastError();
}

cudaError_t simt_shard_scores(const ScoreJob& j, const float2* ml_all, int W, cudaStream_t s) {
    count_launches(2);
    const int rows = j.U * j.nq;
    shard_lse_kernel<<<(rows + 255) / 256, 256, 0, s>>>(ml_all, W, rows, j.lse);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_scores(j, s);
}

}  // namespace kvc

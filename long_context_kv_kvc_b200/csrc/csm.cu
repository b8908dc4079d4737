// csm.cu -- CentroidKV's Chunked Soft Matching: one clustering round over a KV cache.
//
// What it computes (CentroidKV page, sec. 3 "Chunked Soft Matching" and sec. 4
// "Aggregatie"), per row (batch, KV head) of N cached tokens with degrees n_t:
//   * the candidates C = [S, N - w) are cut into chunks of `chunk` tokens; sinks and the
//     recent window are left as they are (sec. 2, Preservation);
//   * inside a chunk the tokens at even offsets form set A, the odd ones set B; each A token
//     is matched with the B token of its chunk whose key has the largest cosine similarity
//     to its own (ties: lower position; a zero key has similarity 0);
//   * the m = min(floor(r |C|), matchable A tokens) matches with the largest similarity
//     merge (ties: lower position): a B token and the A tokens merged into it become their
//     degree-weighted mean, keys and values alike, and their degrees add;
//   * the cache keeps every token except the merged A tokens, in position order.
// Design for B200.  Two HBM passes over the cache (matching needs the row's global top-m
// before any row can be written):
//   1. match: the similarities of a chunk form a dense contraction, so for bf16 keys a
//      persistent tensor-core kernel streams 128-token tiles (a whole number of chunks) with
//      TMA and forms each tile's Gram matrix K K^T in TMEM (tcgen05.mma, fp32 accumulate;
//      products of bf16 values are exact); its diagonal gives the norms, and the thread that
//      owns an A token's TMEM lane takes the argmax over its chunk's B columns.  fp32 keys
//      use a CUDA-core kernel over the chunk staged in shared memory;
//   2. the m best matches per row: the radix top-k over the row's A-token match scores (the
//      A tokens are S + 2i because chunks are even; -inf where there is no match), then merge
//      flags and per-chunk merge counts, and a per-row scan of the kept tokens per chunk that
//      gives every chunk its first output slot;
//   3. write: one CTA per chunk (or per 128 sink / window tokens) brings the block's K and V
//      rows into shared memory with two bulk copies (a block's rows are contiguous), forms
//      the merged means there in fp32 (rounded once to the element type), and sends every
//      run of consecutive kept rows to its output slots with one bulk store per tensor;
//      every other row is thus copied bit for bit.
#include <math.h>

#include <algorithm>
#include <atomic>

#include "kvc_internal.cuh"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

constexpr int D = kHeadDim;
constexpr int kMatchThreads = 256;
constexpr int kKS = D + 4;  // shared-memory row stride of a staged fp32 key (16-byte aligned rows)
constexpr int kScanThreads = 1024;
constexpr int kWriteThreads = 128;  // one thread per token of a block
constexpr int kSeg = 128;  // sink / window tokens per write CTA

// tensor-core match
constexpr int kTileTok = 128;                // Gram tile: MMA M = N = 128 tokens, K = 128 dimensions
constexpr int kHalfBytes = kTileTok * 64 * 2;  // one 64-dimension half of a tile: 16 KiB
constexpr int kTcStages = 5;
constexpr int kTcAcc = 4;                    // TMEM accumulators = epilogue warpgroups
constexpr int kTcThreads = (2 + 4 * kTcAcc) * 32;  // warp 0 TMA, 1 MMA + TMEM owner, 2.. epilogue
constexpr int kTcMaxCtas = 160;
constexpr uint32_t kTcCols = 128 * kTcAcc;

// ------------------------------------------------------------------------ row pieces
// A lane handles 8 elements of a row: one 16-byte vector for bf16, two for fp32.

template <typename T>
struct Vec {
    static constexpr int n = sizeof(T) / 2;
};

__device__ __forceinline__ void to_f8(const uint4 (&r)[1], float (&x)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r[0]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void to_f8(const uint4 (&r)[2], float (&x)[8]) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        x[4 * i] = __uint_as_float(r[i].x);
        x[4 * i + 1] = __uint_as_float(r[i].y);
        x[4 * i + 2] = __uint_as_float(r[i].z);
        x[4 * i + 3] = __uint_as_float(r[i].w);
    }
}
__device__ __forceinline__ void from_f8(const float (&x)[8], uint4 (&r)[1]) {
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r[0]);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
}
__device__ __forceinline__ void from_f8(const float (&x)[8], uint4 (&r)[2]) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
        r[i] = make_uint4(__float_as_uint(x[4 * i]), __float_as_uint(x[4 * i + 1]), __float_as_uint(x[4 * i + 2]),
                          __float_as_uint(x[4 * i + 3]));
}

// ------------------------------------------------------------------------ match, fp32 keys

// One CTA per (row, chunk), blockIdx.x = row * n_chunks + chunk.  Chunks start at even
// offsets from S (chunk is even), so the A tokens are the positions S + 2i: score[i] = the
// match similarity of A token i (-inf without a match), a row of n_A = ceil(|C| / 2) entries;
// best[pos] = the matched B position.  The keys are staged in shared memory; each thread
// forms a 2 x 2 block of A-B dot products.
__global__ void __launch_bounds__(kMatchThreads)
csm_match_f32_kernel(const float* __restrict__ k, int N, long long ld, int S, int w, int chunk, int n_chunks,
                     int n_a_row, float* __restrict__ score, int32_t* __restrict__ best, unsigned* err) {
    extern __shared__ __align__(16) float ks[];  // [chunk][kKS]
    __shared__ float inv_norm[128];
    __shared__ float sim[64][65];                // [A index][B index]
    const int row = blockIdx.x / n_chunks, q = blockIdx.x - row * n_chunks;
    const int hi = N - w;
    const int c0 = S + q * chunk, c1 = min(c0 + chunk, hi);
    const int len = c1 - c0;
    const float* kr = k + (size_t)row * ld * D;
    float* sr = score + (size_t)row * n_a_row + (c0 - S) / 2;  // A token 0 of this chunk
    int32_t* br = best + (size_t)row * N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kW = kMatchThreads / 32;
    // a non-empty chunk of at most 128 tokens (64 A x 64 B similarities) whose A tokens fit the
    // row's score entries
    if (!dcheck(err, len >= 1 && len <= chunk && chunk <= 128 && (c0 - S) / 2 + (len + 1) / 2 <= n_a_row)) return;

    for (int e = threadIdx.x; e < len * (D / 4); e += kMatchThreads) {
        const int t = e / (D / 4), d = (e - t * (D / 4)) * 4;
        *reinterpret_cast<float4*>(ks + t * kKS + d) = __ldcs(reinterpret_cast<const float4*>(kr + (size_t)(c0 + t) * D + d));
    }
    __syncthreads();
    // 1 / |k| (0 for a zero key, which makes its similarity 0)
    for (int t = warp; t < len; t += kW) {
        const float4 v = *reinterpret_cast<const float4*>(ks + t * kKS + 4 * lane);
        float s = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) inv_norm[t] = s > 0.f ? rsqrtf(s) : 0.f;
    }
    __syncthreads();
    const int n_a = (len + 1) / 2, n_b = len / 2;  // A at offsets 0, 2, ...; B at 1, 3, ...
    // thread (ia, ib) forms A {ia, ia + 32} x B {ib, ib + 32} (n_a, n_b <= 64)
    for (int tile = threadIdx.x; tile < 32 * 32; tile += kMatchThreads) {
        const int ia = tile >> 5, ib = tile & 31;
        if (ia >= n_a || ib >= n_b) continue;
        const bool a2 = ia + 32 < n_a, b2 = ib + 32 < n_b;
        const float* pa0 = ks + (2 * ia) * kKS;
        const float* pa1 = ks + (2 * (a2 ? ia + 32 : ia)) * kKS;
        const float* pb0 = ks + (2 * ib + 1) * kKS;
        const float* pb1 = ks + (2 * (b2 ? ib + 32 : ib) + 1) * kKS;
        float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            const float4 x0 = *reinterpret_cast<const float4*>(pa0 + d), x1 = *reinterpret_cast<const float4*>(pa1 + d);
            const float4 y0 = *reinterpret_cast<const float4*>(pb0 + d), y1 = *reinterpret_cast<const float4*>(pb1 + d);
            s00 = fmaf(x0.x, y0.x, s00); s00 = fmaf(x0.y, y0.y, s00); s00 = fmaf(x0.z, y0.z, s00); s00 = fmaf(x0.w, y0.w, s00);
            s01 = fmaf(x0.x, y1.x, s01); s01 = fmaf(x0.y, y1.y, s01); s01 = fmaf(x0.z, y1.z, s01); s01 = fmaf(x0.w, y1.w, s01);
            s10 = fmaf(x1.x, y0.x, s10); s10 = fmaf(x1.y, y0.y, s10); s10 = fmaf(x1.z, y0.z, s10); s10 = fmaf(x1.w, y0.w, s10);
            s11 = fmaf(x1.x, y1.x, s11); s11 = fmaf(x1.y, y1.y, s11); s11 = fmaf(x1.z, y1.z, s11); s11 = fmaf(x1.w, y1.w, s11);
        }
        const float na0 = inv_norm[2 * ia], nb0 = inv_norm[2 * ib + 1];
        sim[ia][ib] = s00 * na0 * nb0;
        if (b2) sim[ia][ib + 32] = s01 * na0 * inv_norm[2 * (ib + 32) + 1];
        if (a2) sim[ia + 32][ib] = s10 * inv_norm[2 * (ia + 32)] * nb0;
        if (a2 && b2) sim[ia + 32][ib + 32] = s11 * inv_norm[2 * (ia + 32)] * inv_norm[2 * (ib + 32) + 1];
    }
    __syncthreads();
    // per A token: the best B, ties to the lower position (a warp per A token, lanes over B)
    for (int ia = warp; ia < n_a; ia += kW) {
        float bs = -INFINITY;
        int bb = -1;
        for (int ib = lane; ib < n_b; ib += 32) {
            const float s = sim[ia][ib];
            if (bb < 0 || s > bs) {
                bs = s;
                bb = ib;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float os = __shfl_xor_sync(0xffffffffu, bs, off);
            const int ob = __shfl_xor_sync(0xffffffffu, bb, off);
            if (ob >= 0 && (bb < 0 || os > bs || (os == bs && ob < bb))) {
                bs = os;
                bb = ob;
            }
        }
        if (lane == 0) {
            sr[ia] = bb >= 0 ? bs : -INFINITY;
            br[c0 + 2 * ia] = bb >= 0 ? c0 + 2 * bb + 1 : -1;
        }
    }
}

// ------------------------------------------------------------------------ match, bf16 keys

struct TcMatchArgs {
    CUtensorMap tmap;  // K as [rows][N][128] bf16, box 64 x 128 x 1, 128-byte swizzle
    float* score;
    int32_t* best;
    unsigned* err;
    int N, S, w, chunk;
    int tt;             // tokens per tile: a whole number of chunks, <= 128
    int tiles_per_row;  // ceil(|C| / tt)
    int total_tiles;
    int n_a_row;        // A tokens per row: score row length
};

struct __align__(1024) MatchSmem {
    uint8_t ring[kTcStages][2][kHalfBytes];  // a tile = two 64-dimension halves
    float inv[kTcAcc][2][kTileTok];          // per warpgroup: 1/|k| of the tile's tokens, double-buffered
    uint64_t full[kTcStages], empty[kTcStages], accfull[kTcAcc], accempty[kTcAcc];
    uint32_t tmem_base;
    int abort;
};

// Bounded wait that ignores the abort flag: used at teardown for operations already issued.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, unsigned* err) {
    const long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kBarrierTimeoutNs) {
            atomicOr(err, kErrTimeout);
            return;
        }
    }
}

// Persistent: CTA c takes the global tiles c, c + P, ...  (row-major over (row, tile)).
// Tile (u, tau) covers tokens t0 = S + tau * tt .. t0 + 127 of row u (tokens past the tile's
// chunks are loaded and ignored; past N they read as 0).  D[r][j] = k_{t0+r} . k_{t0+j}.
// Writes score[u][i] for the row's A tokens S + 2i and best[u][pos] at A positions.
__global__ void __launch_bounds__(kTcThreads, 1) csm_match_tc_kernel(const __grid_constant__ TcMatchArgs a) {
    extern __shared__ uint8_t smem_raw[];
    MatchSmem& sm = *reinterpret_cast<MatchSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x, P = gridDim.x;
    const int n_local = cta < a.total_tiles ? (a.total_tiles - cta + P - 1) / P : 0;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < kTcAcc; ++i) {
            mbar_init(&sm.accfull[i], 1);
            mbar_init(&sm.accempty[i], 4);
        }
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kTcCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap)) : "memory");
            int issued = 0;
            for (int i = 0; i < n_local && !*abort; ++i) {
                const int g = cta + i * P;
                const int u = g / a.tiles_per_row, tau = g - u * a.tiles_per_row;
                const int s = i % kTcStages;
                // the tile starts inside the row's candidates and holds whole chunks
                if (!dcheck(a.err, tau >= 0 && a.S + tau * a.tt < a.N - a.w && a.tt <= kTileTok &&
                                       a.tt % a.chunk == 0)) {
                    *abort = 1;
                    break;
                }
                mbar_wait(&sm.empty[s], ((i / kTcStages) & 1) ^ 1, abort, a.err);
                if (*abort) break;
                mbar_expect_tx(&sm.full[s], 2 * kHalfBytes);
                tma_load_3d(sm.ring[s][0], &a.tmap, &sm.full[s], 0, a.S + tau * a.tt, u);
                tma_load_3d(sm.ring[s][1], &a.tmap, &sm.full[s], 64, a.S + tau * a.tt, u);
                issued = i + 1;
            }
            // every copy this CTA issued has landed before the CTA exits
            for (int i = max(0, issued - kTcStages); i < issued; ++i)
                mbar_drain(&sm.full[i % kTcStages], (i / kTcStages) & 1, a.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int last = -1;
            for (int i = 0; i < n_local && !*abort; ++i) {
                const int s = i % kTcStages, acc = i % kTcAcc;
                mbar_wait(&sm.full[s], (i / kTcStages) & 1, abort, a.err);
                mbar_wait(&sm.accempty[acc], ((i / kTcAcc) & 1) ^ 1, abort, a.err);
                if (*abort) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * kTileTok;
                const uint64_t h0 = sw128_desc(smem_u32(sm.ring[s][0])), h1 = sw128_desc(smem_u32(sm.ring[s][1]));
                umma_half(d, h0, h0, 0);
                umma_half(d, h1, h1, 1);
                umma_commit(&sm.empty[s]);
                umma_commit(&sm.accfull[acc]);
                last = i;
            }
            // the last products have completed before TMEM is released
            if (last >= 0) mbar_drain(&sm.accfull[last % kTcAcc], (last / kTcAcc) & 1, a.err);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warpgroup g (warps 2 + 4g .. 5 + 4g) takes the tiles i = g, g + 4, ... from
        // accumulator g.  Thread r = TMEM lane = the tile's token r.  Every warp of a group
        // runs every one of its iterations (the waits return at once after an abort), so
        // the group's named barrier always sees all four warps.
        const int grp = (warp - 2) >> 2, qd = warp & 3;
        const int r = 32 * qd + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * qd) << 16) + grp * kTileTok;
        for (int i = grp, it = 0; i < n_local; i += kTcAcc, ++it) {
            const int g = cta + i * P;
            const int u = g / a.tiles_per_row, tau = g - u * a.tiles_per_row;
            const int t0 = a.S + tau * a.tt;
            const int valid = min(a.tt, a.N - a.w - t0);
            mbar_wait(&sm.accfull[grp], it & 1, abort, a.err);
            tc_fence_after();
            uint32_t x[32], y[32];
            // the diagonal: this thread's column r sits in column block qd, register `lane`
            // (a select tree over the lane's bits)
            tmem_ld32(lane_base + 32 * qd, x);
            tmem_wait32(x);
            float v16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v16[e] = __uint_as_float((lane & 1) ? x[2 * e + 1] : x[2 * e]);
#pragma unroll
            for (int lv = 1; lv < 5; ++lv) {
#pragma unroll
                for (int e = 0; e < (16 >> lv); ++e) v16[e] = ((lane >> lv) & 1) ? v16[2 * e + 1] : v16[2 * e];
            }
            const float gd = v16[0];
            float* inv = sm.inv[grp][it & 1];
            inv[r] = gd > 0.f ? rsqrtf(gd) : 0.f;
            asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory");
            // A tokens (even offsets of a chunk): argmax over the chunk's B columns (odd
            // offsets; chunk starts are even), ascending so that ties keep the lower column.
            // Column blocks come in pairs with one comparison chain each.
            const int cs = (r / a.chunk) * a.chunk, ce = min(cs + a.chunk, valid);
            const bool is_a = r < valid && ((r - cs) & 1) == 0;
            const float ir = inv[r];
            float bs = -INFINITY;
            int bb = -1;
            const int r_lo = 32 * qd, r_hi = min(32 * qd + 31, valid - 1);
            if (r_lo <= r_hi) {
                const int cb_lo = ((r_lo / a.chunk) * a.chunk) >> 5;
                const int cb_hi = (min((r_hi / a.chunk) * a.chunk + a.chunk, valid) + 31) >> 5;  // exclusive
                for (int cb = cb_lo; cb < cb_hi; cb += 2) {
                    const bool two = cb + 1 < cb_hi;
                    tmem_ld32(lane_base + 32 * cb, x);
                    if (two) tmem_ld32(lane_base + 32 * (cb + 1), y);
                    tmem_wait32(x);
                    if (two) tmem_wait32(y);
                    float s0 = -INFINITY, s1 = -INFINITY;
                    int b0 = -1, b1 = -1;
#pragma unroll
                    for (int e = 1; e < 32; e += 2) {
                        const int j0 = 32 * cb + e, j1 = j0 + 32;
                        const float v0 = __uint_as_float(x[e]) * ir * inv[j0];
                        const float v1 = __uint_as_float(y[e]) * ir * inv[two ? j1 : j0];
                        if (j0 > cs && j0 < ce && (b0 < 0 || v0 > s0)) {
                            s0 = v0;
                            b0 = j0;
                        }
                        if (two && j1 > cs && j1 < ce && (b1 < 0 || v1 > s1)) {
                            s1 = v1;
                            b1 = j1;
                        }
                    }
                    // merge: the earlier (lower) columns win ties
                    if (b1 >= 0 && (b0 < 0 || s1 > s0)) {
                        s0 = s1;
                        b0 = b1;
                    }
                    if (b0 >= 0 && (bb < 0 || s0 > bs)) {
                        bs = s0;
                        bb = b0;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.accempty[grp]);
            if (is_a && dcheck(a.err, (t0 + r - a.S) / 2 < a.n_a_row && t0 + r < a.N - a.w)) {
                // A token (t0 + r - S) / 2 of the row (tiles start at even offsets)
                a.score[(size_t)u * a.n_a_row + (t0 + r - a.S) / 2] = bb >= 0 ? bs : -INFINITY;
                a.best[(size_t)u * a.N + t0 + r] = bb >= 0 ? t0 + bb : -1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols) : "memory");
    }
}

// ------------------------------------------------------------------------ selection bookkeeping

// merged[pos] = 1 for the selected A tokens (sel holds A indices i, position S + 2i);
// cb[row][c] counts the merges of chunk c.
__global__ void csm_mark_kernel(const int32_t* __restrict__ sel, int rows, int N, int S, int w, int chunk, int m,
                                int n_chunks, unsigned char* __restrict__ merged, int32_t* __restrict__ cb,
                                unsigned* __restrict__ err) {
    const long long total = (long long)rows * m;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long row = e / m;
        const int p = S + 2 * sel[e];  // A token sel[e] of the row
        if (sel[e] < 0 || p >= N - w) {  // never for a well-formed selection
            atomicOr(err, kErrIndex);
            continue;
        }
        if (!dcheck(err, (p - S) / chunk < n_chunks)) continue;  // the owner chunk of token p
        merged[row * N + p] = 1;
        atomicAdd(&cb[row * (n_chunks + 1) + (p - S) / chunk], 1);
    }
}

// Per row, in place: cb[c] (merges of chunk c) becomes the number of kept tokens before
// chunk c (sinks included); cb[n_chunks] becomes the number before the window.  Each thread
// owns a contiguous run of chunks.
__global__ void __launch_bounds__(kScanThreads)
csm_base_kernel(int N, int S, int w, int chunk, int n_chunks, int m, int32_t* __restrict__ cb, unsigned* err) {
    __shared__ int warp_tot[kScanThreads / 32];
    int32_t* c = cb + (size_t)blockIdx.x * (n_chunks + 1);
    const int per = (n_chunks + kScanThreads - 1) / kScanThreads;
    const int q0 = min(n_chunks, (int)threadIdx.x * per), q1 = min(n_chunks, q0 + per);
    const int hi = N - w;
    int cnt = 0;
    for (int q = q0; q < q1; ++q) cnt += min(chunk, hi - (S + q * chunk)) - c[q];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int o = S + incl - cnt;
    for (int i = 0; i < warp; ++i) o += warp_tot[i];
    for (int q = q0; q < q1; ++q) {
        const int kept = min(chunk, hi - (S + q * chunk)) - c[q];
        c[q] = o;
        o += kept;
    }
    if (threadIdx.x == kScanThreads - 1) {
        c[n_chunks] = o;  // the last thread ends at the total
        dcheck(err, o == N - w - m);  // exactly m tokens of the row were marked merged
    }
}

// ------------------------------------------------------------------------ write

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"((uint64_t)__cvta_generic_to_global(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"((uint64_t)__cvta_generic_to_global(dst)), "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}

// blockIdx.x = row * n_blk + b: b < n_chunks is chunk b, then ceil(S / 128) sink segments,
// then ceil(w / 128) window segments.  A block's K and V rows are contiguous in HBM: two
// bulk copies bring them into shared memory while the merge flags load; merged means are
// formed in place (a warp per B token: lanes 0-15 its K row, 16-31 its V row, 8 elements
// each); every run of consecutive kept rows then leaves with one bulk store per tensor
// (consecutive kept rows have consecutive output slots).
template <typename T>
__global__ void __launch_bounds__(kWriteThreads)
csm_write_kernel(const T* __restrict__ k, const T* __restrict__ v, const int32_t* __restrict__ deg,
                 const int32_t* __restrict__ pos, int N, long long ld_in, int S, int w, int chunk, int n_chunks,
                 int n_blk, const int32_t* __restrict__ best, const unsigned char* __restrict__ merged,
                 const int32_t* __restrict__ cb, int n_out, long long ld_out, T* __restrict__ k_out,
                 T* __restrict__ v_out, int32_t* __restrict__ deg_out, int32_t* __restrict__ pos_out,
                 unsigned* __restrict__ err) {
    constexpr int V = Vec<T>::n;
    extern __shared__ __align__(128) uint8_t wsm[];  // K rows, then V rows, of this block
    __shared__ uint64_t bar;
    __shared__ int failed;
    __shared__ unsigned char mg[128];
    __shared__ int32_t dg[128], ns[128];
    __shared__ uint32_t amask[64][2];  // per B token (offset / 2): its merged A tokens (offset / 2)
    __shared__ uint32_t mword[4];      // merged flags, 32 tokens per word
    const int row = blockIdx.x / n_blk, b = blockIdx.x - row * n_blk;
    const int hi = N - w;
    const int n_sblk = (S + kSeg - 1) / kSeg;
    int p0, n, o0;
    bool in_c = false;
    if (b < n_chunks) {
        p0 = S + b * chunk;
        n = min(chunk, hi - p0);
        o0 = cb[(size_t)row * (n_chunks + 1) + b];
        in_c = true;
    } else if (b < n_chunks + n_sblk) {
        p0 = (b - n_chunks) * kSeg;
        n = min(kSeg, S - p0);
        o0 = p0;
    } else {
        const int off = (b - n_chunks - n_sblk) * kSeg;
        p0 = hi + off;
        n = min(kSeg, w - off);
        o0 = cb[(size_t)row * (n_chunks + 1) + n_chunks] + off;
    }
    const size_t rN = (size_t)row * N;     // workspace rows (dense)
    const size_t rI = (size_t)row * ld_in;  // input cache rows
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t tensor_bytes = (uint32_t)n * D * sizeof(T);
    T* sk = reinterpret_cast<T*>(wsm);
    T* sv = sk + (size_t)n * D;

    // the block is a non-empty slice of the row that fits the shared arrays, and its first
    // output slot lies inside the output row (the slots it writes are checked one by one)
    if (!dcheck(err, n >= 1 && n <= 128 && p0 >= 0 && p0 + n <= N && o0 >= 0 && o0 < n_out)) return;
    if (tid == 0) {
        failed = 0;
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_expect_tx(&bar, 2 * tensor_bytes);
        bulk_load(sk, k + (rI + p0) * D, tensor_bytes, &bar);
        bulk_load(sv, v + (rI + p0) * D, tensor_bytes, &bar);
    }
    amask[tid >> 1][tid & 1] = 0u;
    if (tid < n) {
        mg[tid] = in_c ? merged[rN + p0 + tid] : 0;
        dg[tid] = deg ? deg[rI + p0 + tid] : 1;
    }
    __syncthreads();
    {
        const bool m = tid < n && mg[tid];
        const unsigned bits = __ballot_sync(0xffffffffu, m);
        if (lane == 0) mword[warp] = bits;
        if (m) {
            const int ob = best[rN + p0 + tid] - p0;  // the B token's offset in the chunk
            if (ob >= 1 && ob < n && (ob & 1) && !(tid & 1))
                atomicOr(&amask[ob >> 1][tid >> 6], 1u << ((tid >> 1) & 31));
            else
                atomicOr(err, kErrIndex);  // never for a well-formed match
        }
    }
    __syncthreads();
    // output slot of a kept token t: o0 + t - (merged tokens before t)
    auto slot_of = [&](int t) {
        int before = __popc(mword[t >> 5] & ((1u << (t & 31)) - 1u));
        for (int i = 0; i < (t >> 5); ++i) before += __popc(mword[i]);
        return o0 + t - before;
    };
    if (tid < n && !mg[tid]) {
        int nsum = dg[tid];
        if (tid & 1) {
#pragma unroll
            for (int wd = 0; wd < 2; ++wd)
                for (uint32_t mm = amask[tid >> 1][wd]; mm; mm &= mm - 1u) nsum += dg[2 * (32 * wd + __ffs(mm) - 1)];
        }
        ns[tid] = nsum;
        const int so = slot_of(tid);
        const size_t o = (size_t)row * ld_out + so;
        if (dcheck(err, so >= o0 && so < n_out)) deg_out[o] = nsum;
        if (dcheck(err, so >= o0 && so < n_out)) pos_out[o] = pos ? pos[rI + p0 + tid] : p0 + tid;
    }
    // the rows have landed (bounded wait; a copy that never lands is reported, not used)
    if (!mbar_try_wait(&bar, 0)) {
        const long long t0 = globaltimer();
        while (!mbar_try_wait(&bar, 0)) {
            if (globaltimer() - t0 > kBarrierTimeoutNs) {
                atomicOr(err, kErrTimeout);
                failed = 1;
                break;
            }
        }
    }
    __syncthreads();
    if (failed) return;
    // merged means in place: the B row first, then its A rows by position, in fp32
    for (int t = 2 * warp + 1; t < n; t += 2 * (kWriteThreads / 32)) {
        const uint32_t m0 = amask[t >> 1][0], m1 = amask[t >> 1][1];
        if (!(m0 | m1)) continue;
        T* base = (lane < 16 ? sk : sv) + 8 * (lane & 15);
        uint4 r[V];
        float acc[8], x[8];
#pragma unroll
        for (int j = 0; j < V; ++j) r[j] = reinterpret_cast<const uint4*>(base + (size_t)t * D)[j];
        to_f8(r, x);
        const float db = (float)dg[t];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = db * x[e];
#pragma unroll
        for (int wd = 0; wd < 2; ++wd) {
            for (uint32_t mm = wd ? m1 : m0; mm; mm &= mm - 1u) {
                const int ta = 2 * (32 * wd + __ffs(mm) - 1);
#pragma unroll
                for (int j = 0; j < V; ++j) r[j] = reinterpret_cast<const uint4*>(base + (size_t)ta * D)[j];
                to_f8(r, x);
                const float da = (float)dg[ta];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(da, x[e], acc[e]);
            }
        }
        const float inv = 1.f / (float)ns[t];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= inv;
        from_f8(acc, r);
#pragma unroll
        for (int j = 0; j < V; ++j) reinterpret_cast<uint4*>(base + (size_t)t * D)[j] = r[j];
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    // one bulk store per tensor for each run of kept rows, issued by the thread of its first row
    if (tid < n && !mg[tid] && (tid == 0 || mg[tid - 1])) {
        int e = n;
        for (int wd = (tid + 1) >> 5; wd < 4; ++wd) {
            uint32_t mm = mword[wd];
            if (wd == ((tid + 1) >> 5)) mm &= ~0u << ((tid + 1) & 31);
            if (mm) {
                e = min(n, 32 * wd + __ffs(mm) - 1);
                break;
            }
        }
        const int so = slot_of(tid);
        const size_t o = (size_t)row * ld_out + so;
        const uint32_t bytes = (uint32_t)(e - tid) * D * sizeof(T);
        // the run's rows land inside the output row
        if (dcheck(err, so >= o0 && so + (e - tid) <= n_out)) {
            bulk_store(k_out + o * D, sk + (size_t)tid * D, bytes);
            bulk_store(v_out + o * D, sv + (size_t)tid * D, bytes);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // shared memory stays valid until the stores have read it
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    }
}

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

int csm_merges(int N, int S, int w, int chunk, float ratio) {
    const int n_c = N - w - S;
    int n_a = 0;
    for (int c0 = 0; c0 < n_c; c0 += chunk) {
        const int len = c0 + chunk < n_c ? chunk : n_c - c0;
        if (len >= 2) n_a += (len + 1) / 2;
    }
    const long long m = (long long)floor((double)ratio * (double)n_c);
    return (int)(m < n_a ? m : n_a);
}

size_t csm_workspace(int rows, int N, int m) {
    const size_t rn = (size_t)rows * N;
    return a256(rn * sizeof(float)) + a256(rn * sizeof(int32_t)) + a256((size_t)rows * (N + 1) * sizeof(int32_t)) +
           a256(rn) + a256((size_t)rows * (m > 0 ? m : 1) * sizeof(int32_t));
}

namespace {

cudaError_t match_tc(const void* k, int rows, int N, long long ld, int S, int w, int chunk, float* score,
                     int32_t* best, cudaStream_t s) {
    TcMatchArgs a{};
    a.score = score;
    a.best = best;
    a.err = device_error_word();
    a.N = N;
    a.S = S;
    a.w = w;
    a.chunk = chunk;
    a.tt = (kTileTok / chunk) * chunk;
    a.tiles_per_row = (N - w - S + a.tt - 1) / a.tt;
    a.n_a_row = (N - w - S + 1) / 2;
    const long long total = (long long)rows * a.tiles_per_row;
    if (total > (1LL << 31) - 1) return cudaErrorInvalidValue;
    a.total_tiles = (int)total;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)ld * D * 2};
    cuuint32_t box[3] = {64, kTileTok, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&a.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int n_sm = sm_count();
    if (n_sm <= 0) return cudaErrorNoDevice;
    const int P = std::min(std::min(n_sm, kTcMaxCtas), a.total_tiles);
    const size_t smem = sizeof(MatchSmem) + 1024;
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev >= 64 || !attr_set[dev].load()) {
        if ((e = cudaFuncSetAttribute(csm_match_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        if (dev < 64) attr_set[dev].store(true);
    }
    csm_match_tc_kernel<<<P, kTcThreads, smem, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t match_f32(const float* k, int rows, int N, long long ld, int S, int w, int chunk, int n_chunks,
                      int n_a_row, float* score, int32_t* best, cudaStream_t s) {
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev >= 64 || !attr_set[dev].load()) {
        if ((e = cudaFuncSetAttribute(csm_match_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      128 * kKS * 4)) != cudaSuccess)
            return e;
        if (dev < 64) attr_set[dev].store(true);
    }
    const long long grid = (long long)rows * n_chunks;
    if (grid > (1LL << 31) - 1) return cudaErrorInvalidValue;
    csm_match_f32_kernel<<<(unsigned)grid, kMatchThreads, (size_t)chunk * kKS * sizeof(float), s>>>(
        k, N, ld, S, w, chunk, n_chunks, n_a_row, score, best, device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t csm(const void* k, const void* v, int dtype, const int32_t* deg, const int32_t* pos, int rows, int N,
                long long ld_in, int S, int w, int chunk, int m, void* k_out, void* v_out, int32_t* deg_out,
                int32_t* pos_out, long long ld_out, void* ws, cudaStream_t s) {
    const size_t rn = (size_t)rows * N;
    char* p = (char*)ws;
    float* score = (float*)p;
    p += a256(rn * sizeof(float));
    int32_t* best = (int32_t*)p;
    p += a256(rn * sizeof(int32_t));
    int32_t* cb = (int32_t*)p;  // [rows][n_chunks + 1] (n_chunks <= N)
    p += a256((size_t)rows * (N + 1) * sizeof(int32_t));
    unsigned char* merged = (unsigned char*)p;
    p += a256(rn);
    int32_t* sel = (int32_t*)p;
    unsigned* err = device_error_word();
    const int n_out = N - m;
    const int hi = N - w;
    const int n_chunks = (hi - S + chunk - 1) / chunk;
    cudaError_t e;

    if ((e = cudaMemsetAsync(merged, 0, rn, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(cb, 0, (size_t)rows * (n_chunks + 1) * sizeof(int32_t), s)) != cudaSuccess) return e;
    if (m > 0 && n_chunks > 0) {
        const int n_a_row = (hi - S + 1) / 2;  // A tokens S, S + 2, ... of C
        e = dtype == KVC_BF16
                ? match_tc(k, rows, N, ld_in, S, w, chunk, score, best, s)
                : match_f32((const float*)k, rows, N, ld_in, S, w, chunk, n_chunks, n_a_row, score, best, s);
        if (e != cudaSuccess) return e;
        // the m best matches over the row of A scores (ties to the lower position), ascending
        e = topk_fused_fits(n_a_row, 0, 0) ? topk_fused(score, rows, n_a_row, 0, 0, m, 1, sel, s)
                                           : topk(score, rows, n_a_row, 0, 0, m, sel, s);
        if (e != cudaSuccess) return e;
        const long long total = (long long)rows * m;
        csm_mark_kernel<<<(int)std::min<long long>((total + 255) / 256, 148LL * 8), 256, 0, s>>>(
            sel, rows, N, S, w, chunk, m, n_chunks, merged, cb, err);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    csm_base_kernel<<<rows, kScanThreads, 0, s>>>(N, S, w, chunk, n_chunks, m, cb, err);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int n_blk = n_chunks + (S + kSeg - 1) / kSeg + (w + kSeg - 1) / kSeg;
    const long long grid = (long long)rows * n_blk;
    if (grid > (1LL << 31) - 1) return cudaErrorInvalidValue;
    // rows of the longest block (a chunk, or a sink / window segment), K and V
    const int max_rows = std::max(n_chunks > 0 ? chunk : 0, std::max(std::min(S, kSeg), std::min(w, kSeg)));
    const size_t esz = dtype == KVC_BF16 ? 2 : 4;
    const size_t smem = 2 * (size_t)max_rows * D * esz;
    static std::atomic<bool> attr_set[2][64];
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    const int ti = dtype == KVC_BF16;
    if (dev >= 64 || !attr_set[ti][dev].load()) {
        const int lim = 2 * kSeg * D * 4;
        e = ti ? cudaFuncSetAttribute(csm_write_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim)
               : cudaFuncSetAttribute(csm_write_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[ti][dev].store(true);
    }
    if (dtype == KVC_BF16)
        csm_write_kernel<__nv_bfloat16><<<(unsigned)grid, kWriteThreads, smem, s>>>(
            (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, deg, pos, N, ld_in, S, w, chunk, n_chunks, n_blk, best,
            merged, cb, n_out, ld_out, (__nv_bfloat16*)k_out, (__nv_bfloat16*)v_out, deg_out, pos_out, err);
    else
        csm_write_kernel<float><<<(unsigned)grid, kWriteThreads, smem, s>>>(
            (const float*)k, (const float*)v, deg, pos, N, ld_in, S, w, chunk, n_chunks, n_blk, best, merged, cb,
            n_out, ld_out, (float*)k_out, (float*)v_out, deg_out, pos_out, err);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvc

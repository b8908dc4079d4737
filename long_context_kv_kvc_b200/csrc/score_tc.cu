// score_tc.cu -- window-softmax saliency scores on the 5th-generation tensor cores.
//
// What it computes (per unit = one (layer, batch, KV head)): for the unit's G*w window
// query rows r (query i of head g sits at position N - w + i and sees keys j <= N - w + i)
//     lse_r = log2 sum_j 2^(y_rj),   y_rj = (q_r . k_j) * log2(e) / sqrt(D)
//     s_j   = sum_r 2^(y_rj - lse_r)                 (visible pairs only)
// i.e. the softmaxed attention of the observation window summed over the window queries
// and the GQA group (FastKV page, sec. 2A: tokens are selected by a saliency score; the
// SnapKV eviction it names scores with the window's attention; StructKV page, sec. 1: the
// same attention scores are summed over layers).
//
// Design for B200.  The softmax normaliser lse_r is global over all N keys, so every
// logit is needed twice: once for lse_r (phase 1) and once for its probability (phase 2).
// Storing logits would cost more HBM traffic than K itself, so K tiles are read twice and
// the schedule makes the second read hit L2:
//   * one persistent CTA per SM (cooperative launch, so all CTAs are resident), 128-key
//     tiles dealt round-robin over the CTAs in global order (unit-major);
//   * each CTA runs phase 1 on its tile i while running phase 2 on its tile i - lag, with
//     lag about one unit's worth of tiles, so the tile is re-read from L2 (~1 unit of K,
//     32 MiB at 128K, is in flight across the GPU);
//   * phase 1:  D1[128 q x 128 keys] = Q K^T (tcgen05.mma kind::f16, M = N = 128, fp32
//     accumulator in TMEM); one thread per query row keeps an online (max, sum) over the
//     CTA's tiles of the unit; the CTA's partial goes to global memory and the last CTA
//     of the unit (atomic counter) merges the partials in a fixed order into lse and
//     raises the unit's ready flag;
//   * phase 2:  D2[128 keys x 128 q] = K Q^T (the transposed product, so a thread owns a
//     key and sums over queries in registers); waits (bounded) for the unit's ready flag.
// Warp roles: warp 0 issues TMA loads (K tiles through a 4-stage ring, Q of the current
// unit for each phase), warp 1 owns TMEM and issues the MMAs from one thread, warps 4-7
// run phase-1 statistics, warps 8-11 run phase-2 sums.  TMEM holds two phase-1 and two
// phase-2 accumulators (4 x 128 columns).  Every wait is bounded: a wait that runs out
// sets the per-device error word and the kernel finishes without blocking.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr int kTileKeys = 128;                         // keys per tile (MMA N / M)
constexpr int kQRows = 128;                            // query rows per unit (padded)
constexpr int kStages = 4;                             // K-tile ring depth
constexpr int kTileBytes = kTileKeys * kHeadDim * 2;   // 32 KiB of bf16
constexpr int kHalfBytes = kTileBytes / 2;             // one 64-column (128-byte) TMA box
constexpr int kThreads = 384;
constexpr int kMaxCtas = 160;                          // partial slots per row (>= #SMs)
constexpr uint32_t kTmemCols = 512;
constexpr long long kBarrierTimeoutNs = 4000000000LL;  // hang guard for intra-CTA waits

// tcgen05 instruction descriptor, kind::f16: fp32 accumulate (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), both K-major, N = 128 (bits 17-22 = N/8), M = 128 (bits 24-28 = M/16)
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct TcArgs {
    CUtensorMap tmap_k;  // K as [U][N][128] bf16, box 64 x 128 x 1, 128-byte swizzle
    CUtensorMap tmap_q;  // padded Q as [U*128][128] bf16, box 64 x 128, 128-byte swizzle
    float* unit_scores;  // [U][N]
    float2* partial;     // [U][128][kMaxCtas] (max, sum) per CTA
    float* lse;          // [U][128]
    unsigned* count;     // [U] CTAs that have published their partial
    unsigned* ready;     // [U] lse published
    unsigned* never;     // a flag nothing sets (wait-timeout injection)
    unsigned* err;
    long long spin_limit;
    int U, N, w, nq, T_u, total_tiles, P, lag, inject;
};

struct __align__(1024) Smem {
    uint8_t ktile[kStages][kTileBytes];
    uint8_t q[2][kTileBytes];
    float lse[kQRows];
    uint64_t full[kStages], empty[kStages];
    uint64_t qfull[2], qempty[2];
    uint64_t d1full[2], d1empty[2], d2full[2], d2empty[2];
    uint32_t tmem_base;
    int abort;
    int flag1, flag2;
};

// ------------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ long long globaltimer() {
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity.  On time-out (a broken
// pipeline, never a normal run) it records the error, puts the CTA in fail-fast mode and
// returns, so that the kernel always terminates.
__device__ __forceinline__ void mbar_wait(uint64_t* bar, uint32_t parity, Smem& sm, unsigned* err) {
    if (mbar_try_wait(bar, parity)) return;
    const long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (*(volatile int*)&sm.abort) return;
        if (globaltimer() - t0 > kBarrierTimeoutNs) {
            atomicOr(err, kErrTimeout);
            *(volatile int*)&sm.abort = 1;
            return;
        }
    }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand in the 128-byte swizzled layout
// that TMA writes: rows of 128 bytes, 8-row (1024-byte) swizzle atoms stacked along M/N.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
    d |= (uint64_t)1u << 16;                          // leading-dimension offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride between 8-row atoms
    d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                          // 128-byte swizzle
    return d;
}

// Descriptor of K-slice kk (16 columns = 32 bytes) of a 128 x 128 bf16 tile stored as two
// 64-column boxes.
__device__ __forceinline__ uint64_t tile_desc(const uint8_t* tile, int kk) {
    return sw128_desc(smem_u32(tile) + (kk >> 2) * kHalfBytes + (kk & 3) * 32);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane; the values are only valid after
// tmem_wait, which takes them as in/out operands so no use can be scheduled before it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Order of jobs of one CTA: phase 1 runs `lag` tiles ahead of phase 2.
struct JobIter {
    int n, lag, i1 = 0, i2 = 0;
    __device__ JobIter(int n_, int lag_) : n(n_), lag(lag_) {}
    __device__ bool next(int& phase, int& i) {
        if (i1 < n && i1 - i2 < lag) {
            phase = 0;
            i = i1++;
            return true;
        }
        if (i2 < n) {
            phase = 1;
            i = i2++;
            return true;
        }
        return false;
    }
};

// ------------------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kThreads, 1) tc_score_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x, P = a.P;
    const int n_local = cta < a.total_tiles ? (a.total_tiles - cta + P - 1) / P : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.qfull[b], 1);
            mbar_init(&sm.qempty[b], 1);
            mbar_init(&sm.d1full[b], 1);
            mbar_init(&sm.d1empty[b], 4);
            mbar_init(&sm.d2full[b], 1);
            mbar_init(&sm.d2empty[b], 4);
        }
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_q)) : "memory");
            JobIter it(n_local, a.lag);
            int ph, i, k = 0;
            int qunit[2] = {-1, -1}, qloads[2] = {0, 0};
            while (it.next(ph, i)) {
                const int t = cta + i * P, u = t / a.T_u, ti = t - u * a.T_u;
                if (u != qunit[ph]) {
                    if (qloads[ph] > 0) mbar_wait(&sm.qempty[ph], (qloads[ph] - 1) & 1, sm, a.err);
                    mbar_expect_tx(&sm.qfull[ph], kTileBytes);
                    tma_load_2d(sm.q[ph], &a.tmap_q, &sm.qfull[ph], 0, u * kQRows);
                    tma_load_2d(sm.q[ph] + kHalfBytes, &a.tmap_q, &sm.qfull[ph], 64, u * kQRows);
                    qunit[ph] = u;
                    ++qloads[ph];
                }
                const int s = k % kStages;
                mbar_wait(&sm.empty[s], ((k / kStages) & 1) ^ 1, sm, a.err);
                mbar_expect_tx(&sm.full[s], kTileBytes);
                tma_load_3d(sm.ktile[s], &a.tmap_k, &sm.full[s], 0, ti * kTileKeys, u);
                tma_load_3d(sm.ktile[s] + kHalfBytes, &a.tmap_k, &sm.full[s], 64, ti * kTileKeys, u);
                ++k;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            JobIter it(n_local, a.lag);
            int ph, i, k = 0, n1 = 0, n2 = 0;
            int qunit[2] = {-1, -1}, qloads[2] = {0, 0};
            while (it.next(ph, i)) {
                const int t = cta + i * P, u = t / a.T_u;
                if (u != qunit[ph]) {
                    // the previous Q of this phase is free once every MMA issued so far is done
                    if (qunit[ph] >= 0) umma_commit(&sm.qempty[ph]);
                    mbar_wait(&sm.qfull[ph], qloads[ph] & 1, sm, a.err);
                    qunit[ph] = u;
                    ++qloads[ph];
                }
                const int s = k % kStages;
                mbar_wait(&sm.full[s], (k / kStages) & 1, sm, a.err);
                uint32_t d;
                const uint8_t *A, *B;
                uint64_t* done;
                if (ph == 0) {
                    const int b = n1 & 1;
                    mbar_wait(&sm.d1empty[b], ((n1 >> 1) & 1) ^ 1, sm, a.err);
                    d = tmem + b * 128;
                    A = sm.q[0];
                    B = sm.ktile[s];
                    done = &sm.d1full[b];
                    ++n1;
                } else {
                    const int b = n2 & 1;
                    mbar_wait(&sm.d2empty[b], ((n2 >> 1) & 1) ^ 1, sm, a.err);
                    d = tmem + 256 + b * 128;
                    A = sm.ktile[s];
                    B = sm.q[1];
                    done = &sm.d2full[b];
                    ++n2;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) umma_bf16(d, tile_desc(A, kk), tile_desc(B, kk), kk > 0);
                umma_commit(&sm.empty[s]);
                umma_commit(done);
                ++k;
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ phase 1: statistics
        const int r = threadIdx.x - 128;  // query row == TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const int t_r = a.N - a.w + (r % a.w);  // last key this row sees
        int cur = -1;
        float m = -INFINITY, l = 0.f;
        for (int i = 0; i <= n_local; ++i) {
            const int t = cta + i * P;
            const int u = i < n_local ? t / a.T_u : -2;
            if (u != cur && cur >= 0) {
                // publish this CTA's (max, sum) of unit `cur`; the last CTA merges them
                a.partial[((size_t)cur * kQRows + r) * kMaxCtas + cta] = make_float2(m, l);
                named_sync(1, 128);
                if (r == 0) {
                    __threadfence();
                    const int n_contrib = min(a.T_u, P);
                    const unsigned old = atomicAdd(&a.count[cur], 1u);
                    sm.flag1 = (old == (unsigned)(n_contrib - 1));
                }
                named_sync(1, 128);
                if (sm.flag1) {
                    __threadfence();
                    const int n_contrib = min(a.T_u, P);
                    const float2* pr = a.partial + ((size_t)cur * kQRows + r) * kMaxCtas;
                    float M = -INFINITY;
                    for (int c = 0; c < n_contrib; ++c) M = fmaxf(M, __ldcg(pr + (cur * a.T_u + c) % P).x);
                    float S = 0.f;
                    for (int c = 0; c < n_contrib; ++c) {
                        const float2 v = __ldcg(pr + (cur * a.T_u + c) % P);
                        if (v.x != -INFINITY) S += v.y * exp2f(v.x - M);
                    }
                    a.lse[(size_t)cur * kQRows + r] = M + log2f(S);
                    __threadfence();
                    named_sync(1, 128);
                    if (r == 0) atomicExch(&a.ready[cur], 1u);
                }
            }
            if (i == n_local) break;
            if (u != cur) {
                cur = u;
                m = -INFINITY;
                l = 0.f;
            }
            const int ti = t - u * a.T_u;
            const int b = i & 1;
            mbar_wait(&sm.d1full[b], (i >> 1) & 1, sm, a.err);
            tc_fence_after();
            const bool full_tile = (ti + 1) * kTileKeys <= a.N - a.w + 1;
            const int j0 = ti * kTileKeys;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t x[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + b * 128 + c * 32, x);
                tmem_wait(x);
                if (c == 3) {
                    // the accumulator is free for the next MMA once all four chunks are loaded
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.d1empty[b]);
                }
                float cm = -INFINITY;
                if (full_tile) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) cm = fmaxf(cm, __uint_as_float(x[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0 + c * 32 + e <= t_r) cm = fmaxf(cm, __uint_as_float(x[e]));
                }
                if (cm != -INFINITY) {
                    const float mn = fmaxf(m, cm * kLog2eOverSqrtD);
                    float sum = 0.f;
                    if (full_tile) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) sum += ex2(fmaf(__uint_as_float(x[e]), kLog2eOverSqrtD, -mn));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j0 + c * 32 + e <= t_r) sum += ex2(fmaf(__uint_as_float(x[e]), kLog2eOverSqrtD, -mn));
                    }
                    l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + sum;
                    m = mn;
                }
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------------ phase 2: scores
        const int r = threadIdx.x - 256;  // key within the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        int cur = -1;
        bool gave_up = false;
        for (int i = 0; i < n_local; ++i) {
            const int t = cta + i * P, u = t / a.T_u, ti = t - u * a.T_u;
            if (u != cur) {
                named_sync(2, 128);  // all threads are done with the previous unit's lse
                if (r == 0) {
                    const unsigned* flag = a.inject ? a.never : a.ready + u;
                    bool ok = ld_acquire(flag) != 0;
                    for (long long spins = 0; !ok && !gave_up && spins < a.spin_limit; ++spins) {
                        __nanosleep(64);
                        ok = ld_acquire(flag) != 0;
                    }
                    if (!ok) {
                        atomicOr(a.err, kErrTimeout);
                        gave_up = true;  // later units do not wait again
                    }
                    sm.flag2 = ok;
                }
                named_sync(2, 128);
                const bool ok = sm.flag2;
                sm.lse[r] = (ok && r < a.nq) ? __ldcg(a.lse + (size_t)u * kQRows + r) : INFINITY;
                named_sync(2, 128);
                cur = u;
            }
            const int b = i & 1;
            mbar_wait(&sm.d2full[b], (i >> 1) & 1, sm, a.err);
            tc_fence_after();
            const int j = ti * kTileKeys + r;
            const bool full_tile = (ti + 1) * kTileKeys <= a.N - a.w + 1;
            float s = 0.f;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t x[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + 256 + b * 128 + c * 32, x);
                tmem_wait(x);
                if (c == 3) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.d2empty[b]);
                }
                const float4* L4 = reinterpret_cast<const float4*>(sm.lse + c * 32);
                if (full_tile) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 L = L4[e4];
                        s += ex2(fmaf(__uint_as_float(x[4 * e4 + 0]), kLog2eOverSqrtD, -L.x));
                        s += ex2(fmaf(__uint_as_float(x[4 * e4 + 1]), kLog2eOverSqrtD, -L.y));
                        s += ex2(fmaf(__uint_as_float(x[4 * e4 + 2]), kLog2eOverSqrtD, -L.z));
                        s += ex2(fmaf(__uint_as_float(x[4 * e4 + 3]), kLog2eOverSqrtD, -L.w));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int qr = c * 32 + e;
                        if (qr < a.nq && j <= a.N - a.w + (qr % a.w))
                            s += ex2(fmaf(__uint_as_float(x[e]), kLog2eOverSqrtD, -sm.lse[qr]));
                    }
                }
            }
            if (j < a.N) a.unit_scores[(size_t)u * a.N + j] = s;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// Copies the unit's query rows into a zero-padded [U][128][128] block (rows >= nq are 0)
// and clears the per-unit counters and flags of this call.
__global__ void tc_prep_kernel(const __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ qpad, int U, int nq,
                               unsigned* __restrict__ flags, int n_flags) {
    const long long total = (long long)U * kQRows * (kHeadDim / 8);  // 16-byte pieces
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int piece = (int)(e % (kHeadDim / 8));
        const long long row = e / (kHeadDim / 8);
        const int r = (int)(row % kQRows);
        const long long u = row / kQRows;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < nq) v = *reinterpret_cast<const uint4*>(q + ((u * nq + r) * kHeadDim + piece * 8));
        *reinterpret_cast<uint4*>(qpad + (row * kHeadDim + piece * 8)) = v;
    }
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_flags;
         e += (long long)gridDim.x * blockDim.x)
        flags[e] = 0u;
}

// ------------------------------------------------------------------------ host side

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

struct TcLayout {
    size_t qpad, partial, lse, flags, total;
};

TcLayout tc_layout(int U) {
    TcLayout L;
    size_t off = 0;
    L.qpad = off;
    off = a256(off + (size_t)U * kQRows * kHeadDim * 2);
    L.partial = off;
    off = a256(off + (size_t)U * kQRows * kMaxCtas * sizeof(float2));
    L.lse = off;
    off = a256(off + (size_t)U * kQRows * sizeof(float));
    L.flags = off;  // count[U], ready[U], never
    off = a256(off + (size_t)(2 * U + 1) * sizeof(unsigned));
    L.total = off;
    return L;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::atomic<void*> fn{nullptr};
    void* f = fn.load();
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn.store(f);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 64) cache[dev] = n;
    return n;
}

}  // namespace

bool tc_score_supported(const ScoreJob& j) {
    return j.dtype == KVC_BF16 && j.nq >= 1 && j.nq <= kQRows && j.N >= 1 && j.U >= 1 &&
           (long long)j.U * kQRows < (1LL << 31);
}

size_t tc_score_workspace(int U, int /*N*/, int /*nq*/) { return tc_layout(U).total; }

cudaError_t tc_score(const ScoreJob& j, cudaStream_t s) {
    const TcLayout L = tc_layout(j.U);
    char* ws = (char*)j.tc_ws;
    if (j.tc_ws_bytes < L.total) return cudaErrorInvalidValue;
    __nv_bfloat16* qpad = (__nv_bfloat16*)(ws + L.qpad);
    unsigned* flags = (unsigned*)(ws + L.flags);

    TcArgs a{};
    a.unit_scores = j.unit_scores;
    a.partial = (float2*)(ws + L.partial);
    a.lse = (float*)(ws + L.lse);
    a.count = flags;
    a.ready = flags + j.U;
    a.never = flags + 2 * j.U;
    a.err = j.err;
    a.spin_limit = j.spin_limit;
    a.U = j.U;
    a.N = j.N;
    a.w = j.window;
    a.nq = j.nq;
    a.T_u = (j.N + kTileKeys - 1) / kTileKeys;
    a.total_tiles = a.U * a.T_u;
    const int n_sm = sm_count();
    if (n_sm <= 0) return cudaErrorNoDevice;
    a.P = min(min(n_sm, kMaxCtas), a.total_tiles);
    a.lag = (a.T_u + a.P - 1) / a.P + 1;
    a.inject = j.inject_timeout;

    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    {
        cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)j.N, (cuuint64_t)j.U};
        cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)j.N * kHeadDim * 2};
        cuuint32_t box[3] = {64, kTileKeys, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        if (encode(&a.tmap_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(j.k), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)j.U * kQRows};
        cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
        cuuint32_t box[2] = {64, kQRows};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&a.tmap_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qpad, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }

    const long long pieces = (long long)j.U * kQRows * (kHeadDim / 8);
    const int prep_grid = (int)std::min<long long>((pieces + 255) / 256, 148LL * 8);
    tc_prep_kernel<<<prep_grid, 256, 0, s>>>((const __nv_bfloat16*)j.q, qpad, j.U, j.nq, flags, 2 * j.U + 1);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev >= 64 || !attr_set[dev].load()) {
        e = cudaFuncSetAttribute(tc_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev].store(true);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, tc_score_kernel, a);
    count_launches(1);
    return e;
}

}  // namespace kvc

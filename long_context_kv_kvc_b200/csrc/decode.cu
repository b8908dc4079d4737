// decode.cu -- decode attention over a clustered KV cache.
//
// What it computes (CentroidKV page, sec. 4 "Aggregatie": attention runs over the centroids
// with the cluster degree as a log term in the softmax): for decode query row i of query
// head g, over the n cached rows t of KV head h = g / G,
//     x_t = q . k_t / sqrt(D) + ln n_t,   out = sum_t softmax(x)_t v_t
// (n_t = 1 for every row when no degrees are given: plain attention).  Every cached row
// precedes the decode queries, so there is no mask.
//
// Design for B200.  With G * nq <= 8 query rows per KV head the work is 2 x 4 x 128 FMA per
// cached row against 512 bytes of K and V (bf16): ~2 FMA per byte, an HBM stream whose
// limit is instruction issue, not arithmetic.
// bf16 caches (decode_tc_kernel): persistent CTAs take balanced contiguous ranges of the
// (unit, 128-row tile) sequence.  A TMA producer streams each tile's K, V and the unit's Q
// through a 3-stage ring; one thread issues Q K^T as tcgen05.mma with M = 128 cached rows
// and N = 16 query rows (fp32 accumulate in TMEM), so the logits arrive one cached row per
// TMEM lane with no CUDA-core work; two epilogue warpgroups (alternate tiles) take the
// warp's 32 rows' logits, run the online softmax in base 2 with log2(degree) added, and
// accumulate P V on the CUDA cores in fp32 (lane l owns dimensions 4l..4l+3; the weights
// are broadcast from shared memory, V is read from the swizzled stage).  Every warp keeps
// its own state per unit and writes it as a partial; a combine kernel merges them.
// fp32 caches (decode_attn_kernel), a split-K "flash decoding" on the CUDA cores:
//   * a warp owns a contiguous span of one row's cache; lane l owns dimensions 4l..4l+3,
//     so every key and value row is one coalesced 512-byte warp load, and the next
//     sub-tile's loads are in flight while the current one is computed;
//   * a sub-tile is 32 / R keys for R (padded) query rows, i.e. 32 (key, row) pairs: each
//     lane forms the pairs' partial dot products over its 4 dimensions and a 5-level
//     butterfly reduce-scatter leaves lane p with the full dot product of pair p (31
//     shuffles per 32 dot products instead of 5 per dot product);
//   * online softmax in base 2 (the degree enters as log2 n_t, the logit scale as
//     log2(e) / sqrt(D)) per row, then each lane accumulates its dimensions of R outputs;
//   * every warp writes its (max, sum, output) state; a second kernel merges the spans.
#include <math.h>

#include <algorithm>
#include <atomic>

#include "kvc_internal.cuh"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

constexpr int D = kHeadDim;
constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecCtasPerSm = 1;
constexpr int kDecMaxRows = 8;      // G * nq query rows per KV head
constexpr int kSpanQuantum = 32;    // spans are whole multiples of every sub-tile size
constexpr int kMinSpan = 256;       // a warp streams at least this many rows
constexpr int kMaxSmForSizing = 160;
constexpr int kL2Ahead = 64;        // rows of K and V prefetched into L2 ahead of the loads
constexpr unsigned kFull = 0xffffffffu;

// rows [t, t + rows) of one unit's K and V into L2 (bulk prefetch: one instruction per tensor)
template <typename T>
__device__ __forceinline__ void l2_prefetch_rows(const T* k_row0, const T* v_row0, int t, int rows) {
    if (rows <= 0) return;
    const uint32_t bytes = (uint32_t)rows * D * sizeof(T);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"((uint64_t)__cvta_generic_to_global(k_row0 + (size_t)t * D)),
                 "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"((uint64_t)__cvta_generic_to_global(v_row0 + (size_t)t * D)),
                 "r"(bytes) : "memory");
}

// 4 elements of an fp32 row as raw bits (16 bytes)
template <typename T>
struct Raw4;
template <>
struct Raw4<float> {
    uint4 u;
};

__device__ __forceinline__ void ld4(const float* p, Raw4<float>& r) { r.u = __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void zero4(Raw4<float>& r) { r.u = make_uint4(0, 0, 0, 0); }
__device__ __forceinline__ void cvt4(const Raw4<float>& r, float (&x)[4]) {
    x[0] = __uint_as_float(r.u.x);
    x[1] = __uint_as_float(r.u.y);
    x[2] = __uint_as_float(r.u.z);
    x[3] = __uint_as_float(r.u.w);
}

// Warp w of the grid handles span sp of unit u = (batch, KV head): rows
// [sp * span, min(n, (sp + 1) * span)).  Unit u's cache rows start at u * ld; its Rv query
// rows (the G heads' nq queries) at u * Rv.  R = Rv rounded up to a power of two.
template <int R, typename T>
__global__ void __launch_bounds__(kDecThreads, kDecCtasPerSm)
decode_attn_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const int32_t* __restrict__ deg, int U, int Rv, int n, long long ld, int splits, int span,
                   float2* __restrict__ part_ml, float* __restrict__ part_o, unsigned* __restrict__ err) {
    constexpr int KT = 32 / R;  // keys per sub-tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * kDecWarps + warp;
    if (gw >= (long long)U * splits) return;
    const int u = (int)(gw / splits), sp = (int)(gw - (long long)u * splits);
    const int t_beg = sp * span, t_end = min(n, t_beg + span);
    // the split's rows lie inside the unit's cache rows
    if (!dcheck(err, t_beg >= 0 && n <= ld)) return;
    const T* k_row0 = k + (size_t)u * ld * D;
    const T* v_row0 = v + (size_t)u * ld * D;
    const T* kr = k_row0 + 4 * lane;
    const T* vr = v_row0 + 4 * lane;
    const int32_t* dr = deg ? deg + (size_t)u * ld : nullptr;
    if (lane == 0) l2_prefetch_rows(k_row0, v_row0, t_beg, min(kL2Ahead, t_end - t_beg));

    float qv[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (r < Rv) {
            Raw4<T> raw;
            ld4(q + ((size_t)u * Rv + r) * D + 4 * lane, raw);
            cvt4(raw, qv[r]);
#pragma unroll
            for (int d = 0; d < 4; ++d) qv[r][d] *= kLog2eOverSqrtD;
        } else {
#pragma unroll
            for (int d = 0; d < 4; ++d) qv[r][d] = 0.f;
        }
    }
    float o[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int d = 0; d < 4; ++d) o[r][d] = 0.f;
    float m = -INFINITY, l = 0.f;  // of row (lane % R), replicated over that row's lanes

    Raw4<T> kc[KT], vc[KT];
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        if (t_beg + j < t_end) {
            ld4(kr + (size_t)(t_beg + j) * D, kc[j]);
            ld4(vr + (size_t)(t_beg + j) * D, vc[j]);
        } else {
            zero4(kc[j]);
            zero4(vc[j]);
        }
    }
    const int my_key = lane / R;  // the pair this lane ends with: key my_key, row lane % R
    for (int t0 = t_beg; t0 < t_end; t0 += KT) {
        // keep the L2 stream kL2Ahead rows ahead (every 32 rows)
        if (lane == 0 && ((t0 - t_beg) & 31) == 0)
            l2_prefetch_rows(k_row0, v_row0, t0 + kL2Ahead, min(32, t_end - (t0 + kL2Ahead)));
        // next sub-tile's rows
        Raw4<T> kn[KT], vn[KT];
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            const int t = t0 + KT + j;
            if (t < t_end) {
                ld4(kr + (size_t)t * D, kn[j]);
                ld4(vr + (size_t)t * D, vn[j]);
            } else {
                zero4(kn[j]);
                zero4(vn[j]);
            }
        }
        // log2 of the degree of key (t0 + lane), lanes < KT
        float bias = 0.f;
        if (dr && lane < KT && t0 + lane < t_end) {
            int dg = dr[t0 + lane];
            if (dg < 1) {  // degrees count merged tokens: never below 1
                atomicOr(err, kErrIndex);
                dg = 1;
            }
            bias = log2f((float)dg);
        }
        // partial dot products of the 32 (key, row) pairs over this lane's dimensions
        float part[32];
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            float kf[4];
            cvt4(kc[j], kf);
#pragma unroll
            for (int r = 0; r < R; ++r)
                part[j * R + r] = fmaf(qv[r][3], kf[3], fmaf(qv[r][2], kf[2], fmaf(qv[r][1], kf[1], qv[r][0] * kf[0])));
        }
        // butterfly reduce-scatter: after the level with offset h, a lane whose bit h is set
        // holds the upper half of the remaining pairs; lane p ends with pair p
#pragma unroll
        for (int h = 16; h >= 1; h >>= 1) {
            const bool up = lane & h;
#pragma unroll
            for (int i = 0; i < h; ++i) {
                const float send = up ? part[i] : part[i + h];
                const float keep = up ? part[i + h] : part[i];
                part[i] = keep + __shfl_xor_sync(kFull, send, h);
            }
        }
        float y = part[0] + __shfl_sync(kFull, bias, my_key);
        if (t0 + my_key >= t_end) y = -INFINITY;
        // online softmax of row (lane % R) over the sub-tile's keys (lanes lane ^ (R, 2R, ..))
        float tm = y;
#pragma unroll
        for (int off = R; off < 32; off <<= 1) tm = fmaxf(tm, __shfl_xor_sync(kFull, tm, off));
        const float m_new = fmaxf(m, tm);  // finite: a sub-tile holds at least one key
        const float alpha = exp2f(m - m_new);
        const float p = exp2f(y - m_new);
        float ps = p;
#pragma unroll
        for (int off = R; off < 32; off <<= 1) ps += __shfl_xor_sync(kFull, ps, off);
        l = l * alpha + ps;
        m = m_new;
        // this lane's dimensions of every row's output
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float a = __shfl_sync(kFull, alpha, r);
#pragma unroll
            for (int d = 0; d < 4; ++d) o[r][d] *= a;
        }
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            float vf[4];
            cvt4(vc[j], vf);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float pr = __shfl_sync(kFull, p, j * R + r);
#pragma unroll
                for (int d = 0; d < 4; ++d) o[r][d] = fmaf(pr, vf[d], o[r][d]);
            }
        }
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            kc[j] = kn[j];
            vc[j] = vn[j];
        }
    }
    if (lane < R) part_ml[gw * R + lane] = make_float2(m, l);
#pragma unroll
    for (int r = 0; r < R; ++r)
        *reinterpret_cast<float4*>(part_o + ((size_t)gw * R + r) * D + 4 * lane) =
            make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
}

// ------------------------------------------------------------------------ bf16, tensor cores

constexpr int kDtStages = 3;
constexpr int kDtGroups = 2;                          // epilogue warpgroups (alternate tiles)
constexpr int kDtEpiWarps = 4 * kDtGroups;
constexpr int kDtThreads = (2 + kDtEpiWarps) * 32;    // warp 0 TMA, 1 MMA + TMEM owner, 2.. epilogue
constexpr int kDtTile = 128;                          // cached rows per tile (MMA M)
constexpr int kDtQRows = 16;                          // MMA N: query rows, padded
constexpr int kDtHalf = kDtTile * 64 * 2;             // 64-dimension half of a K or V tile
constexpr int kDtQHalf = kDtQRows * 64 * 2;
constexpr int kDtMaxCtas = 160;
constexpr uint32_t kDtCols = 32;                      // two 16-column accumulators
// kind::f16, fp32 accumulate, bf16 A and B, K-major, N = 16, M = 128
constexpr uint32_t kIdescN16 = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

struct DecTcArgs {
    CUtensorMap tmap_k, tmap_v;  // [U][ld][128] bf16, box 64 x 128 x 1, 128-byte swizzle
    CUtensorMap tmap_q;          // [U * Rv][128] bf16, box 64 x 16, 128-byte swizzle
    const int32_t* deg;
    float2* part_ml;             // [(P + U) * kDtEpiWarps][8]
    float* part_o;               // [(P + U) * kDtEpiWarps][8][128]
    unsigned* err;
    int U, Rv, n, T_u;
    long long ld, X;             // X = U * T_u tiles
};

struct __align__(1024) DecSmem {
    uint8_t k[kDtStages][2][kDtHalf];
    uint8_t v[kDtStages][2][kDtHalf];
    uint8_t q[kDtStages][2][kDtQHalf];
    float4 p[kDtEpiWarps][32][4];  // per epilogue warp: (p_r, p_r) pairs of its 32 rows, rows 0..7
    uint64_t full[kDtStages], empty[kDtStages], accfull[kDtGroups], accempty[kDtGroups];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(DecSmem) + 1024 <= 232448, "decode stages exceed the shared memory of a CTA");

template <int ACC>
__device__ __forceinline__ void umma_n16(uint32_t d, uint64_t a, uint64_t b) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(kIdescN16), "n"(ACC)
        : "memory");
}

// 8 consecutive fp32 columns of this thread's TMEM lane (valid after the wait)
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
}

__device__ __forceinline__ void mbar_drain_dec(uint64_t* bar, uint32_t parity, unsigned* err) {
    const long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kBarrierTimeoutNs) {
            atomicOr(err, kErrTimeout);
            return;
        }
    }
}

__device__ __forceinline__ long long item_start(int c, int P, long long X) { return (long long)c * X / P; }

template <int R>
__global__ void __launch_bounds__(kDtThreads, 1) decode_tc_kernel(const __grid_constant__ DecTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, P = gridDim.x;
    const long long g0 = item_start(c, P, a.X), g1 = item_start(c + 1, P, a.X);
    const int n_local = (int)(g1 - g0);
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDtStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 4);  // the four warps of the group that used the stage
        }
        for (int g = 0; g < kDtGroups; ++g) {
            mbar_init(&sm.accfull[g], 1);
            mbar_init(&sm.accempty[g], 4);
        }
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kDtCols)
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
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_v)) : "memory");
            int issued = 0;
            for (int i = 0; i < n_local && !*abort; ++i) {
                const long long g = g0 + i;
                const int u = (int)(g / a.T_u), tau = (int)(g - (long long)u * a.T_u);
                const int s = i % kDtStages;
                // the tile starts inside the unit's cached rows
                if (!dcheck(a.err, u >= 0 && u < a.U && tau >= 0 && (long long)tau * kDtTile < a.n && a.n <= a.ld)) {
                    *abort = 1;
                    break;
                }
                mbar_wait(&sm.empty[s], ((i / kDtStages) & 1) ^ 1, abort, a.err);
                if (*abort) break;
                mbar_expect_tx(&sm.full[s], 4 * kDtHalf + 2 * kDtQHalf);
                for (int h = 0; h < 2; ++h) {
                    tma_load_3d(sm.k[s][h], &a.tmap_k, &sm.full[s], 64 * h, tau * kDtTile, u);
                    tma_load_3d(sm.v[s][h], &a.tmap_v, &sm.full[s], 64 * h, tau * kDtTile, u);
                    tma_load_2d(sm.q[s][h], &a.tmap_q, &sm.full[s], 64 * h, u * a.Rv);
                }
                issued = i + 1;
            }
            for (int i = max(0, issued - kDtStages); i < issued; ++i)
                mbar_drain_dec(&sm.full[i % kDtStages], (i / kDtStages) & 1, a.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer: D = K Q^T
        if (lane == 0) {
            int last = -1;
            for (int i = 0; i < n_local && !*abort; ++i) {
                const int s = i % kDtStages, g = i % kDtGroups;
                mbar_wait(&sm.full[s], (i / kDtStages) & 1, abort, a.err);
                mbar_wait(&sm.accempty[g], ((i / kDtGroups) & 1) ^ 1, abort, a.err);
                if (*abort) break;
                tc_fence_after();
                const uint32_t d = tmem + g * kDtQRows;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint64_t dk = sw128_desc(smem_u32(sm.k[s][h])), dq = sw128_desc(smem_u32(sm.q[s][h]));
                    if (h == 0) umma_n16<0>(d, dk, dq);
                    else umma_n16<1>(d, dk, dq);
                    umma_n16<1>(d, dk + 2, dq + 2);
                    umma_n16<1>(d, dk + 4, dq + 4);
                    umma_n16<1>(d, dk + 6, dq + 6);
                }
                umma_commit(&sm.accfull[g]);
                last = i;
            }
            if (last >= 0) mbar_drain_dec(&sm.accfull[last % kDtGroups], (last / kDtGroups) & 1, a.err);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warp wi (group grp, TMEM lane quadrant qd) takes rows 32 qd .. 32 qd + 31 of the
        // tiles i = grp, grp + 2, ...; its online-softmax state covers those rows of one unit
        // and is written out whenever the unit changes (an empty state for a unit of the
        // range it saw no tile of), so that every (range, unit, warp) slot is written.
        const int wi = warp - 2, grp = wi >> 2, qd = warp & 3;
        const int u_first = n_local > 0 ? (int)(g0 / a.T_u) : 0;
        const int u_last = n_local > 0 ? (int)((g1 - 1) / a.T_u) : -1;
        float m[R], l[R], o[R][4];
        int cur_u = u_first;
        auto reset = [&]() {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                m[r] = -INFINITY;
                l[r] = 0.f;
#pragma unroll
                for (int d = 0; d < 4; ++d) o[r][d] = 0.f;
            }
        };
        auto flush = [&](int u) {
            // partial slots: (P + U) * kDtEpiWarps, CTA c's k-th unit boundary at c + k
            if (!dcheck(a.err, u >= 0 && c + u < P + a.U)) return;
            const size_t slot = ((size_t)(c + u)) * kDtEpiWarps + wi;
            float mm = -INFINITY, ll = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (lane == r) {
                    mm = m[r];
                    ll = l[r];
                }
            if (lane < 8) a.part_ml[slot * 8 + lane] = make_float2(mm, ll);
#pragma unroll
            for (int r = 0; r < R; ++r)
                *reinterpret_cast<float4*>(a.part_o + (slot * 8 + r) * D + 4 * lane) =
                    make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
        };
        reset();
        float4* pw = sm.p[wi][0];
        for (int i = grp, it = 0; i < n_local; i += kDtGroups, ++it) {
            const long long g = g0 + i;
            const int u = (int)(g / a.T_u), tau = (int)(g - (long long)u * a.T_u);
            if (u != cur_u) {
                flush(cur_u);
                reset();
                for (int uu = cur_u + 1; uu < u; ++uu) flush(uu);  // units of the range this warp saw no tile of
                cur_u = u;
            }
            const int t = tau * kDtTile + 32 * qd + lane;  // this lane's cached row
            const bool valid = t < a.n;
            float bias = 0.f;
            if (a.deg && valid) {
                int dg = a.deg[(size_t)u * a.ld + t];
                if (dg < 1) {
                    atomicOr(a.err, kErrIndex);
                    dg = 1;
                }
                bias = log2f((float)dg);
            }
            mbar_wait(&sm.accfull[grp], it & 1, abort, a.err);
            tc_fence_after();
            uint32_t x[8];
            tmem_ld8(tmem + ((uint32_t)(32 * qd) << 16) + grp * kDtQRows, x);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.accempty[grp]);
            // online softmax of each query row over the warp's 32 cached rows
            float p[R], alpha[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float y = valid ? fmaf(__uint_as_float(x[r]), kLog2eOverSqrtD, bias) : -INFINITY;
                float tm = y;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) tm = fmaxf(tm, __shfl_xor_sync(kFull, tm, off));
                const float m_new = fmaxf(m[r], tm);
                const float ms = m_new == -INFINITY ? 0.f : m_new;  // nothing seen yet: keep 0 weights
                alpha[r] = exp2f(m[r] - ms);
                p[r] = exp2f(y - ms);
                float ps = p[r];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(kFull, ps, off);
                l[r] = fmaf(l[r], alpha[r], ps);
                m[r] = m_new;
            }
#pragma unroll
            for (int r2 = 0; r2 < R / 2; ++r2)
                pw[lane * 4 + r2] = make_float4(p[2 * r2], p[2 * r2], p[2 * r2 + 1], p[2 * r2 + 1]);
            __syncwarp();
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int d = 0; d < 4; ++d) o[r][d] *= alpha[r];
            // P V over the warp's valid rows (V from the stage, 128-byte swizzle: 16-byte chunk
            // c of row j sits at chunk c ^ (j % 8))
            const int s = i % kDtStages;
            const int nvalid = min(32, max(0, a.n - (tau * kDtTile + 32 * qd)));
            const uint8_t* vbox = sm.v[s][lane >> 4];
            const int chunk = (lane & 15) >> 1, half8 = (lane & 1) << 3;
            for (int j = 0; j < nvalid; ++j) {
                const int row = 32 * qd + j;
                const uint2 raw = *reinterpret_cast<const uint2*>(vbox + row * 128 + ((chunk ^ (row & 7)) << 4) + half8);
                const float v0 = __uint_as_float(raw.x << 16), v1 = __uint_as_float(raw.x & 0xffff0000u);
                const float v2 = __uint_as_float(raw.y << 16), v3 = __uint_as_float(raw.y & 0xffff0000u);
#pragma unroll
                for (int r2 = 0; r2 < R / 2; ++r2) {
                    const float4 pp = pw[j * 4 + r2];
                    o[2 * r2][0] = fmaf(pp.x, v0, o[2 * r2][0]);
                    o[2 * r2][1] = fmaf(pp.y, v1, o[2 * r2][1]);
                    o[2 * r2][2] = fmaf(pp.x, v2, o[2 * r2][2]);
                    o[2 * r2][3] = fmaf(pp.y, v3, o[2 * r2][3]);
                    o[2 * r2 + 1][0] = fmaf(pp.z, v0, o[2 * r2 + 1][0]);
                    o[2 * r2 + 1][1] = fmaf(pp.w, v1, o[2 * r2 + 1][1]);
                    o[2 * r2 + 1][2] = fmaf(pp.z, v2, o[2 * r2 + 1][2]);
                    o[2 * r2 + 1][3] = fmaf(pp.w, v3, o[2 * r2 + 1][3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        if (u_last >= u_first) {
            flush(cur_u);
            reset();
            for (int uu = cur_u + 1; uu <= u_last; ++uu) flush(uu);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDtCols) : "memory");
    }
}

// One warp per (unit, query row): merges the (range, warp) partials of every range that
// touches the unit.  The partials' (max, sum) are read 32 at a time, one per lane (the max
// and the weighted sum are warp reductions); each lane accumulates its 4 dimensions over
// the partials in order with kCombineDepth loads in flight, the weights broadcast by shuffles.
constexpr int kCombineDepth = 8;
__global__ void __launch_bounds__(256)
decode_tc_combine_kernel(const float2* __restrict__ part_ml, const float* __restrict__ part_o, int U, int Rv, int P,
                         long long X, int T_u, float* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= (long long)U * Rv) return;
    const int u = (int)(gw / Rv), r = (int)(gw - (long long)u * Rv);
    const long long lo = (long long)u * T_u, hi = lo + T_u;
    // the ranges [start(c), start(c + 1)) that overlap [lo, hi): start() is monotonic
    int c_lo = 0, c_hi = P - 1;
    for (int b = P - 1; c_lo < b;) {  // first c with start(c + 1) > lo
        const int mid = (c_lo + b) / 2;
        if (item_start(mid + 1, P, X) > lo) b = mid;
        else c_lo = mid + 1;
    }
    for (int a0 = 0; a0 < c_hi;) {  // last c with start(c) < hi
        const int mid = (a0 + c_hi + 1) / 2;
        if (item_start(mid, P, X) < hi) a0 = mid;
        else c_hi = mid - 1;
    }
    // slot s = 0 .. n_slots - 1 is partial (c_lo + u) * kDtEpiWarps + s (ranges and warps in order)
    const int n_slots = (c_hi - c_lo + 1) * kDtEpiWarps;
    const size_t slot0 = ((size_t)(c_lo + u)) * kDtEpiWarps;
    float M = -INFINITY;
    for (int s0 = 0; s0 < n_slots; s0 += 32) {
        const int sl = s0 + lane;
        if (sl < n_slots) M = fmaxf(M, part_ml[(slot0 + sl) * 8 + r].x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* po = part_o + (slot0 * 8 + r) * D + 4 * lane;
    for (int s0 = 0; s0 < n_slots; s0 += 32) {
        // lane t holds the weight of slot s0 + t (0 past the end and for empty states)
        const int sl = s0 + lane;
        const float2 ml = sl < n_slots ? part_ml[(slot0 + sl) * 8 + r] : make_float2(-INFINITY, 0.f);
        const float wt = ml.y == 0.f ? 0.f : exp2f(ml.x - M);
        L = fmaf(ml.y, wt, L);
        const int cnt = min(32, n_slots - s0);
        for (int t0 = 0; t0 < cnt; t0 += kCombineDepth) {
            float4 ov[kCombineDepth];
            float wg[kCombineDepth];
#pragma unroll
            for (int t = 0; t < kCombineDepth; ++t) {
                wg[t] = __shfl_sync(kFull, wt, (t0 + t) & 31);
                ov[t] = wg[t] != 0.f ? *reinterpret_cast<const float4*>(po + (size_t)(s0 + t0 + t) * 8 * D)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int t = 0; t < kCombineDepth; ++t) {
                acc[0] = fmaf(ov[t].x, wg[t], acc[0]);
                acc[1] = fmaf(ov[t].y, wg[t], acc[1]);
                acc[2] = fmaf(ov[t].z, wg[t], acc[2]);
                acc[3] = fmaf(ov[t].w, wg[t], acc[3]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(kFull, L, off);
    const float inv = 1.f / L;
    *reinterpret_cast<float4*>(out + (size_t)gw * D + 4 * lane) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
}

// One warp per (unit, query row): merges the spans' states in span order.
__global__ void __launch_bounds__(256)
decode_combine_kernel(const float2* __restrict__ part_ml, const float* __restrict__ part_o, int U, int R, int Rv,
                      int splits, float* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= (long long)U * Rv) return;
    const int u = (int)(gw / Rv), r = (int)(gw - (long long)u * Rv);
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part_ml[((size_t)u * splits + s) * R + r].x);
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < splits; ++s) {
        const size_t i = ((size_t)u * splits + s) * R + r;
        const float2 ml = part_ml[i];
        const float wgt = exp2f(ml.x - M);
        L = fmaf(ml.y, wgt, L);
        const float4 ov = *reinterpret_cast<const float4*>(part_o + i * D + 4 * lane);
        acc[0] = fmaf(ov.x, wgt, acc[0]);
        acc[1] = fmaf(ov.y, wgt, acc[1]);
        acc[2] = fmaf(ov.z, wgt, acc[2]);
        acc[3] = fmaf(ov.w, wgt, acc[3]);
    }
    const float inv = 1.f / L;
    *reinterpret_cast<float4*>(out + (size_t)gw * D + 4 * lane) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
}

// query rows per KV head, padded to a power of two and to at least 4 (sub-tiles of at most
// 8 keys keep the double-buffered K and V pieces in registers)
int pad_rows(int Rv) {
    int R = 4;
    while (R < Rv) R <<= 1;
    return R;
}

// spans per unit for n cached rows: enough warps to fill n_sm SMs, at least kMinSpan rows each
int decode_splits(int U, int n, int n_sm, int* span) {
    const int by_len = std::max(1, (n + kMinSpan - 1) / kMinSpan);
    const int by_sm = std::max(1, n_sm * kDecWarps * kDecCtasPerSm / U);
    int s = std::min(by_len, by_sm);
    int sp = (n + s - 1) / s;
    sp = (sp + kSpanQuantum - 1) / kSpanQuantum * kSpanQuantum;
    *span = sp;
    return (n + sp - 1) / sp;
}

template <int R, typename T>
cudaError_t launch_decode(const void* q, const void* k, const void* v, const int32_t* deg, int U, int Rv, int n,
                          long long ld, int splits, int span, float2* ml, float* po, unsigned* err, cudaStream_t s) {
    const long long warps = (long long)U * splits;
    const long long grid = (warps + kDecWarps - 1) / kDecWarps;
    if (grid > (1LL << 31) - 1) return cudaErrorInvalidValue;
    decode_attn_kernel<R, T><<<(unsigned)grid, kDecThreads, 0, s>>>((const T*)q, (const T*)k, (const T*)v, deg, U,
                                                                    Rv, n, ld, splits, span, ml, po, err);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_rows(int R, const void* q, const void* k, const void* v, const int32_t* deg, int U, int Rv,
                          int n, long long ld, int splits, int span, float2* ml, float* po, unsigned* err,
                          cudaStream_t s) {
    switch (R) {
        case 4: return launch_decode<4, T>(q, k, v, deg, U, Rv, n, ld, splits, span, ml, po, err, s);
        case 8: return launch_decode<8, T>(q, k, v, deg, U, Rv, n, ld, splits, span, ml, po, err, s);
        default: return cudaErrorInvalidValue;
    }
}

// One warp per new row (unit, i): copies its K and V row into slot n + i of the unit's cache
// (16-byte pieces) and sets that slot's degree to 1 and position to pos0 + i.
template <typename T>
__global__ void __launch_bounds__(256)
append_kernel(T* __restrict__ k_cache, T* __restrict__ v_cache, int32_t* __restrict__ deg_cache,
              int32_t* __restrict__ pos_cache, int U, long long ld, int n, const T* __restrict__ k_new,
              const T* __restrict__ v_new, int t_new, int pos0, unsigned* err) {
    constexpr int kPieces = D * (int)sizeof(T) / 16;  // 16-byte pieces per row
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= (long long)U * t_new) return;
    const int u = (int)(gw / t_new), i = (int)(gw - (long long)u * t_new);
    if (!dcheck(err, n + i < ld)) return;  // the new row fits the unit's cache rows
    const size_t src = ((size_t)u * t_new + i) * D, dst = ((size_t)u * ld + n + i) * D;
    for (int c = lane; c < 2 * kPieces; c += 32) {
        const bool isv = c >= kPieces;
        const int pc = isv ? c - kPieces : c;
        const uint4 x = reinterpret_cast<const uint4*>((isv ? v_new : k_new) + src)[pc];
        reinterpret_cast<uint4*>((isv ? v_cache : k_cache) + dst)[pc] = x;
    }
    if (lane == 0) {
        if (deg_cache) deg_cache[(size_t)u * ld + n + i] = 1;
        if (pos_cache) pos_cache[(size_t)u * ld + n + i] = pos0 + i;
    }
}

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

bool decode_rows_supported(int rows_per_kv_head) { return rows_per_kv_head >= 1 && rows_per_kv_head <= kDecMaxRows; }

size_t decode_workspace(int U, int Rv, int n) {
    int span = 0;
    const int splits = decode_splits(U, n, kMaxSmForSizing, &span);
    const size_t simt = (size_t)U * splits * pad_rows(Rv);                  // fp32 caches
    const size_t tc = (size_t)(kDtMaxCtas + U) * kDtEpiWarps * 8;           // bf16 caches
    const size_t slots = std::max(simt, tc);
    return a256(slots * sizeof(float2)) + a256(slots * D * sizeof(float));
}

namespace {

cudaError_t decode_tc(const void* q, const void* k, const void* v, const int32_t* deg, int U, int Rv, int n,
                      long long ld, float* out, void* ws, cudaStream_t s) {
    DecTcArgs a{};
    a.deg = deg;
    a.err = device_error_word();
    a.U = U;
    a.Rv = Rv;
    a.n = n;
    a.ld = ld;
    a.T_u = (n + kDtTile - 1) / kDtTile;
    a.X = (long long)U * a.T_u;
    const int n_sm = sm_count();
    if (n_sm <= 0) return cudaErrorNoDevice;
    const int P = (int)std::min<long long>(std::min(n_sm, kDtMaxCtas), a.X);
    const size_t slots = (size_t)(P + U) * kDtEpiWarps * 8;
    a.part_ml = (float2*)ws;
    a.part_o = (float*)((char*)ws + a256(slots * sizeof(float2)));
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    cuuint32_t estr[3] = {1, 1, 1};
    {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)ld, (cuuint64_t)U};
        cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)ld * D * 2};
        cuuint32_t box[3] = {64, kDtTile, 1};
        if (encode(&a.tmap_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            encode(&a.tmap_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(v), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)U * Rv};
        cuuint64_t strides[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, kDtQRows};
        if (encode(&a.tmap_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(DecSmem) + 1024;
    const int R = pad_rows(Rv);
    static std::atomic<bool> attr_set[2][64];
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    const int ri = R == 8;
    if (dev >= 64 || !attr_set[ri][dev].load()) {
        e = ri ? cudaFuncSetAttribute(decode_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
               : cudaFuncSetAttribute(decode_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[ri][dev].store(true);
    }
    if (ri)
        decode_tc_kernel<8><<<P, kDtThreads, smem, s>>>(a);
    else
        decode_tc_kernel<4><<<P, kDtThreads, smem, s>>>(a);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long cw = (long long)U * Rv;
    decode_tc_combine_kernel<<<(unsigned)((cw + 7) / 8), 256, 0, s>>>(a.part_ml, a.part_o, U, Rv, P, a.X, a.T_u, out);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t decode_attention(const void* q, const void* k, const void* v, const int32_t* deg, int dtype, int U,
                             int Rv, int n, long long ld, float* out, void* ws, cudaStream_t s) {
    if (dtype == KVC_BF16) return decode_tc(q, k, v, deg, U, Rv, n, ld, out, ws, s);
    int n_sm = 0, dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    n_sm = std::min(n_sm, kMaxSmForSizing);  // the workspace is sized for at most this many
    int span = 0;
    const int splits = decode_splits(U, n, n_sm, &span);
    const int R = pad_rows(Rv);
    const size_t slots = (size_t)U * splits * R;
    float2* ml = (float2*)ws;
    float* po = (float*)((char*)ws + a256(slots * sizeof(float2)));
    unsigned* err = device_error_word();
    e = dispatch_rows<float>(R, q, k, v, deg, U, Rv, n, ld, splits, span, ml, po, err, s);
    count_launches(1);
    if (e != cudaSuccess) return e;
    const long long cw = (long long)U * Rv;
    decode_combine_kernel<<<(unsigned)((cw + 7) / 8), 256, 0, s>>>(ml, po, U, R, Rv, splits, out);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t append_rows(void* k_cache, void* v_cache, int32_t* deg_cache, int32_t* pos_cache, int dtype, int U,
                        long long ld, int n, const void* k_new, const void* v_new, int t_new, int pos0,
                        cudaStream_t s) {
    const long long warps = (long long)U * t_new;
    if (warps == 0) return cudaSuccess;
    const long long grid = (warps + 7) / 8;
    if (grid > (1LL << 31) - 1) return cudaErrorInvalidValue;
    if (dtype == KVC_BF16)
        append_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, s>>>(
            (__nv_bfloat16*)k_cache, (__nv_bfloat16*)v_cache, deg_cache, pos_cache, U, ld, n,
            (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, t_new, pos0, device_error_word());
    else
        append_kernel<float><<<(unsigned)grid, 256, 0, s>>>((float*)k_cache, (float*)v_cache, deg_cache, pos_cache, U,
                                                            ld, n, (const float*)k_new, (const float*)v_new, t_new,
                                                            pos0, device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvc

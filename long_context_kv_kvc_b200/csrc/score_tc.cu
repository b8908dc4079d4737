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
// Storing logits would cost more HBM traffic than K itself, so K is read twice and the
// second read is scheduled to hit L2.  With 128 query rows per unit the work is two
// exponentials per byte of K, which makes the special-function unit, not HBM, the
// tightest resource; the kernel is therefore organised to keep every consumer warp fed:
//   * one persistent CTA per SM (cooperative launch: all CTAs resident), 128-key tiles
//     dealt round-robin over the CTAs in global (unit-major) order;
//   * phase 1 streams K from HBM: D[128 q x 128 keys] = Q K^T (tcgen05.mma kind::f16,
//     M = N = 128, fp32 accumulator in TMEM); phase 2 re-reads each tile a bounded number
//     of tiles later (so it comes from L2, loaded evict-first): D[128 keys x 128 q] = K Q^T;
//   * two MMA issuers (one per phase) claim job numbers from a shared counter when their
//     next job is ready -- a phase-2 tile once its unit's lse is known -- and job n fills
//     TMEM accumulator n % 4; four consumer warpgroups each drain one accumulator and handle
//     either kind of job, so the exponentials do not wait on the cross-CTA dependency while
//     phase-1 work exists.  Accumulators are taken in job order and the phase-1 record ring
//     is released through a monotonic counter: a parity wait on an mbarrier that may lag two
//     phases behind its waiter would pass early;
//   * a phase-1 job yields per query row the tile's sum of 2^(y - ref) relative to a fixed
//     per-row reference ref (the row's logit with the key at its own position, computed
//     before the kernel; a tile with a much larger logit records its own shift of the
//     reference); a publisher warp adds the records in fp64 -- without an exponential
//     unless the reference moved -- and adds the CTA's part of a unit to the unit's fp64
//     total with fire-and-forget atomics, then bumps the unit's arrival count (fp64 addition
//     order moves the total by ~1e-16, far below fp32);
//   * an lse warp waits for each unit's count, turns the totals into lse = ref + log2(total)
//     in shared memory and releases the unit's phase-2 jobs; a phase-2 job gives each key
//     of the tile its sum over the query rows of 2^(y - lse).
// Phase 1 streams each 128-key tile from HBM as one 32 KiB TMA op (both 64-column halves, the
// 128-byte swizzle atom) into a 2-tile ring; phase 2 re-reads each tile as two 16 KiB halves,
// issued by two threads, into a 3-stage ring (a single issuing thread completes TMA ops at a
// roughly fixed rate, so large ops and several issuers stream faster).  Warps: 0 phase-1 TMA,
// 1 TMEM owner + phase-1 MMA, 2 and 6 phase-2 TMA (halves 0 and 1), 3 phase-2 MMA, 4 lse,
// 5 publisher, 7 idle, 8-23 consumers (four warpgroups, one per accumulator).  Every
// wait is bounded: a wait that runs out sets the per-device error word and the kernel
// still ends.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>

#include "kvc_internal.cuh"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

constexpr int kTileKeys = 128;                         // keys per tile (MMA N / M)
constexpr int kQRows = 128;                            // query rows per unit (padded)
constexpr int kBoxBytes = kTileKeys * 64 * 2;          // a 128-row x 64-column bf16 box: 16 KiB
#ifndef KVC_TC_STAGES_A
#define KVC_TC_STAGES_A 4
#endif
#ifndef KVC_TC_STAGES_B
#define KVC_TC_STAGES_B 3
#endif
#ifndef KVC_TC_Q_SLOTS
#define KVC_TC_Q_SLOTS 3
#endif
#ifndef KVC_TC_LEAD_SLACK
#define KVC_TC_LEAD_SLACK 5
#endif
constexpr int kStagesA = KVC_TC_STAGES_A;              // phase-1 ring, in 16 KiB halves (HBM stream)
constexpr int kTilesA = kStagesA / 2;                  // the same ring in whole tiles (one op each)
constexpr int kStagesB = KVC_TC_STAGES_B;              // phase-2 ring (L2 re-read)
// A single-phase launch (kStats, kScores) has no phase-2 ring: its tiles stream through the
// phase-1 ring extended over the phase-2 ring's memory (which follows it), one more tile in
// flight per SM.
constexpr int kTiles1 = (kStagesA + kStagesB) / 2;
constexpr int kQSlots = KVC_TC_Q_SLOTS;                // Q of the CTA's last units, by unit ordinal
constexpr int kLeadSlack = KVC_TC_LEAD_SLACK;          // phase-1 lead beyond one unit, in tiles
constexpr int kAcc = 4;                // TMEM accumulators (128 columns each) = consumer warpgroups
constexpr int kRec = 8;                // phase-1 tile records between consumers and publisher
constexpr int kWarps = 24;
constexpr int kThreads = kWarps * 32;
constexpr int kConsumer0 = 8;          // first consumer warp
#ifndef KVC_TC_SUM_COPIES
#define KVC_TC_SUM_COPIES 8
#endif
constexpr int kSumCopies = KVC_TC_SUM_COPIES;  // copies of each unit's totals (CTA c adds to copy c % kSumCopies)
constexpr int kMaxCtas = 160;                          // upper bound on the persistent grid
constexpr int kRefSamples = 8;         // kStats: keys whose largest logit is a row's reference
constexpr uint32_t kTmemCols = 512;

struct TcArgs {
    CUtensorMap tmap_k;  // K as [U][N][128] bf16, box 64 x 128 x 1, 128-byte swizzle (a half tile)
    CUtensorMap tmap_k4; // K as [U][2 halves][N][64] (strides: key 256 B, half 128 B), box 64 x 128 x 2 x 1,
                         // 128-byte swizzle: a whole tile in one op, the two halves one after the other
    CUtensorMap tmap_q;  // padded Q as [U*128][128] bf16, box 64 x 128, 128-byte swizzle
    float* unit_scores;  // [U][N]
    const float* ref;    // [U][128] per-row reference logit (base 2): the row's own-position key
    double* sum;         // [U][kSumCopies][128] sums over keys of 2^(y - ref); CTA c adds into copy
                         // c % kSumCopies, which spreads the atomics of the 148 CTAs over more addresses
    double* sum_t;       // [U][kSumCopies][128] sums of 2^(y - ref) (y - ref), for the entropy
    float* entropy;      // [U][nq] attention entropy (nats) per window row, or null
    unsigned* count;     // [U] CTAs that have added their part of unit u
    unsigned* never;     // a counter nothing increments (wait-timeout injection)
    unsigned* err;
    long long spin_limit;
    int U, N, w, nq, T_u, total_tiles, P, max_lead, inject;
    // sequence sharding: the N keys are positions key_off .. key_off + N - 1 of a sequence of
    // n_total (0 and N when not sharded); window row i sits at position n_total - w + i
    int key_off, n_total;
    float2* ml_out;       // kStats: per (unit, row) (m, l) with l 2^m = the row's sum of 2^y over the block
    const float* lse_in;  // kScores: [U][128] each row's log-sum-exp (base 2) over the whole sequence
};

// What a launch computes: the whole two-phase scoring, only the per-row normalisers of this
// block of keys (phase 1), or only the scores given the normalisers (phase 2).
enum TcMode { kFull = 0, kStats = 1, kScores = 2 };

struct __align__(1024) Smem {
    uint8_t ringA[kStagesA][kBoxBytes];
    uint8_t ringB[kStagesB][kBoxBytes];
    uint8_t q[kQSlots][2 * kBoxBytes];  // Q of the CTA's k-th unit in slot k % kQSlots (two boxes)
    float2 rec[kRec][kQRows];           // phase-1 tile i: per row (m - ref, sum of 2^(y - m))
    float rec_t[kRec][kQRows];          // with the entropy: sum of 2^(y - m) (y - m)
    float nlse[2][kQRows];              // -lse of the CTA's k-th unit in slot k % 2
    int4 job[kAcc];                     // {kind, unit, tile within unit, record or lse slot}
    uint64_t fullA[kStagesA], emptyA[kStagesA], fullB[kStagesB], emptyB[kStagesB];
    uint64_t qfull[kQSlots], qempty[kQSlots];
    uint64_t qempty2[kQSlots];  // single-phase launches: the second issuer's release of a Q slot
    uint64_t accfull[kAcc], accempty[kAcc];
    uint64_t recfull[kRec];
    uint64_t lsefull[2];
    unsigned lse_done[2];  // consumer warps done with the lse slot (monotonic)
    int next_job;          // job numbers claimed by the two MMA issuers
    int jobs_started;      // jobs that own their accumulator (taken in job order)
    int rec_consumed;      // phase-1 records the publisher has read (monotonic)
    uint32_t tmem_base;
    int abort;
    int p1_issued, p2_issued;  // tiles whose loads each producer has issued (L2 lead control)
};

static_assert(offsetof(Smem, ringB) == offsetof(Smem, ringA) + sizeof(Smem::ringA) && kTiles1 <= kStagesA &&
                  2 * kTiles1 <= kStagesA + kStagesB,
              "the single-phase ring spans the phase-1 and phase-2 rings");

// Spinning bounded wait (no suspension) for the single-thread roles, which must react fast.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_spin(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned* err) {
    if (mbar_test(bar, parity)) return;
    const long long t0 = globaltimer();
    while (!mbar_test(bar, parity)) {
        if (*abort) return;
        if (globaltimer() - t0 > kBarrierTimeoutNs) {
            atomicOr(err, kErrTimeout);
            *abort = 1;
            return;
        }
    }
}

// Bounded wait that ignores the fail-fast flag: after a time-out elsewhere, the producers
// wait for their own copies still in flight before the CTA exits.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned* err) {
    const long long t0 = globaltimer();
    while (!mbar_test(bar, parity)) {
        if (globaltimer() - t0 > kBarrierTimeoutNs) {
            atomicOr(err, kErrTimeout);
            return;
        }
    }
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// x * 2^d in fp64 for fp32 x and finite d: 2^d = 2^e * 2^f with e = floor(d), f in [0, 1);
// 2^f on the special-function unit (relative error ~2^-22), 2^e exact from its exponent bits.
__device__ __forceinline__ double scale_exp2(float x, float d) {
    const float e = floorf(d);
    const int ei = (int)fminf(fmaxf(e, -1022.f), 1023.f);
    return (double)(x * ex2(d - e)) * __longlong_as_double((long long)(ei + 1023) << 52);
}

// log2 of a positive normal fp64 value: its binary exponent plus log2 of the mantissa in
// [1/2, 1) on the special-function unit (absolute error ~2^-22).
__device__ __forceinline__ float log2_pos(double v) {
    const long long b = __double_as_longlong(v);
    const int e = (int)((b >> 52) & 0x7FF) - 1022;
    const double m = __longlong_as_double((b & ~(0x7FFLL << 52)) | (1022LL << 52));
    return (float)e + lg2((float)m);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Largest of 32 logits.
__device__ __forceinline__ float chunk_max(const uint32_t (&x)[32]) {
    float mx[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) mx[g] = __uint_as_float(x[g]);
#pragma unroll
    for (int e = 8; e < 32; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(x[e]));
    return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// Packed fp32 pairs (Blackwell's f32x2 FMA/ADD): one instruction for two lanes' worth of
// elementwise work.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// 2^y for both halves of a pair (special-function unit)
__device__ __forceinline__ uint64_t ex2_pair(uint64_t y) {
    float a, b;
    unpack2(y, a, b);
    return pack2(ex2(a), ex2(b));
}
__device__ __forceinline__ float hsum2(uint64_t v) {
    float a, b;
    unpack2(v, a, b);
    return a + b;
}

// Sum over 32 logits (invisible keys already set to kMasked) of 2^(y - m) for a fixed m;
// with ENT also tsum = sum of 2^(y - m) (y - m).
constexpr float kMasked = -3.0e38f;  // a masked logit: 2^(y - m) is 0 and so is its product with y - m
template <bool ENT>
__device__ __forceinline__ float sum_exp2_shifted(const uint32_t (&x)[32], float m, float& tsum) {
    const uint64_t c2 = pack2(kLog2eOverSqrtD, kLog2eOverSqrtD), nm2 = pack2(-m, -m);
    uint64_t acc0 = 0, acc1 = 0, at0 = 0, at1 = 0;  // (+0, +0) pairs
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        const uint64_t y0 = fma2(pack2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), c2, nm2);
        const uint64_t y1 = fma2(pack2(__uint_as_float(x[e + 2]), __uint_as_float(x[e + 3])), c2, nm2);
        const uint64_t e0 = ex2_pair(y0), e1 = ex2_pair(y1);
        acc0 = add2(acc0, e0);
        acc1 = add2(acc1, e1);
        if (ENT) {
            at0 = fma2(e0, y0, at0);
            at1 = fma2(e1, y1, at1);
        }
    }
    if (ENT) tsum = hsum2(add2(at0, at1));
    return hsum2(add2(acc0, acc1));
}

// Sum over 32 query rows (invisible ones already set to -inf) of 2^(y - lse) for this
// thread's key; nlse holds -lse per row.
__device__ __forceinline__ float prob_sum(const uint32_t (&x)[32], const float* nlse) {
    const uint64_t c2 = pack2(kLog2eOverSqrtD, kLog2eOverSqrtD);
    const ulonglong2* L = reinterpret_cast<const ulonglong2*>(nlse);
    uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
        const ulonglong2 l = L[e4];
        const int e = 4 * e4;
        const uint64_t y0 = fma2(pack2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), c2, l.x);
        const uint64_t y1 = fma2(pack2(__uint_as_float(x[e + 2]), __uint_as_float(x[e + 3])), c2, l.y);
        acc0 = add2(acc0, ex2_pair(y0));
        acc1 = add2(acc1, ex2_pair(y1));
    }
    return hsum2(add2(acc0, acc1));
}

// ------------------------------------------------------------------------ the kernel

// The CTA's local tiles i = 0, 1, ... are the global tiles cta + i * P; these helpers give
// their unit and the local range of each unit.
struct TileSeq {
    int cta, P, T_u, n_local;
    __device__ __forceinline__ int unit(int i) const { return (cta + i * P) / T_u; }
    __device__ __forceinline__ int tile(int i) const { return cta + i * P - unit(i) * T_u; }
    // first local tile whose global index is >= g
    __device__ __forceinline__ int first_at(long long g) const {
        const long long d = g - cta;
        const long long i = d <= 0 ? 0 : (d + P - 1) / P;
        return (int)(i < n_local ? i : n_local);
    }
    __device__ __forceinline__ int count(int u) const {
        return first_at((long long)(u + 1) * T_u) - first_at((long long)u * T_u);
    }
};

template <bool ENT, int MODE>
__global__ void __launch_bounds__(kThreads, 1) tc_score_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kRing = MODE == kFull ? kTilesA : kTiles1;  // tiles of the HBM ring
    const int cta = blockIdx.x, P = a.P;
    const int n_local = cta < a.total_tiles ? (a.total_tiles - cta + P - 1) / P : 0;
    const TileSeq seq{cta, P, a.T_u, n_local};
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesA; ++s) {
            mbar_init(&sm.fullA[s], 1);
            mbar_init(&sm.emptyA[s], 1);
        }
        for (int s = 0; s < kStagesB; ++s) {
            mbar_init(&sm.fullB[s], 1);
            mbar_init(&sm.emptyB[s], 1);
        }
        for (int b = 0; b < kQSlots; ++b) {
            mbar_init(&sm.qfull[b], 1);
            mbar_init(&sm.qempty[b], 1);
            mbar_init(&sm.qempty2[b], 1);
        }
        for (int b = 0; b < kAcc; ++b) {
            mbar_init(&sm.accfull[b], 2);   // the issuer's arrive (job record) + the MMA commit
            mbar_init(&sm.accempty[b], 4);  // one arrive per consumer warp
        }
        for (int b = 0; b < kRec; ++b) {
            mbar_init(&sm.recfull[b], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.lsefull[b], 1);
            sm.lse_done[b] = 0u;
        }
        sm.abort = 0;
        sm.next_job = 0;
        sm.jobs_started = 0;
        sm.rec_consumed = 0;
        sm.p1_issued = 0;
        sm.p2_issued = 0;
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

    if (warp == 0 || warp == 2 || warp == 6) {
        // ------------------------------------------------------------ TMA producers
        // Warp 0 streams the phase-1 tiles from HBM, one 32 KiB op per tile (both 64-column
        // halves); warps 2 and 6 issue the phase-2 re-reads, half 0 and half 1 of every tile.
        // A single issuing thread completes TMA ops at a roughly fixed rate, so the phase-1
        // stream uses large ops and the phase-2 stream two threads.  kStats: no phase-2
        // re-reads; kScores: no phase 1, so warp 0 streams the tiles (from HBM, one 32 KiB op
        // each) straight to the phase-2 jobs.  Both single-phase modes stream through a ring of
        // kTiles1 tiles (the phase-2 ring's memory added), which keeps more of HBM's latency
        // covered than the two tiles of the two-phase launch.
        if (lane == 0 && !(MODE != kFull && warp != 0)) {
            const int ph = warp == 0 ? 0 : 1, hh = warp == 6 ? 1 : 0;
            const CUtensorMap* mk = ph == 0 ? &a.tmap_k4 : &a.tmap_k;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(mk)) : "memory");
            const uint64_t evict_first = policy_evict_first();
            volatile int* other = ph == 0 ? &sm.p2_issued : &sm.p1_issued;
            int qunit = -1, ord = -1, i = 0;
            for (; i < n_local && !*abort; ++i) {
                const int u = seq.unit(i), ti = seq.tile(i);
                // the tile's coordinates address the unit's keys (and its Q block)
                if (!dcheck(a.err, u >= 0 && u < a.U && ti >= 0 && (long long)ti * kTileKeys < a.N)) {
                    *abort = 1;
                    break;
                }
                // phase 1 stays at most max_lead tiles ahead of phase 2 (L2 footprint);
                // phase 2 never loads a tile before phase 1 has (so its read hits L2)
                const bool lead_rule = ph == 1 || MODE == kFull;
                if (lead_rule && (ph == 0 ? (i - *other >= a.max_lead) : (i >= *other))) {
                    const long long t0 = globaltimer();
                    while (ph == 0 ? (i - *other >= a.max_lead) : (i >= *other)) {
                        if (*abort) break;
                        if (globaltimer() - t0 > kBarrierTimeoutNs) {
                            atomicOr(a.err, kErrTimeout);
                            *abort = 1;
                            break;
                        }
                        __nanosleep(32);
                    }
                }
                if (ph == 0 && u != qunit) {
                    // the CTA's ord-th unit: load its Q into slot ord % kQSlots once phase 2
                    // is done with the unit that used the slot kQSlots units ago
                    qunit = u;
                    ++ord;
                    const int slot = ord % kQSlots;
                    if (ord >= kQSlots) {
                        mbar_spin(&sm.qempty[slot], ((ord / kQSlots) - 1) & 1, abort, a.err);
                        if (MODE != kFull) mbar_spin(&sm.qempty2[slot], ((ord / kQSlots) - 1) & 1, abort, a.err);
                    }
                    mbar_expect_tx(&sm.qfull[slot], 2 * kBoxBytes);
                    tma_load_2d(sm.q[slot], &a.tmap_q, &sm.qfull[slot], 0, u * kQRows);
                    tma_load_2d(sm.q[slot] + kBoxBytes, &a.tmap_q, &sm.qfull[slot], 64, u * kQRows);
                }
                if (ph == 0) {
                    const int st = i % kRing;
                    mbar_spin(&sm.emptyA[st], ((i / kRing) & 1) ^ 1, abort, a.err);
                    mbar_expect_tx(&sm.fullA[st], 2 * kBoxBytes);
                    tma_load_4d(&sm.ringA[0][0] + (size_t)2 * st * kBoxBytes, mk, &sm.fullA[st], 0, ti * kTileKeys, 0, u);
                    *reinterpret_cast<volatile int*>(&sm.p1_issued) = i + 1;
                } else {
                    const int k = 2 * i + hh, st = k % kStagesB;
                    mbar_spin(&sm.emptyB[st], ((k / kStagesB) & 1) ^ 1, abort, a.err);
                    mbar_expect_tx(&sm.fullB[st], kBoxBytes);
                    tma_load_3d_hint(sm.ringB[st], mk, &sm.fullB[st], 64 * hh, ti * kTileKeys, u, evict_first);
                    if (hh == 0) *reinterpret_cast<volatile int*>(&sm.p2_issued) = i + 1;
                }
            }
            if (*abort) {
                // copies still in flight land before the CTA exits
                if (ph == 0) {
                    for (int n = std::max(0, i - kRing); n < i; ++n)
                        drain_wait(&sm.fullA[n % kRing], (n / kRing) & 1, a.err);
                    for (int o = std::max(0, ord - kQSlots + 1); o <= ord; ++o)
                        drain_wait(&sm.qfull[o % kQSlots], (o / kQSlots) & 1, a.err);
                } else {
                    for (int n = std::max(0, i - 2); n < i; ++n) {
                        const int k = 2 * n + hh;
                        drain_wait(&sm.fullB[k % kStagesB], (k / kStagesB) & 1, a.err);
                    }
                }
            }
        }
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------------------ MMA issuers
        // Warp 1 issues the phase-1 jobs, warp 3 the phase-2 jobs (a phase-2 tile once its
        // unit's lse is in shared memory).  Each claims the next job number n when its job is
        // ready and fills accumulator n % kAcc, so the consumers see one stream of jobs.  Two
        // issuers keep the tensor pipe busy while either does its bookkeeping.  kStats has only
        // phase-1 jobs, kScores only phase-2 jobs: there both warps issue the one phase,
        // warp 1 the even and warp 3 the odd local tiles (a single issuer was the slower side
        // of those launches), and each releases the Q slots through its own barriers.
        const int ph = MODE == kFull ? (warp == 1 ? 0 : 1) : (MODE == kStats ? 0 : 1);
        const int parity = warp == 1 ? 0 : 1;  // single-phase launches: the local tiles this warp issues
        uint64_t* qrelease = MODE != kFull && warp == 3 ? sm.qempty2 : sm.qempty;
        if (lane == 0) {
            const uint64_t dK0 = sw128_desc(smem_u32(ph == 0 ? sm.ringA[0] : sm.ringB[0]));
            const uint64_t dQ0 = sw128_desc(smem_u32(sm.q[0]));
            constexpr uint64_t kBoxStep = kBoxBytes >> 4, kQStep = (2 * kBoxBytes) >> 4;
            int u = cta / a.T_u, t = cta - (cta / a.T_u) * a.T_u;  // unit and tile of local tile i
            int ord = 0, qslot = 0;                                 // unit ordinal, its Q slot
            int s = 0;
            uint32_t sph = 0;  // phase-2 ring stage and phase
            bool have_q = false;
            for (int i = 0; i < n_local && !*abort; ++i) {
                if (MODE == kFull || (i & 1) == parity) {
                    if (!have_q) {
                        // the unit's Q (its slot is not refilled before phase 2 releases it)
                        mbar_spin(&sm.qfull[qslot], (ord / kQSlots) & 1, abort, a.err);
                        have_q = true;
                    }
                    // phase 2 of a tile waits until its unit's lse is in shared memory
                    if (ph == 1) mbar_spin(&sm.lsefull[ord & 1], (ord >> 1) & 1, abort, a.err);
                    if (ph == 0 || MODE == kScores)
                        mbar_spin(&sm.fullA[i % kRing], (i / kRing) & 1, abort, a.err);
                    else
                        mbar_spin(&sm.fullB[s], sph, abort, a.err);
                    const int n = atomicAdd(&sm.next_job, 1);
                    const int slot = n % kAcc;
                    // Accumulators are taken in job order: job n waits for the release of job
                    // n - kAcc only after job n - 1 has taken its own, so that the accumulator's
                    // barrier is never two phases behind this wait (a parity wait would pass).
                    spin_until_at_least(&sm.jobs_started, n, abort, a.err);
                    mbar_spin(&sm.accempty[slot], ((n / kAcc) & 1) ^ 1, abort, a.err);
                    tc_fence_after();
                    *reinterpret_cast<volatile int*>(&sm.jobs_started) = n + 1;
                    sm.job[slot] = make_int4(ph, u, t, ph == 0 ? i : (ord & 1));
                    mbar_arrive(&sm.accfull[slot]);
                    const uint32_t d = tmem + slot * 128;
                    const uint64_t dq = dQ0 + (uint64_t)qslot * kQStep;
                    if (ph == 0) {
                        // both halves of the tile arrived with one op
                        const int st = i % kRing;
                        const uint64_t dk = dK0 + (uint64_t)(2 * st) * kBoxStep;
                        umma_half(d, dq, dk, 0);
                        umma_half(d, dq + kBoxStep, dk + kBoxStep, 1);
                        umma_commit(&sm.emptyA[st]);
                    } else if (MODE == kScores) {
                        // phase 2 alone: the tile came through the phase-1 ring
                        const int st = i % kRing;
                        const uint64_t dk = sw128_desc(smem_u32(sm.ringA[0])) + (uint64_t)(2 * st) * kBoxStep;
                        tc_fence_after();
                        umma_half(d, dk, dq, 0);
                        umma_half(d, dk + kBoxStep, dq + kBoxStep, 1);
                        umma_commit(&sm.emptyA[st]);
                    } else {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (h == 1) mbar_spin(&sm.fullB[s], sph, abort, a.err);
                            tc_fence_after();
                            const uint64_t dk = dK0 + (uint64_t)s * kBoxStep;
                            umma_half(d, dk, dq + h * kBoxStep, h);
                            umma_commit(&sm.emptyB[s]);
                            if (++s == kStagesB) {
                                s = 0;
                                sph ^= 1u;
                            }
                        }
                    }
                    umma_commit(&sm.accfull[slot]);
                }
                // next tile; a new unit moves to the next Q slot (phase 2 releases the old one)
                t += P;
                int nu = u;
                while (t >= a.T_u) {
                    t -= a.T_u;
                    ++nu;
                }
                if (nu != u) {
                    // the last phase that reads the unit's Q releases its slot
                    if ((ph == 1 || MODE == kStats) && i + 1 < n_local) umma_commit(&qrelease[qslot]);
                    u = nu;
                    ++ord;
                    if (++qslot == kQSlots) qslot = 0;
                    have_q = false;
                }
            }
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------ lse of each unit
        // lane l handles query rows l, l + 32, l + 64, l + 96
        int cur = -1, ord = -1;
        unsigned target[2] = {0u, 0u};
        bool gave_up = false;
        const unsigned n_contrib = (unsigned)min(a.T_u, a.P);
        for (int i = 0; i < n_local && !*abort; ++i) {
            const int u = seq.unit(i);
            if (u == cur) continue;
            cur = u;
            ++ord;
            const int slot = ord & 1;
            // every phase-2 job of the unit that used this slot before has read it
            if (MODE != kStats && lane == 0 &&
                *reinterpret_cast<volatile unsigned*>(&sm.lse_done[slot]) < target[slot]) {
                const long long t0 = globaltimer();
                while (*reinterpret_cast<volatile unsigned*>(&sm.lse_done[slot]) < target[slot]) {
                    if (*abort) break;
                    if (globaltimer() - t0 > kBarrierTimeoutNs) {
                        atomicOr(a.err, kErrTimeout);
                        *abort = 1;
                        break;
                    }
                }
            }
            target[slot] += 4u * (unsigned)seq.count(u);
            if (MODE == kScores) {
                // the normalisers come from the caller (every shard's, merged)
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int r = lane + 32 * rr;
                    const float lse = r < a.nq && dcheck_idx(a.err, u, a.U)
                                          ? __ldg(a.lse_in + (size_t)u * kQRows + r) : INFINITY;
                    sm.nlse[slot][r] = -lse;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.lsefull[slot]);
                continue;
            }
            // unit u is complete once every CTA holding tiles of it has added its part
            int ok = 0;
            if (lane == 0) {
                const unsigned* cnt = a.inject ? a.never : a.count + u;
                bool done = ld_acquire(cnt) >= n_contrib;
                for (long long spins = 0; !done && !gave_up && spins < a.spin_limit && !*abort; ++spins) {
                    __nanosleep(32);
                    done = ld_acquire(cnt) >= n_contrib;
                }
                if (!done) {
                    atomicOr(a.err, kErrTimeout);
                    gave_up = true;  // later units do not wait again
                }
                ok = done;
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();
            // the unit's total per row: the copies added in a fixed order
            double tot[4] = {0.0, 0.0, 0.0, 0.0}, tott[4] = {0.0, 0.0, 0.0, 0.0};
            const double* su = a.sum + (size_t)u * kSumCopies * kQRows;
            const double* st = a.sum_t + (size_t)u * kSumCopies * kQRows;
#pragma unroll
            for (int c = 0; c < kSumCopies; ++c)
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    tot[rr] += __ldcg(su + c * kQRows + lane + 32 * rr);
                    if (ENT) tott[rr] += __ldcg(st + c * kQRows + lane + 32 * rr);
                }
            if (ENT && ok) {
                // entropy (nats) = ln2 (lse - E[y]) = ln2 (log2 total - E[y - ref])
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int r = lane + 32 * rr;
                    if (r < a.nq && tot[rr] > 0.0 && dcheck_idx(a.err, u, a.U))
                        a.entropy[(size_t)u * a.nq + r] =
                            (float)(0.69314718055994531 * ((double)log2_pos(tot[rr]) - tott[rr] / tot[rr]));
                }
            }
            if (MODE == kStats) {
                // this block's part of each row's normaliser as (m, l) with l in [1, 2):
                // total 2^ref = l 2^m; every CTA of the unit writes the same values
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int r = lane + 32 * rr;
                    if (r >= a.nq) continue;
                    float2 ml = make_float2(-INFINITY, 0.f);
                    if (ok && tot[rr] > 0.0) {
                        const long long b = __double_as_longlong(tot[rr]);
                        const int e = (int)((b >> 52) & 0x7FF) - 1023;
                        const double f = __longlong_as_double((b & ~(0x7FFLL << 52)) | (1023LL << 52));
                        ml = make_float2(__ldg(a.ref + (size_t)u * kQRows + r) + (float)e, (float)f);
                    }
                    if (dcheck_idx(a.err, u, a.U)) a.ml_out[(size_t)u * a.nq + r] = ml;
                }
                continue;
            }
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = lane + 32 * rr;
                // the total is >= ~1: it holds the row's own-position key, whose logit is ref
                sm.nlse[slot][r] = (ok && r < a.nq && tot[rr] > 0.0)
                                       ? -(__ldg(a.ref + (size_t)u * kQRows + r) + log2_pos(tot[rr]))
                                       : -INFINITY;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.lsefull[slot]);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ publisher
        // lane l holds query rows l + 32 k; adds the phase-1 tile records to the CTA's part of
        // each unit's total relative to the row's reference logit, in fp64: a record (d, l)
        // with d = m - ref adds l 2^d, which is l itself unless the tile moved the reference
        // (so the common case needs no exponential), and the part goes to the unit's total
        // after the CTA's last tile of the unit
        double L[4] = {0.0, 0.0, 0.0, 0.0}, T[4] = {0.0, 0.0, 0.0, 0.0};
        int u = cta / a.T_u, t = cta - (cta / a.T_u) * a.T_u;
        for (int i = 0; i < (MODE == kScores ? 0 : n_local); ++i) {
            const int s = i % kRec;
            mbar_wait(&sm.recfull[s], (i / kRec) & 1, abort, a.err);
            if (*abort) break;
            float2 v[4];
            float vt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[k] = sm.rec[s][lane + 32 * k];
                if (ENT) vt[k] = sm.rec_t[s][lane + 32 * k];
            }
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                *reinterpret_cast<volatile int*>(&sm.rec_consumed) = i + 1;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float d = v[k].x;
                L[k] += d == 0.f ? (double)v[k].y : scale_exp2(v[k].y, d);
                // sum of 2^(y - ref) (y - ref) = 2^d (t + d l)
                if (ENT) T[k] += d == 0.f ? (double)vt[k] : scale_exp2(fmaf(d, v[k].y, vt[k]), d);
            }
            t += P;
            int nu = u;
            while (t >= a.T_u) {
                t -= a.T_u;
                ++nu;
            }
            if (nu == u && i + 1 < n_local) continue;
            // last tile of unit u on this CTA
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const size_t at = ((size_t)u * kSumCopies + cta % kSumCopies) * kQRows + lane + 32 * k;
                if (L[k] != 0.0) atomicAdd(a.sum + at, L[k]);
                if (ENT && T[k] != 0.0) atomicAdd(a.sum_t + at, T[k]);
                L[k] = 0.0;
                T[k] = 0.0;
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(a.count + u, 1u);
            u = nu;
        }
    } else if (warp >= kConsumer0) {
        // ------------------------------------------------------------ consumers
        // warpgroup g drains accumulator g: jobs g, g + kAcc, ...; thread = TMEM lane, i.e.
        // a query row for phase-1 jobs and a key of the tile for phase-2 jobs
        const int g = (warp - kConsumer0) >> 2;
        const int r = threadIdx.x - 32 * kConsumer0 - 128 * g;
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + g * 128;
        const int n_jobs = MODE == kFull ? 2 * n_local : n_local;
        // the last local key index row q sees is min(N - 1, hz0 + q % w) (sharding: a key's
        // position is key_off + its local index; row q sits at n_total - w + q % w)
        const int hz0 = a.n_total - a.w - a.key_off;
        for (int n = g; n < n_jobs; n += kAcc) {
            mbar_wait(&sm.accfull[g], (n / kAcc) & 1, abort, a.err);
            if (*abort) break;
            tc_fence_after();
            int4 jb;
            asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(jb.x), "=r"(jb.y), "=r"(jb.z), "=r"(jb.w)
                         : "r"(smem_u32(&sm.job[g]))
                         : "memory");
            const int u = jb.y, ti = jb.z;
            const bool full_tile = (ti + 1) * kTileKeys <= min(a.N, a.n_total - a.w - a.key_off + 1);
            if (jb.x == 0) {
                // phase 1: this row's (m, sum of 2^(y - m)) over the tile's visible keys.  m is
                // the row's reference logit (its own-position key), so no running max is
                // needed; a chunk whose sum is not below 2^100 (a logit ~100 above the
                // reference) is redone with its exact max.
                const int t_r = min(a.N - 1, hz0 + r % a.w);  // last key this row sees
                const float ref = __ldg(a.ref + (size_t)u * kQRows + r);
                float m = ref, l = 0.f, t = 0.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t x[32];
                    __syncwarp();
                    tmem_ld32(tl + c * 32, x);
                    tmem_wait32(x);
                    if (c == 3) {
                        // the accumulator can take the next job once it is in registers
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.accempty[g]);
                    }
                    if (!full_tile) {
                        const int j0 = ti * kTileKeys + c * 32;
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j0 + e > t_r) x[e] = __float_as_uint(kMasked);
                    }
                    float ct = 0.f;
                    const float cs = sum_exp2_shifted<ENT>(x, m, ct);
                    if (cs < 0x1p100f) {
                        l += cs;
                        if (ENT) t += ct;
                    } else {
                        // move the reference to the chunk's max: sums scale by 2^(m - mn), each
                        // y - m shifts by m - mn
                        const float mn = fmaxf(m, chunk_max(x) * kLog2eOverSqrtD);
                        const float f = ex2(m - mn);
                        if (ENT) t = f * (t + (m - mn) * l);
                        l = l * f + sum_exp2_shifted<ENT>(x, mn, ct);
                        if (ENT) t += ct;
                        m = mn;
                    }
                }
                // record slot i % kRec is free once the publisher has read record i - kRec
                const int i = jb.w, s = i % kRec;
                if (lane == 0) spin_until_at_least(&sm.rec_consumed, i - kRec + 1, abort, a.err);
                __syncwarp();
                sm.rec[s][r] = make_float2(m - ref, l);  // 0 unless a chunk moved the reference
                if (ENT) sm.rec_t[s][r] = t;
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.recfull[s]);
            } else {
                // phase 2: this key's sum over the query rows of 2^(y - lse)
                const float* nlse = sm.nlse[jb.w];
                const int j = ti * kTileKeys + r;
                float sc = 0.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t x[32];
                    __syncwarp();
                    tmem_ld32(tl + c * 32, x);
                    tmem_wait32(x);
                    if (c == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.accempty[g]);
                    }
                    if (!full_tile) {
                        // query row q (position N - w + q % w) sees this key iff j <= that
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j > min(a.N - 1, hz0 + (c * 32 + e) % a.w)) x[e] = __float_as_uint(-INFINITY);
                    }
                    sc += prob_sum(x, nlse + c * 32);
                }
                if (j < a.N && dcheck_idx(a.err, u, a.U)) a.unit_scores[(size_t)u * a.N + j] = sc;
                __syncwarp();
                if (lane == 0) atomicAdd(&sm.lse_done[jb.w], 1u);
            }
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

// Copies the unit's query rows into a zero-padded [U][128][128] block (rows >= nq are 0),
// computes each row's reference logit (base 2) with the key at the row's own position, and
// clears the per-unit sums and counters of this call.
__global__ void tc_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                               __nv_bfloat16* __restrict__ qpad, float* __restrict__ ref, double* __restrict__ sum,
                               unsigned* __restrict__ flags, int n_flags, int U, int N, int w, int nq, int mode,
                               int key_off, int n_total, unsigned* err) {
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
    // one warp per (unit, row): lane l takes dimensions 4l .. 4l + 3 (8-byte loads), then a
    // butterfly sum
    const int lane = threadIdx.x & 31;
    const long long n_warps = (long long)gridDim.x * blockDim.x / 32;
    for (long long e = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / 32; e < (long long)U * kQRows;
         e += n_warps) {
        const int r = (int)(e % kQRows);
        const long long u = e / kQRows;
        // The reference logit.  kFull: the key at the row's own position.  kStats (the block
        // may not hold the row's own position): the largest logit over kRefSamples keys spread
        // evenly over the ones the row sees, so that the phase-1 sums rarely have to move
        // their reference.  Rows that see no key of the block keep 0 (their sums stay 0).
        const int t_r = mode == kFull ? N - w + r % w : min(N - 1, n_total - w + r % w - key_off);
        const bool has_ref = r < nq && (mode == kFull || (mode == kStats && t_r >= 0));
        const int n_s = mode == kFull ? 1 : kRefSamples;
        float best = -INFINITY;
        if (has_ref) {
            // all the samples' loads first, then the dot products (one round of load latency)
            const uint2 qv = *reinterpret_cast<const uint2*>(q + (u * nq + r) * kHeadDim + 4 * lane);
            const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(&qv);
            uint2 kv[kRefSamples];
#pragma unroll
            for (int si = 0; si < kRefSamples; ++si) {
                const int kj = mode == kFull ? t_r : (int)((long long)si * t_r / (kRefSamples - 1));
                const bool use = si < n_s && dcheck(err, kj >= 0 && kj < N);
                kv[si] = use ? *reinterpret_cast<const uint2*>(k + (u * N + kj) * kHeadDim + 4 * lane)
                             : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int si = 0; si < kRefSamples; ++si) {
                if (si >= n_s) break;
                const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&kv[si]);
                float x = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float2 qf = __bfloat1622float2(qh[h]), kf = __bfloat1622float2(kh[h]);
                    x = fmaf(qf.x, kf.x, x);
                    x = fmaf(qf.y, kf.y, x);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                best = fmaxf(best, x);
            }
        }
        if (lane == 0) ref[e] = has_ref ? best * kLog2eOverSqrtD : 0.f;
    }
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < 2LL * U * kSumCopies * kQRows;
         e += (long long)gridDim.x * blockDim.x)
        sum[e] = 0.0;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_flags;
         e += (long long)gridDim.x * blockDim.x)
        flags[e] = 0u;
}

// Each row's log-sum-exp (base 2) from every shard's (m, l) (l 2^m = the shard's sum of 2^y
// over its keys), merged in shard order so that every shard computes the same value:
// ml_all [W][U][nq] -> lse [U][128] (rows >= nq: +inf).
__global__ void tc_shard_lse_kernel(const float2* __restrict__ ml_all, int W, int U, int nq, float* __restrict__ lse) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < U * kQRows; i += gridDim.x * blockDim.x) {
        const int u = i / kQRows, r = i % kQRows;
        if (r >= nq) {
            lse[i] = INFINITY;
            continue;
        }
        const size_t rows = (size_t)U * nq, at = (size_t)u * nq + r;
        float M = -INFINITY;
        for (int s = 0; s < W; ++s) M = fmaxf(M, ml_all[s * rows + at].x);
        float S = 0.f;
        for (int s = 0; s < W; ++s) {
            const float2 v = ml_all[s * rows + at];
            if (v.x != -INFINITY) S += v.y * exp2f(v.x - M);
        }
        lse[i] = M + log2f(S);
    }
}

// ------------------------------------------------------------------------ host side

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

struct TcLayout {
    size_t qpad, ref, sum, lse, flags, n_flags, total;
};

TcLayout tc_layout(int U) {
    TcLayout L;
    size_t off = 0;
    L.qpad = off;
    off = a256(off + (size_t)U * kQRows * kHeadDim * 2);
    L.ref = off;
    off = a256(off + (size_t)U * kQRows * sizeof(float));
    L.sum = off;  // the totals, then the entropy's totals
    off = a256(off + 2 * (size_t)U * kSumCopies * kQRows * sizeof(double));
    L.lse = off;  // kScores: the merged log-sum-exp per (unit, padded row)
    off = a256(off + (size_t)U * kQRows * sizeof(float));
    L.flags = off;  // count[U], never
    L.n_flags = (size_t)U + 1;
    off = a256(off + L.n_flags * sizeof(unsigned));
    L.total = off;
    return L;
}

}  // namespace

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
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < 64 && cache[dev].load()) return cache[dev].load();
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 64) cache[dev].store(n);
    return n;
}

bool tc_score_supported(const ScoreJob& j) {
    return j.dtype == KVC_BF16 && j.nq >= 1 && j.nq <= kQRows && j.N >= 1 && j.U >= 1 &&
           (long long)j.U * kQRows < (1LL << 31);
}

size_t tc_score_workspace(int U, int /*N*/, int /*nq*/) { return tc_layout(U).total; }

namespace {

template <int MODE>
cudaError_t launch_kernel(const TcArgs& a, bool ent, size_t smem, cudaStream_t s) {
    static std::atomic<bool> attr_set[2][64];
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev >= 64 || !attr_set[ent][dev].load()) {
        e = ent ? cudaFuncSetAttribute(tc_score_kernel<true, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                : cudaFuncSetAttribute(tc_score_kernel<false, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[ent][dev].store(true);
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
    e = ent ? cudaLaunchKernelEx(&cfg, tc_score_kernel<true, MODE>, a)
            : cudaLaunchKernelEx(&cfg, tc_score_kernel<false, MODE>, a);
    count_launches(1);
    return e;
}

// The prep kernel and one launch of the score kernel in the given mode.
cudaError_t tc_launch(const ScoreJob& j, int mode, float2* ml_out, cudaStream_t s) {
    const TcLayout L = tc_layout(j.U);
    char* ws = (char*)j.tc_ws;
    if (j.tc_ws_bytes < L.total) return cudaErrorInvalidValue;
    __nv_bfloat16* qpad = (__nv_bfloat16*)(ws + L.qpad);
    unsigned* flags = (unsigned*)(ws + L.flags);

    TcArgs a{};
    a.unit_scores = j.unit_scores;
    a.ref = (const float*)(ws + L.ref);
    a.sum = (double*)(ws + L.sum);
    a.sum_t = a.sum + (size_t)j.U * kSumCopies * kQRows;
    a.entropy = j.entropy;
    a.count = flags;
    a.never = flags + j.U;
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
    a.P = std::min(std::min(n_sm, kMaxCtas), a.total_tiles);
    // phase 1 may run this many tiles ahead of phase 2: a unit's worth plus slack for the
    // merge, while keeping the tiles between the two reads (max_lead x P x 32 KiB) in L2
    a.max_lead = (a.T_u + a.P - 1) / a.P + kLeadSlack;
    a.inject = j.inject_timeout;
    a.key_off = j.key_off;
    a.n_total = j.n_total > 0 ? j.n_total : j.N;
    a.ml_out = ml_out;
    a.lse_in = (const float*)(ws + L.lse);
    if (mode != kFull && j.entropy) return cudaErrorInvalidValue;

    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    {
        // K as [U][2 halves][N][64]: a box of 64 x 128 x 2 lands the tile's two 64-column halves
        // one after the other, each in the 128-byte-swizzled layout the MMA reads
        cuuint64_t dims4[4] = {64, (cuuint64_t)j.N, 2, (cuuint64_t)j.U};
        cuuint64_t strides4[3] = {(cuuint64_t)kHeadDim * 2, 128, (cuuint64_t)j.N * kHeadDim * 2};
        cuuint32_t box4[4] = {64, kTileKeys, 2, 1};
        cuuint32_t estr4[4] = {1, 1, 1, 1};
        if (encode(&a.tmap_k4, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(j.k), dims4, strides4, box4,
                   estr4, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
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
    tc_prep_kernel<<<prep_grid, 256, 0, s>>>((const __nv_bfloat16*)j.q, (const __nv_bfloat16*)j.k, qpad,
                                             (float*)(ws + L.ref), (double*)(ws + L.sum), flags, (int)L.n_flags,
                                             j.U, j.N, j.window, j.nq, mode, a.key_off, a.n_total, j.err);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const size_t smem = sizeof(Smem) + 1024;
    const bool ent = j.entropy != nullptr;
    if (mode == kStats) return launch_kernel<kStats>(a, false, smem, s);
    if (mode == kScores) return launch_kernel<kScores>(a, false, smem, s);
    return launch_kernel<kFull>(a, ent, smem, s);
}

}  // namespace

cudaError_t tc_score(const ScoreJob& j, cudaStream_t s) { return tc_launch(j, kFull, nullptr, s); }

cudaError_t tc_shard_stats(const ScoreJob& j, float2* ml, cudaStream_t s) { return tc_launch(j, kStats, ml, s); }

cudaError_t tc_shard_scores(const ScoreJob& j, const float2* ml_all, int W, cudaStream_t s) {
    const TcLayout L = tc_layout(j.U);
    if (j.tc_ws_bytes < L.total) return cudaErrorInvalidValue;
    const long long n = (long long)j.U * kQRows;
    tc_shard_lse_kernel<<<(int)std::min<long long>((n + 255) / 256, 148LL * 8), 256, 0, s>>>(
        ml_all, W, j.U, j.nq, (float*)((char*)j.tc_ws + L.lse));
    count_launches(1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return tc_launch(j, kScores, nullptr, s);
}

}  // namespace kvc

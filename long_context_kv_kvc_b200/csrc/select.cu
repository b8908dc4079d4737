// select.cu -- score sums, 1-D max-pool and top-k selection of kept positions.
//
// Top-k is a radix select on order-preserving 32-bit keys of the pooled fp32 scores,
// followed by a stable compaction that writes the kept candidate positions in ascending
// order: every candidate above the threshold value T, and the lowest-indexed candidates
// equal to T up to the budget.  Sinks [0, S) and the recent window [N - w, N) are written
// around them (CentroidKV page, "Inferentie Pipeline": sinks and recent tokens are
// preserved; FastKV page, sec. 2A: the selected tokens plus a window of the newest tokens).
// Two kernels:
//   * topk_cluster_kernel (the compress path's default): one 8-CTA cluster per row; each
//     CTA max-pools its slice of the candidates into shared memory (counting the first
//     digit's histogram as it forms the keys), and the cluster runs an 11/11/10-bit radix
//     select whose per-CTA histograms are combined through distributed shared memory;
//   * topk_kernel (rows too long for the clusters' shared memory): one CTA of 1024 threads
//     per row, four 8-bit digits; each warp owns a contiguous segment of the row, so all
//     loads are coalesced and the only block-wide steps are the digit search and one scan
//     of per-warp counts.
#include <cooperative_groups.h>

#include <atomic>

#include "kvc_internal.cuh"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

// ------------------------------------------------------------------------------- sums

__global__ void reduce_units_kernel(const float* __restrict__ units, int L, int B, int Hkv, int N,
                                    int all_heads, float* __restrict__ out, unsigned* err) {
    const long long n_units = (long long)L * B * Hkv * N;
    const int Hs = all_heads ? 1 : Hkv;
    const long long total = (long long)B * Hs * N;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(e % N);
        const long long bh = e / N;
        const int hs = (int)(bh % Hs);
        const int b = (int)(bh / Hs);
        const int h0 = all_heads ? 0 : hs, h1 = all_heads ? Hkv : hs + 1;
        float s = 0.f;
        for (int l = 0; l < L; ++l)
            for (int h = h0; h < h1; ++h) {
                const long long i = (((long long)l * B + b) * Hkv + h) * N + j;
                if (dcheck_idx(err, i, n_units)) s += units[i];
            }
        out[e] = s;
    }
}

__global__ void accumulate_kernel(float* __restrict__ acc, const float* __restrict__ src, int B,
                                  int Hi, int Ho, int N, unsigned* err) {
    const int R = Hi / Ho;
    const long long n_src = (long long)B * Hi * N;
    const long long total = (long long)B * Ho * N;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(e % N);
        const long long bo = e / N;
        const int o = (int)(bo % Ho);
        const int b = (int)(bo / Ho);
        float s = acc[e];
        for (int r = 0; r < R; ++r) {
            const long long i = ((long long)b * Hi + o * R + r) * N + j;
            if (dcheck_idx(err, i, n_src)) s += src[i];
        }
        acc[e] = s;
    }
}

// ------------------------------------------------------------------------------- pool

__global__ void pool_kernel(const float* __restrict__ in, float* __restrict__ out, int rows, int N,
                            int lo, int hi, int radius, unsigned* err) {
    const long long total = (long long)rows * N;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(e % N);
        const float* r = in + (e - j);
        float m;
        if (j < lo || j >= hi) {
            m = r[j];
        } else {
            const int t0 = max(lo, j - radius), t1 = min(hi - 1, j + radius);
            // the clipped window stays inside the row's candidates
            if (!dcheck(err, t0 >= 0 && t0 <= j && j <= t1 && t1 < N)) continue;
            m = r[t0];
            for (int t = t0 + 1; t <= t1; ++t) m = fmaxf(m, r[t]);
        }
        out[e] = m;
    }
}

// ------------------------------------------------------------------------------- top-k

constexpr int kTopkThreads = 1024;
constexpr int kWarps = kTopkThreads / 32;

// Monotone map from fp32 to uint32 (larger value -> larger key); -0.0 maps like +0.0.
__device__ __forceinline__ uint32_t order_key(float v) {
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ pooled, int N, int S, int w, int budget,
            int32_t* __restrict__ idx, unsigned* err) {
    __shared__ unsigned hist[kWarps][256];
    __shared__ unsigned wsum[8];
    __shared__ uint32_t s_prefix;
    __shared__ int s_krem;
    __shared__ int wcnt_gt[kWarps], wcnt_eq[kWarps];

    const int row = blockIdx.x;
    const float* v = pooled + (size_t)row * N;
    int32_t* out = idx + (size_t)row * budget;
    const int lo = S, hi = N - w, k_sel = budget - S - w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // warp `warp` owns candidates [seg0, seg1)
    const int n_c = hi - lo;
    const int seg = (n_c + kWarps - 1) / kWarps;
    const int seg0 = lo + min(n_c, warp * seg), seg1 = lo + min(n_c, (warp + 1) * seg);

    // sinks fill [0, S), the window [budget - w, budget); the selected go between them
    for (int i = tid; i < S; i += kTopkThreads)
        if (dcheck(err, i < budget - w)) out[i] = i;
    for (int i = tid; i < w; i += kTopkThreads)
        if (dcheck(err, budget - w + i >= S)) out[budget - w + i] = N - w + i;

    if (tid == 0) {
        s_prefix = 0u;
        s_krem = k_sel;
    }
    uint32_t prefix = 0, mask = 0;
    int krem = k_sel;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < kWarps * 256; i += kTopkThreads) (&hist[0][0])[i] = 0u;
        __syncthreads();
        for (int j = seg0 + lane; j < seg1; j += 32) {
            const uint32_t key = order_key(v[j]);
            if ((key & mask) == prefix) {
                const unsigned digit = (key >> shift) & 255u;
                const unsigned peers = __match_any_sync(__activemask(), digit);
                if (lane == __ffs(peers) - 1) atomicAdd(&hist[warp][digit], (unsigned)__popc(peers));
            }
        }
        __syncthreads();
        // bins are scanned from the top: incl(d) = #keys with digit >= d
        unsigned incl = 0, tot = 0;
        if (tid < 256) {
            for (int wi = 0; wi < kWarps; ++wi) tot += hist[wi][tid];
            incl = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned y = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += y;
            }
            if (lane == 0) wsum[warp] = incl;
        }
        __syncthreads();
        if (tid < 256) {
            for (int wi = warp + 1; wi < 8; ++wi) incl += wsum[wi];
            const unsigned excl = incl - tot;
            if (excl < (unsigned)krem && (unsigned)krem <= incl) {
                s_prefix = prefix | ((uint32_t)tid << shift);
                s_krem = krem - (int)excl;
            }
        }
        __syncthreads();
        prefix = s_prefix;
        krem = s_krem;
        mask |= 255u << shift;
    }
    const uint32_t T = prefix;  // the k_sel-th largest key; take krem of the keys equal to T

    // counts per warp segment
    int n_gt = 0, n_eq = 0;
    for (int j = seg0 + lane; j < seg1; j += 32) {
        const uint32_t key = order_key(v[j]);
        n_gt += key > T;
        n_eq += key == T;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        n_gt += __shfl_xor_sync(0xffffffffu, n_gt, off);
        n_eq += __shfl_xor_sync(0xffffffffu, n_eq, off);
    }
    if (lane == 0) {
        wcnt_gt[warp] = n_gt;
        wcnt_eq[warp] = n_eq;
    }
    __syncthreads();
    int gt_before = 0, eq_before = 0;
    for (int wi = 0; wi < warp; ++wi) {
        gt_before += wcnt_gt[wi];
        eq_before += wcnt_eq[wi];
    }
    // stable compaction in position order
    int taken = gt_before + min(eq_before, krem);
    int eq_seen = eq_before;
    for (int base = seg0; base < seg1; base += 32) {
        const int j = base + lane;
        const uint32_t key = j < seg1 ? order_key(v[j]) : 0u;
        const bool gt = j < seg1 && key > T;
        const bool eq = j < seg1 && key == T;
        const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eq_mask & lanemask_lt()) < krem);
        const unsigned take_mask = __ballot_sync(0xffffffffu, take);
        const int pos = taken + __popc(take_mask & lanemask_lt());
        if (take && dcheck(err, pos < k_sel && j >= lo && j < hi)) out[S + pos] = j;
        taken += __popc(take_mask);
        eq_seen += __popc(eq_mask);
    }
    // the last warp's running count is the row's: exactly k_sel were written
    if (warp == kWarps - 1 && lane == 0) dcheck(err, taken == k_sel);
}

// --------------------------------------------------------------- cluster top-k (fused pool)
//
// One 8-CTA thread-block cluster owns a row.  CTA k of the cluster pools the candidates
// [lo + k*seg, lo + (k+1)*seg) (reading the raw scores with their pool halo) into
// order-preserving keys in its shared memory; the radix select then runs three digit
// passes (11, 11 and 10 bits) over shared memory, combining the CTAs' histograms through
// distributed shared memory, and every CTA takes the same digit decision.  The stable
// compaction writes the kept positions in ascending order: CTA k starts after the
// candidates its lower-ranked siblings keep.

constexpr int kClusterCtas = 8;
constexpr int kCtThreads = 512;
constexpr int kCtWarps = kCtThreads / 32;
constexpr int kBins = 2048;
constexpr int kSegMax = 24576;  // keys per CTA: 96 KiB of shared memory (two CTAs per SM)

// Adds `n` keys of histogram bin `d` for each thread of the warp that holds a run (has):
// threads with the same bin combine their counts, one shared-memory atomic per bin.
__device__ __forceinline__ void hist_add_runs(uint32_t* hist, bool has, unsigned d, unsigned n, int lane) {
    if (!has) return;
    const unsigned peers = __match_any_sync(__activemask(), d);
    const unsigned sum = __reduce_add_sync(peers, n);
    if (lane == __ffs(peers) - 1) atomicAdd(&hist[d], sum);
}

// Counts digit (key >> shift) & dmask of the keys among k[0..7] that are valid and match
// the prefix, as runs of equal digits (neighbouring positions mostly share the leading
// digits): a run that ends is added directly, the last goes through hist_add_runs.
__device__ __forceinline__ void hist_count8(uint32_t* hist, const uint32_t (&k)[8], unsigned valid, uint32_t mask,
                                            uint32_t prefix, int shift, uint32_t dmask, int lane) {
    unsigned run_d = 0xffffffffu, run_n = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (!((valid >> i) & 1u) || (k[i] & mask) != prefix) continue;
        const unsigned d = (k[i] >> shift) & dmask;
        if (d != run_d) {
            if (run_n) atomicAdd(&hist[run_d], run_n);
            run_d = d;
            run_n = 0;
        }
        ++run_n;
    }
    hist_add_runs(hist, run_n > 0, run_d, run_n, lane);
}

struct TopkSmem {
    uint32_t hist[kBins];
    uint32_t slice_tot[kBins / kClusterCtas];  // this CTA's slice of the cluster-wide totals
    uint32_t slice_sum;
    int gt, eq;
    int wcnt_gt[kCtWarps], wcnt_eq[kCtWarps];
    alignas(16) uint32_t keys[kSegMax];  // slot x: the key of row position (s0 & ~3) + x (16-byte accesses)
};
constexpr int kSlotPad = 16;  // slots beyond a CTA's candidates: alignment to 4 and whole groups of 8
static_assert(offsetof(TopkSmem, keys) % 16 == 0, "16-byte key accesses");

// R >= 0: the pool radius, scores rows 16-byte aligned (vector loads); R = -1: any radius
// (scalar loads, runtime radius).
template <int R>
__global__ void __launch_bounds__(kCtThreads, 2) __cluster_dims__(kClusterCtas, 1, 1)
topk_cluster_kernel(const float* __restrict__ scores, int N, int S, int w, int budget, int radius, int seg,
                    int32_t* __restrict__ idx, unsigned* err) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.x / kClusterCtas;
    const float* v = scores + (size_t)row * N;
    int32_t* out = idx + (size_t)row * budget;
    const int lo = S, hi = N - w, k_sel = budget - S - w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s0 = lo + min(hi - lo, rank * seg), s1 = lo + min(hi - lo, (rank + 1) * seg);
    const int n_mine = s1 - s0;

    if (rank == 0) {
        for (int i = tid; i < S; i += kCtThreads)
            if (dcheck(err, i < budget - w)) out[i] = i;
        for (int i = tid; i < w; i += kCtThreads)
            if (dcheck(err, budget - w + i >= S)) out[budget - w + i] = N - w + i;
    }
    // Slot x of keys[] holds row position A0 + x, A0 = s0 rounded down to 4 (16-byte aligned
    // when the vector loads are used); this CTA's candidates are slots [off, off + n_mine).
    const int A0 = R >= 0 ? (s0 & ~3) : s0, off = s0 - A0, n_slots = off + n_mine;
    // this CTA's keys fit its shared memory
    if (tid == 0) dcheck(err, n_mine <= seg && seg + kSlotPad <= kSegMax);
    // pooled keys of this CTA's candidates (max over the clipped window of raw scores); the
    // first digit's histogram (the top 11 bits of every key) is counted as they are formed.
    // A thread forms 8 neighbouring keys at a time from 16 raw scores (positions p - 4 ..
    // p + 11, four 16-byte loads; outside [lo, hi) they count as -inf).
    for (int i = tid; i < kBins; i += kCtThreads) sm.hist[i] = 0u;
    __syncthreads();
    for (int x = 8 * tid; x < n_slots; x += 8 * kCtThreads) {
        const int p = A0 + x;
        uint32_t kk[8];
        if constexpr (R >= 0) {
            float r16[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const int q = p - 4 + 4 * q4;
                if (q >= lo && q + 3 < hi) {
                    const float4 f = __ldg(reinterpret_cast<const float4*>(v + q));
                    r16[4 * q4] = f.x;
                    r16[4 * q4 + 1] = f.y;
                    r16[4 * q4 + 2] = f.z;
                    r16[4 * q4 + 3] = f.w;
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        r16[4 * q4 + c] = (q + c >= lo && q + c < hi) ? __ldg(v + q + c) : -INFINITY;
                }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float m = r16[4 + k];
#pragma unroll
                for (int d = 1; d <= R; ++d) m = fmaxf(m, fmaxf(r16[4 + k - d], r16[4 + k + d]));
                kk[k] = order_key(m);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int j = min(max(p + k, lo), hi - 1);  // slots outside the candidates are never read
                const int t0 = max(lo, j - radius), t1 = min(hi - 1, j + radius);
                float m = 0.f;
                if (dcheck(err, t0 >= 0 && t0 <= j && j <= t1 && t1 < N)) {
                    m = __ldg(v + t0);
                    for (int t = t0 + 1; t <= t1; ++t) m = fmaxf(m, __ldg(v + t));
                }
                kk[k] = order_key(m);
            }
        }
        if (dcheck(err, x + 8 <= kSegMax)) {
            *reinterpret_cast<uint4*>(&sm.keys[x]) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
            *reinterpret_cast<uint4*>(&sm.keys[x + 4]) = make_uint4(kk[4], kk[5], kk[6], kk[7]);
        }
        unsigned valid = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) valid |= (x + k >= off && x + k < n_slots) ? 1u << k : 0u;
        hist_count8(sm.hist, kk, valid, 0u, 0u, 21, 0x7ffu, lane);
    }

    uint32_t prefix = 0, mask = 0;
    int krem = k_sel;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = shifts[pass];
        const uint32_t dmask = (1u << widths[pass]) - 1u;
        if (pass > 0) {  // the first pass's histogram was built with the keys
            for (int i = tid; i < kBins; i += kCtThreads) sm.hist[i] = 0u;
            __syncthreads();
            for (int x = 8 * tid; x < n_slots; x += 8 * kCtThreads) {
                const uint4 a4 = *reinterpret_cast<const uint4*>(&sm.keys[x]);
                const uint4 b4 = *reinterpret_cast<const uint4*>(&sm.keys[x + 4]);
                const uint32_t kk[8] = {a4.x, a4.y, a4.z, a4.w, b4.x, b4.y, b4.z, b4.w};
                unsigned valid = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) valid |= (x + k >= off && x + k < n_slots) ? 1u << k : 0u;
                hist_count8(sm.hist, kk, valid, mask, prefix, shift, dmask, lane);
            }
        }
        cluster.sync();  // every CTA's histogram is complete
        // this CTA totals the bins [rank*256, rank*256 + 256) over the cluster
        constexpr int kSlice = kBins / kClusterCtas;
        if (tid < kSlice) {
            const int bin = rank * kSlice + tid;
            uint32_t t = 0;
#pragma unroll
            for (int c = 0; c < kClusterCtas; ++c) t += cluster.map_shared_rank(sm.hist, c)[bin];
            sm.slice_tot[tid] = t;
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t t = 0;
            for (int i = lane; i < kSlice; i += 32) t += sm.slice_tot[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            if (lane == 0) sm.slice_sum = t;
        }
        cluster.sync();  // slice totals are visible cluster-wide
        // every CTA finds the same digit: the slice holding the krem-th largest, then the bin
        if (warp == 0) {
            uint32_t above = 0;
            int s_star = 0;
            for (int c = kClusterCtas - 1; c >= 0; --c) {
                const uint32_t t = *cluster.map_shared_rank(&sm.slice_sum, c);
                if (above + t >= (uint32_t)krem) {
                    s_star = c;
                    break;
                }
                above += t;
            }
            const uint32_t* tot = cluster.map_shared_rank(sm.slice_tot, s_star);
            // scan the slice's 256 bins from the top, 32 at a time
            int digit = -1;
            for (int base = kSlice - 32; base >= 0 && digit < 0; base -= 32) {
                const uint32_t t = tot[base + lane];
                // inclusive suffix sum within this group of 32 (lane 31 is the top bin)
                uint32_t incl = t;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
                    if (lane + off < 32) incl += y;
                }
                const uint32_t excl = incl - t;
                const bool hit = above + excl < (uint32_t)krem && (uint32_t)krem <= above + incl;
                const unsigned b = __ballot_sync(0xffffffffu, hit);
                if (b) {
                    const int l = __ffs(b) - 1;
                    const uint32_t ex = __shfl_sync(0xffffffffu, excl, l);
                    digit = s_star * kSlice + base + l;
                    if (lane == 0) {
                        sm.gt = digit;
                        sm.eq = krem - (int)(above + ex);
                    }
                }
                above += __shfl_sync(0xffffffffu, incl, 0);
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sm.gt << shift;
        mask |= dmask << shift;
        krem = sm.eq;
        // (no cluster barrier here: every remote read of this pass -- the histograms before
        // the second barrier, the slice totals in the digit search -- ends before the readers
        // reach the next pass's first barrier, and only then are they overwritten)
    }
    const uint32_t T = prefix;  // the k_sel-th largest key; keep krem of the keys equal to T

    // per-warp counts over contiguous warp segments of this CTA's keys
    const int wseg = (n_mine + kCtWarps - 1) / kCtWarps;
    const int w0 = min(n_mine, warp * wseg), w1 = min(n_mine, (warp + 1) * wseg);
    int n_gt = 0, n_eq = 0;
    for (int e = w0 + lane; e < w1; e += 32) {
        const uint32_t key = sm.keys[e + off];
        n_gt += key > T;
        n_eq += key == T;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        n_gt += __shfl_xor_sync(0xffffffffu, n_gt, off);
        n_eq += __shfl_xor_sync(0xffffffffu, n_eq, off);
    }
    if (lane == 0) {
        sm.wcnt_gt[warp] = n_gt;
        sm.wcnt_eq[warp] = n_eq;
    }
    __syncthreads();
    if (tid == 0) {
        int g = 0, q = 0;
        for (int i = 0; i < kCtWarps; ++i) {
            g += sm.wcnt_gt[i];
            q += sm.wcnt_eq[i];
        }
        sm.gt = g;
        sm.eq = q;
    }
    cluster.sync();  // CTA totals visible
    int gt_before = 0, eq_before = 0;
    for (int c = 0; c < rank; ++c) {
        gt_before += *cluster.map_shared_rank(&sm.gt, c);
        eq_before += *cluster.map_shared_rank(&sm.eq, c);
    }
    for (int i = 0; i < warp; ++i) {
        gt_before += sm.wcnt_gt[i];
        eq_before += sm.wcnt_eq[i];
    }
    int taken = gt_before + min(eq_before, krem);
    int eq_seen = eq_before;
    for (int base = w0; base < w1; base += 32) {
        const int e = base + lane;
        const uint32_t key = e < w1 ? sm.keys[e + off] : 0u;
        const bool gt = e < w1 && key > T;
        const bool eq = e < w1 && key == T;
        const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eq_mask & lanemask_lt()) < krem);
        const unsigned take_mask = __ballot_sync(0xffffffffu, take);
        const int pos = taken + __popc(take_mask & lanemask_lt());
        if (take && dcheck(err, pos < k_sel && s0 + e >= lo && s0 + e < hi)) out[S + pos] = s0 + e;
        taken += __popc(take_mask);
        eq_seen += __popc(eq_mask);
    }
    // the last CTA's last warp ends at the row's count: exactly k_sel were written
    if (rank == kClusterCtas - 1 && warp == kCtWarps - 1 && lane == 0) dcheck(err, taken == k_sel);
    cluster.sync();  // siblings may still read this CTA's counts until here
}

// --------------------------------------------------------------- row statistics
//
// Two of the signals StructKV watches to find its pivot layer (StructKV page, sec. 2
// "Dynamische Pivot Detectie": sparsity and variance of the attention), per score row:
// the share of the row's mass held by its kept positions, and the population variance of
// the row over the candidates C = [S, N - w).  One CTA per row, fp64 partial sums in a
// fixed order (deterministic).

constexpr int kRsThreads = 1024;

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // red may still be read by a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < kRsThreads / 32; ++i) t += red[i];
    return t;
}

__global__ void __launch_bounds__(kRsThreads)
row_stats_kernel(const float* __restrict__ scores, int N, int S, int w, const int32_t* __restrict__ idx,
                 int budget, float* __restrict__ kept_mass, float* __restrict__ cand_var, unsigned* err) {
    __shared__ double red[kRsThreads / 32];
    const int row = blockIdx.x;
    const float* s = scores + (size_t)row * N;
    const int lo = S, hi = N - w;
    double tot = 0.0, csum = 0.0;
    for (int j = threadIdx.x; j < N; j += kRsThreads) {
        const double v = s[j];
        tot += v;
        if (j >= lo && j < hi) csum += v;
    }
    tot = block_sum(tot, red);
    csum = block_sum(csum, red);
    const double mean = csum / (hi - lo);
    double var = 0.0;
    for (int j = lo + threadIdx.x; j < hi; j += kRsThreads) {
        const double d = s[j] - mean;
        var += d * d;
    }
    var = block_sum(var, red);
    double kept = 0.0;
    if (idx) {
        for (int t = threadIdx.x; t < budget; t += kRsThreads) {
            const int j = idx[(size_t)row * budget + t];
            if (j >= 0 && j < N)
                kept += s[j];
            else
                atomicOr(err, kErrIndex);
        }
        kept = block_sum(kept, red);
    }
    if (threadIdx.x == 0) {
        cand_var[row] = (float)(var / (hi - lo));
        if (idx) kept_mass[row] = (float)(kept / tot);
    }
}

int grid_for(long long total, int threads) {
    long long g = (total + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (int)(g < 1 ? 1 : g);
}

// ------------------------------------------------------------------------ distributed select
// Sequence sharding splits a score row across GPUs; the radix select then runs digit by
// digit over all shards: each shard histograms the digit of its candidates that match the
// prefix found so far (the histograms are summed across shards), and once the threshold key
// is known each shard writes its candidates above it plus its share of the ties.

constexpr int kHistThreads = 256;
constexpr int kHistBlocksPerRow = 16;

// hist[row][d] += #candidates j in [lo, hi) of the row whose key's top prefix_bits equal
// prefix[row]'s and whose next digit_bits are d.
__global__ void __launch_bounds__(kHistThreads)
select_hist_kernel(const float* __restrict__ v, int n, int lo, int hi, const uint32_t* __restrict__ prefix,
                   int prefix_bits, int digit_bits, uint32_t* __restrict__ hist, unsigned* err) {
    extern __shared__ uint32_t h[];
    const int row = blockIdx.y, nb = 1 << digit_bits;
    for (int i = threadIdx.x; i < nb; i += kHistThreads) h[i] = 0u;
    __syncthreads();
    const uint32_t want = prefix[row];
    const int shift = 32 - prefix_bits - digit_bits;
    const float* vr = v + (size_t)row * n;
    const int span = (hi - lo + gridDim.x - 1) / gridDim.x;
    const int j0 = lo + blockIdx.x * span, j1 = min(hi, j0 + span);
    for (int j = j0 + threadIdx.x; j < j1; j += kHistThreads) {
        if (!dcheck(err, j >= 0 && j < n)) continue;
        const uint32_t key = order_key(vr[j]);
        const bool match = prefix_bits == 0 || (key >> (32 - prefix_bits)) == (want >> (32 - prefix_bits));
        if (match && dcheck(err, shift >= 0 && shift + digit_bits <= 32)) atomicAdd(&h[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += kHistThreads)
        if (h[i]) atomicAdd(&hist[(size_t)row * nb + i], h[i]);
}

// One CTA per row: writes, in position order, pos_offset + j for the candidates j in [lo, hi)
// with key > thr[row] and for the first ties[row] candidates with key == thr[row]; count[row]
// = the number written (at most cap; more sets KVC_ERR_INDEX and is not written).
__global__ void __launch_bounds__(kTopkThreads)
select_emit_kernel(const float* __restrict__ v, int n, int lo, int hi, const uint32_t* __restrict__ thr,
                   const int32_t* __restrict__ ties, int pos_offset, int32_t* __restrict__ out, int cap,
                   int32_t* __restrict__ count, unsigned* __restrict__ err) {
    __shared__ int wsel[kWarps], weq[kWarps];
    __shared__ int base_sel, base_eq;
    const int row = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float* vr = v + (size_t)row * n;
    int32_t* o = out + (size_t)row * cap;
    const uint32_t T = thr[row];
    const int take = ties[row];
    if (tid == 0) {
        base_sel = 0;
        base_eq = 0;
    }
    __syncthreads();
    for (int j0 = lo; j0 < hi; j0 += kTopkThreads) {
        const int j = j0 + tid;
        const bool in = j < hi && dcheck(err, j >= 0 && j < n);
        const uint32_t key = in ? order_key(vr[j]) : 0u;
        const bool gt = in && key > T, eq = in && key == T;
        const unsigned beq = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) weq[warp] = __popc(beq);
        __syncthreads();
        int eq_before = base_eq;  // ties before j, in position order
        for (int i = 0; i < warp; ++i) eq_before += weq[i];
        eq_before += __popc(beq & lanemask_lt());
        const bool sel = gt || (eq && eq_before < take);
        const unsigned bsel = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) wsel[warp] = __popc(bsel);
        __syncthreads();
        int at = base_sel;
        for (int i = 0; i < warp; ++i) at += wsel[i];
        at += __popc(bsel & lanemask_lt());
        if (sel) {
            if (at < cap) o[at] = pos_offset + j;
            else atomicOr(err, kErrIndex);
        }
        __syncthreads();
        if (tid == 0) {
            int a = 0, b = 0;
            for (int i = 0; i < kWarps; ++i) {
                a += wsel[i];
                b += weq[i];
            }
            base_sel += a;
            base_eq += b;
        }
        __syncthreads();
    }
    if (tid == 0) count[row] = min(base_sel, cap);
}

}  // namespace

cudaError_t reduce_units(const float* units, int L, int B, int Hkv, int N, int all_heads, float* out,
                         cudaStream_t s) {
    const long long total = (long long)B * (all_heads ? 1 : Hkv) * N;
    reduce_units_kernel<<<grid_for(total, 256), 256, 0, s>>>(units, L, B, Hkv, N, all_heads, out,
                                                             device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t accumulate(float* acc, const float* src, int B, int Hi, int Ho, int N, cudaStream_t s) {
    const long long total = (long long)B * Ho * N;
    if (total == 0) return cudaSuccess;
    accumulate_kernel<<<grid_for(total, 256), 256, 0, s>>>(acc, src, B, Hi, Ho, N, device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t pool(const float* in, float* out, int rows, int N, int lo, int hi, int kernel,
                 cudaStream_t s) {
    const long long total = (long long)rows * N;
    if (total == 0) return cudaSuccess;
    pool_kernel<<<grid_for(total, 256), 256, 0, s>>>(in, out, rows, N, lo, hi, (kernel - 1) / 2,
                                                     device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

bool topk_fused_fits(int N, int n_sink, int window) {
    const int n_c = N - n_sink - window;
    return (n_c + kClusterCtas - 1) / kClusterCtas + kSlotPad <= kSegMax;
}

namespace {

template <int R>
cudaError_t launch_topk_cluster(const float* scores, int rows, int N, int n_sink, int window, int budget, int radius,
                                int seg, int32_t* idx, size_t smem, cudaStream_t s) {
    static std::atomic<bool> attr_done[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_done[dev].load()) {
        e = cudaFuncSetAttribute(topk_cluster_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(TopkSmem));
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done[dev].store(true);
    }
    topk_cluster_kernel<R><<<rows * kClusterCtas, kCtThreads, smem, s>>>(scores, N, n_sink, window, budget, radius, seg,
                                                                        idx, device_error_word());
    return cudaGetLastError();
}

}  // namespace

cudaError_t topk_fused(const float* scores, int rows, int N, int n_sink, int window, int budget, int kernel,
                       int32_t* idx, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int n_c = N - n_sink - window;
    const int seg = (n_c + kClusterCtas - 1) / kClusterCtas;
    if (seg + kSlotPad > kSegMax) return cudaErrorInvalidValue;
    const size_t smem = sizeof(TopkSmem) - sizeof(uint32_t) * (size_t)(kSegMax - seg - kSlotPad);
    const int radius = (kernel - 1) / 2;
    // 16-byte loads need every row 16-byte aligned
    const bool vec = N % 4 == 0 && reinterpret_cast<uintptr_t>(scores) % 16 == 0;
    count_launches(1);
    if (vec) switch (radius) {
            case 0: return launch_topk_cluster<0>(scores, rows, N, n_sink, window, budget, radius, seg, idx, smem, s);
            case 1: return launch_topk_cluster<1>(scores, rows, N, n_sink, window, budget, radius, seg, idx, smem, s);
            case 2: return launch_topk_cluster<2>(scores, rows, N, n_sink, window, budget, radius, seg, idx, smem, s);
            case 3: return launch_topk_cluster<3>(scores, rows, N, n_sink, window, budget, radius, seg, idx, smem, s);
            case 4: return launch_topk_cluster<4>(scores, rows, N, n_sink, window, budget, radius, seg, idx, smem, s);
            default: break;
        }
    return launch_topk_cluster<-1>(scores, rows, N, n_sink, window, budget, radius, seg, idx, smem, s);
}

cudaError_t topk(const float* pooled, int rows, int N, int n_sink, int window, int budget,
                 int32_t* idx, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    topk_kernel<<<rows, kTopkThreads, 0, s>>>(pooled, N, n_sink, window, budget, idx, device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t row_stats(const float* scores, int rows, int N, int S, int w, const int32_t* idx, int budget,
                      float* kept_mass, float* cand_var, unsigned* err, cudaStream_t s) {
    row_stats_kernel<<<rows, kRsThreads, 0, s>>>(scores, N, S, w, idx, budget, kept_mass, cand_var, err);
    count_launches(1);
    return cudaGetLastError();
}

namespace {

// One warp per row: the bucket (scanned from the top) that holds the need-th largest key of
// the row's histogram summed over shards, the keys still needed inside it, the prefix
// extended by the bucket, and this shard's count in that bucket.
__global__ void select_pick_kernel(const uint32_t* __restrict__ hist, const uint32_t* __restrict__ hist_local,
                                   int rows, int digit_bits, int prefix_bits, int32_t* __restrict__ need,
                                   uint32_t* __restrict__ prefix, int32_t* __restrict__ eq_local, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (row >= rows) return;
    const int nb = 1 << digit_bits;
    const int per = (nb + 31) / 32;  // buckets per lane, lane 0 holding the top ones
    const uint32_t* h = hist + (size_t)row * nb;
    const long long want = need[row];
    // this lane's buckets, from the top: nb - 1 - lane*per down to nb - (lane+1)*per
    long long seg = 0;
    for (int t = 0; t < per; ++t) {
        const int b = nb - 1 - (lane * per + t);
        if (b >= 0) seg += h[b];
    }
    long long incl = seg;  // inclusive prefix over lanes (from the top)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const long long excl = incl - seg;
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= want);
    const int owner = hit ? __ffs(hit) - 1 : 31;
    if (lane == owner) {
        long long above = excl;
        int b = 0;
        long long inside = want - above;
        for (int t = 0; t < per; ++t) {
            const int bb = nb - 1 - (lane * per + t);
            if (bb < 0) break;
            b = bb;
            if (above + (long long)h[bb] >= want) break;
            above += h[bb];
        }
        inside = want - above;
        // the bucket holds the need-th largest: 1 <= inside <= its count
        dcheck(err, hit != 0 && inside >= 1 && inside <= (long long)h[b]);
        need[row] = (int32_t)inside;
        prefix[row] |= (uint32_t)b << (32 - prefix_bits - digit_bits);
        eq_local[row] = (int32_t)hist_local[(size_t)row * nb + b];
    }
}

// take[row] = min(max(need[row] - sum of eq_all[s][row] over shards s < rank, 0), eq_all[rank][row])
__global__ void select_ties_kernel(const int32_t* __restrict__ eq_all, int W, int rank, int rows,
                                   const int32_t* __restrict__ need, int32_t* __restrict__ take) {
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x) {
        long long before = 0;
        for (int s = 0; s < rank; ++s) before += eq_all[(size_t)s * rows + r];
        const long long t = (long long)need[r] - before;
        const long long mine = eq_all[(size_t)rank * rows + r];
        take[r] = (int32_t)(t < 0 ? 0 : (t > mine ? mine : t));
    }
}

// The block's kept rows in position order: its sinks, its selected positions, its window
// keys; global positions (-1 past the count) and local indices (0 past the count).
__global__ void select_kept_kernel(const int32_t* __restrict__ sel, const int32_t* __restrict__ cnt, int rows,
                                   int cap_sel, int N, int S, int w, int key_off, int n_local, int cap,
                                   int32_t* __restrict__ pos, int32_t* __restrict__ local, int32_t* __restrict__ count,
                                   unsigned* __restrict__ err) {
    const int row = blockIdx.x;
    const int s_lo = max(0, key_off), s_hi = min(S, key_off + n_local);            // sinks in the block
    const int w_lo = max(N - w, key_off), w_hi = min(N, key_off + n_local);        // window keys in the block
    const int n_s = max(0, s_hi - s_lo), n_w = max(0, w_hi - w_lo), n_sel = cnt[row];
    const int total = n_s + n_sel + n_w;
    if (threadIdx.x == 0) {
        count[row] = total;
        if (total > cap) atomicOr(err, kErrIndex);
    }
    for (int e = threadIdx.x; e < cap; e += blockDim.x) {
        int gp = -1;
        if (e < n_s) gp = s_lo + e;
        else if (e < n_s + n_sel) {
            if (dcheck(err, e - n_s < cap_sel)) gp = sel[(size_t)row * cap_sel + (e - n_s)];
            dcheck(err, gp >= max(S, key_off) && gp < min(N - w, key_off + n_local));
        }
        else if (e < total) gp = w_lo + (e - n_s - n_sel);
        pos[(size_t)row * cap + e] = gp;
        local[(size_t)row * cap + e] = gp >= 0 ? gp - key_off : 0;
    }
}

}  // namespace

cudaError_t select_pick(const uint32_t* hist, const uint32_t* hist_local, int rows, int digit_bits, int prefix_bits,
                        int32_t* need, uint32_t* prefix, int32_t* eq_local, cudaStream_t s) {
    count_launches(1);
    select_pick_kernel<<<(rows + 7) / 8, 256, 0, s>>>(hist, hist_local, rows, digit_bits, prefix_bits, need, prefix,
                                                      eq_local, device_error_word());
    return cudaGetLastError();
}

cudaError_t select_ties(const int32_t* eq_all, int W, int rank, int rows, const int32_t* need, int32_t* take,
                        cudaStream_t s) {
    count_launches(1);
    select_ties_kernel<<<(rows + 255) / 256, 256, 0, s>>>(eq_all, W, rank, rows, need, take);
    return cudaGetLastError();
}

cudaError_t select_kept(const int32_t* sel, const int32_t* cnt, int rows, int cap_sel, int N, int S, int w,
                        int key_off, int n_local, int cap, int32_t* pos, int32_t* local, int32_t* count,
                        unsigned* err, cudaStream_t s) {
    count_launches(1);
    select_kept_kernel<<<rows, 256, 0, s>>>(sel, cnt, rows, cap_sel, N, S, w, key_off, n_local, cap, pos, local,
                                            count, err);
    return cudaGetLastError();
}

cudaError_t select_hist(const float* pooled, int rows, int n, int lo, int hi, const uint32_t* prefix, int prefix_bits,
                        int digit_bits, uint32_t* hist, cudaStream_t s) {
    const int nb = 1 << digit_bits;
    cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)rows * nb * sizeof(uint32_t), s);
    if (e != cudaSuccess || hi <= lo) return e;
    dim3 grid(kHistBlocksPerRow, rows);
    select_hist_kernel<<<grid, kHistThreads, nb * sizeof(uint32_t), s>>>(pooled, n, lo, hi, prefix, prefix_bits,
                                                                          digit_bits, hist, device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t select_emit(const float* pooled, int rows, int n, int lo, int hi, const uint32_t* thr, const int32_t* ties,
                        int pos_offset, int32_t* out, int cap, int32_t* count, cudaStream_t s) {
    select_emit_kernel<<<rows, kTopkThreads, 0, s>>>(pooled, n, lo, hi, thr, ties, pos_offset, out, cap, count,
                                                     device_error_word());
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvc

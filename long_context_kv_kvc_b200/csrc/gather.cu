// gather.cu -- compact-cache row gather: dst row r = src row idx[r], byte for byte.
//
// The kept K/V rows of a KV head (FastKV page, sec. 2B: KV entries retained per layer for
// decoding) or the propagated hidden-state rows (sec. 2A, Token-Selective Propagation)
// are copied with 16-byte vector loads and stores; consecutive threads copy consecutive
// 16-byte pieces of a row, so both sides are coalesced.  Two tensors that share the index
// list (K and V) are copied by the same launch.  An index outside [0, N) is never
// dereferenced: the destination row is zero-filled and the per-device error word records
// it.
#include "kvc_internal.cuh"

namespace kvc {
namespace {

__global__ void __launch_bounds__(256)
gather_kernel(const uint4* __restrict__ src0, uint4* __restrict__ dst0,
              const uint4* __restrict__ src1, uint4* __restrict__ dst1, int Hsrc, int N, int cpr,
              const int32_t* __restrict__ idx, int Hidx, int K, long long total,
              unsigned* __restrict__ err) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long row = e / cpr;         // destination row over [B][Hsrc][K]
        const int piece = (int)(e - row * cpr);
        const int r = (int)(row % K);
        const long long bh = row / K;          // b * Hsrc + h
        const int h = (int)(bh % Hsrc);
        const long long b = bh / Hsrc;
        const int j = __ldg(idx + (b * Hidx + (Hidx == 1 ? 0 : h)) * K + r);
        uint4 a = make_uint4(0, 0, 0, 0), c = make_uint4(0, 0, 0, 0);
        if ((unsigned)j < (unsigned)N) {
            const long long s = (bh * N + j) * cpr + piece;
            if (!dcheck_idx(err, s, total / K * N)) continue;  // B * Hsrc * N rows of cpr pieces
            a = __ldcs(src0 + s);
            if (src1) c = __ldcs(src1 + s);
        } else if (piece == 0) {
            atomicOr(err, kErrIndex);
        }
        __stcs(dst0 + e, a);
        if (dst1) __stcs(dst1 + e, c);
    }
}

}  // namespace

cudaError_t gather(const void* src0, void* dst0, const void* src1, void* dst1, int B, int Hsrc, int N,
                   size_t row_bytes, const int32_t* idx, int Hidx, int K, unsigned* err,
                   cudaStream_t s) {
    const int cpr = (int)(row_bytes / 16);
    const long long total = (long long)B * Hsrc * K * cpr;
    if (total == 0) return cudaSuccess;
    long long grid = (total + 255) / 256;
    if (grid > 148LL * 16) grid = 148LL * 16;
    gather_kernel<<<(int)grid, 256, 0, s>>>((const uint4*)src0, (uint4*)dst0, (const uint4*)src1,
                                            (uint4*)dst1, Hsrc, N, cpr, idx, Hidx, K, total, err);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace kvc

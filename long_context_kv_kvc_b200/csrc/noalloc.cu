// noalloc.cu -- kvc_score_noalloc: saliency scores for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand this library a workspace: an inference engine that has
// already carved all of device memory into its own pool and exposes no allocator at the
// point where compaction runs, or a plugin interface that forbids cudaMalloc/cudaFree
// during a step (both may synchronise the device and stall every other stream).  For
// them this entry point scores with the CUDA-core kernels and keeps their scratch (the
// partial softmax statistics, the per-row log-sum-exp and, when several layers or all
// heads are summed, the per-unit score rows) in one fixed array compiled into the library.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes bytes.  Every GPU on
// which the library is loaded holds that much memory until the process exits.  Host code
// cannot use the array's name as a device address, so the first call on each device (with
// that device current) looks the address up with cudaGetSymbolAddress and caches it; make
// that first call before any stream capture starts.  The cached address stays valid for the
// life of the device's context: do not keep using the library across cudaDeviceReset or a
// reset of the primary context.  All calls on a device share the one
// array: two calls whose kernels overlap on the GPU (different streams, no ordering
// between them) overwrite each other's scratch and give wrong results, so callers must
// order them.  Every byte the kernels read from the array is written earlier in the same
// call, so nothing needs clearing between calls.
#include <atomic>

#include "kvc_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB per device

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_static_scratch on the current device (looked up once per device).
void* static_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev].store(p, std::memory_order_release);
    return p;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" kvc_status kvc_score_noalloc(const kvc_params* p, const void* q, const void* k, float* scores,
                                        kvc_stream_t stream) {
    // parameter checks shared with the other entry points
    size_t ws_unused = 0;
    const kvc_status st = kvc_workspace_size(p, &ws_unused);
    if (st != KVC_OK) return st;

    kvc::ScoreJob job{};
    job.q = q;
    job.k = k;
    job.dtype = p->dtype;
    job.U = p->n_layers * p->B * p->Hkv;
    job.N = p->N;
    job.window = p->window;
    job.G = p->Hq / p->Hkv;
    job.nq = job.G * p->window;
    const bool units = p->n_layers > 1 || p->scope == KVC_SCOPE_ALL_HEADS;

    const size_t partial_bytes = kvc::simt_score_workspace(job.U, job.N, job.nq, &job.n_chunks, &job.chunk);
    const size_t lse_off = round256(partial_bytes);
    const size_t units_off = round256(lse_off + (size_t)job.U * job.nq * sizeof(float));
    const size_t need = units ? units_off + (size_t)job.U * job.N * sizeof(float) : units_off;
    // the size check comes before the pointer checks, so that a parameter set that does not
    // fit is rejected whatever buffers come with it
    if (need > kStaticScratchBytes) return KVC_ERR_WORKSPACE;  // larger than the fixed array
    if (!q || !k || !scores) return KVC_ERR_ARG;
    if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)scores) & 15u) return KVC_ERR_ALIGN;

    char* scratch = (char*)static_scratch();
    if (!scratch) return KVC_ERR_CUDA;
    job.partial = (float2*)scratch;
    job.lse = (float*)(scratch + lse_off);
    job.unit_scores = units ? (float*)(scratch + units_off) : scores;
    job.err = kvc::device_error_word();
    if (!job.err) return KVC_ERR_CUDA;

    cudaStream_t s = (cudaStream_t)stream;
    if (kvc::simt_score(job, s) != cudaSuccess) return KVC_ERR_CUDA;
    if (units && kvc::reduce_units(job.unit_scores, p->n_layers, p->B, p->Hkv, p->N,
                                   p->scope == KVC_SCOPE_ALL_HEADS, scores, s) != cudaSuccess)
        return KVC_ERR_CUDA;
    return KVC_OK;
}

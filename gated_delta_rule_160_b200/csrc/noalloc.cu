// noalloc.cu -- gdn2_chunk_fwd_noalloc: prefill for callers that cannot allocate device
// memory.
//
// gdn2_chunk_fwd asks its caller for a small device workspace whenever sequences are
// packed with cu_seqlens: the longest-first order of the sequences, 4 bytes each. Some
// callers have no way to provide it: code that owns no device allocator of its own
// (a plug-in running inside another runtime's memory pool), code that must not allocate
// after start-up (a serving loop with a fixed memory budget), or code running where a
// cudaMalloc would synchronise the device at the wrong moment. This entry point keeps that
// scratch in a file-scope device array instead, so it allocates nothing at all.
//
// Limits and sharing:
//   * at most kNoAllocMaxSeqs sequences per call; larger batches are rejected with
//     GDN2_ERR_INVALID_ARG before anything is queued;
//   * the array (64 KB) is part of the library image: every GPU that loads the library
//     holds it until the process exits;
//   * all calls on a device share the one array. Each call writes every entry it reads
//     (the order kernel fills entries [0, n_seq) before the prefill kernel reads them, in
//     stream order), so nothing has to start at zero, but calls whose work overlaps on the
//     GPU (different streams running at the same time) race on it;
//   * the first call on each device looks up the array's device address (with that device
//     current) and caches it; make that first call before any stream capture.
#include <mutex>

#include "internal.cuh"

namespace gdn2 {
namespace {

constexpr int kNoAllocMaxSeqs = 16384;
__device__ __align__(256) int32_t g_noalloc_order[kNoAllocMaxSeqs];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_order on the current device. In host code the symbol names a
// host-side stand-in, so a kernel must be given this address instead.
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_order);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = ptr;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace gdn2

extern "C" {

gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_shape* shape, const void* q, const void* k, const void* v,
                                   const float* log_alpha, const void* b, const void* w, const float* S0,
                                   const int32_t* cu_seqlens, void* o, float* S_T, gdn2_stream_t stream) {
    if (shape && cu_seqlens && shape->n_seq > gdn2::kNoAllocMaxSeqs)
        return gdn2::report_error(GDN2_ERR_INVALID_ARG,
                                  "gdn2_chunk_fwd_noalloc takes at most 16384 packed sequences per call");
    void* scratch = nullptr;
    if (cu_seqlens) {
        const cudaError_t e = gdn2::noalloc_scratch(&scratch);
        if (e != cudaSuccess) return gdn2::report_error(GDN2_ERR_CUDA, cudaGetErrorString(e));
    }
    return gdn2_chunk_fwd(shape, q, k, v, log_alpha, b, w, S0, cu_seqlens, o, S_T, scratch,
                          scratch ? sizeof(int32_t) * gdn2::kNoAllocMaxSeqs : 0, stream);
}

}  // extern "C"

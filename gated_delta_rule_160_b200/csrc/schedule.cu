// schedule.cu -- longest-first order of packed sequences for the prefill kernels.
//
// Work items of a packed batch have very different lengths; dispatching the longest
// sequences first keeps the last wave short. order[rank] = sequence, ranked by length
// (descending), ties by index, so the order is deterministic. The same pass checks that
// cu_seqlens is a valid packing (0 = c_0 <= ... <= c_n = T_total) and flags the device
// status word if not.
#include "internal.cuh"

namespace gdn2 {
namespace {

// Device status word of this file's kernels (kStatus* bits), read and cleared by
// gdn2_device_status.
__device__ unsigned int g_status_sched = 0;

// Is cu_seqlens 0 = c_0 <= c_1 <= ... <= c_n = T_total around entry i (i in [0, n_seq))?
__device__ __forceinline__ bool seqlens_ok_at(const int32_t* cu, int n_seq, int T_total, int i) {
    bool ok = cu[i] <= cu[i + 1];
    if (i == 0) ok = ok && cu[0] == 0;
    if (i == n_seq - 1) ok = ok && cu[n_seq] == T_total;
    return ok;
}

__global__ void varlen_order_kernel(const int32_t* __restrict__ cu, int n_seq, int T_total,
                                    int32_t* __restrict__ order) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_seq; i += gridDim.x * blockDim.x) {
        if (!seqlens_ok_at(cu, n_seq, T_total, i)) atomicOr(&g_status_sched, kStatusBadSeqlens);
        const int li = cu[i + 1] - cu[i];
        int rank = 0;
        for (int j = 0; j < n_seq; ++j) {
            const int lj = cu[j + 1] - cu[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

__global__ void check_seqlens_kernel(const int32_t* __restrict__ cu, int n_seq, int T_total) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_seq; i += gridDim.x * blockDim.x)
        if (!seqlens_ok_at(cu, n_seq, T_total, i)) atomicOr(&g_status_sched, kStatusBadSeqlens);
}

}  // namespace

cudaError_t launch_varlen_order(const Params& p, int32_t* order, cudaStream_t s) {
    const int threads = 128;
    const int blocks = (p.n_seq + threads - 1) / threads;
    varlen_order_kernel<<<blocks, threads, 0, s>>>(p.cu_seqlens, p.n_seq, p.T_total, order);
    return cudaGetLastError();
}

cudaError_t launch_check_seqlens(const Params& p, cudaStream_t s) {
    const int threads = 128;
    const int blocks = (p.n_seq + threads - 1) / threads;
    check_seqlens_kernel<<<blocks, threads, 0, s>>>(p.cu_seqlens, p.n_seq, p.T_total);
    return cudaGetLastError();
}

cudaError_t read_clear_status_schedule(unsigned int* out, cudaStream_t s) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_status_sched, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    static const unsigned int zero = 0;
    return cudaMemcpyToSymbolAsync(g_status_sched, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s);
}

}  // namespace gdn2

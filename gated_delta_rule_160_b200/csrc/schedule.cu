// schedule.cu -- longest-first order of packed sequences for the prefill kernels.
//
// Work items of a packed batch have very different lengths; dispatching the longest
// sequences first keeps the last wave short. order[rank] = sequence, ranked by length
// (descending), ties by index, so the order is deterministic.
#include "internal.cuh"

namespace gdn2 {
namespace {

__global__ void varlen_order_kernel(const int32_t* __restrict__ cu, int n_seq, int32_t* __restrict__ order) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_seq; i += gridDim.x * blockDim.x) {
        const int li = cu[i + 1] - cu[i];
        int rank = 0;
        for (int j = 0; j < n_seq; ++j) {
            const int lj = cu[j + 1] - cu[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

}  // namespace

cudaError_t launch_varlen_order(const Params& p, int32_t* order, cudaStream_t s) {
    const int threads = 128;
    const int blocks = (p.n_seq + threads - 1) / threads;
    varlen_order_kernel<<<blocks, threads, 0, s>>>(p.cu_seqlens, p.n_seq, order);
    return cudaGetLastError();
}

}  // namespace gdn2

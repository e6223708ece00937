// Work order of a packed ragged batch: sequence indices sorted by length,
// longest first (ties by index), computed on the device from cu_seqlens so
// the host never waits for the lengths.  The persistent tensor-core kernel
// deals items out in this order, which keeps per-CTA token totals balanced.
#pragma once

namespace lcl {
namespace vorder {

constexpr int NUM_THREADS = 1024;
constexpr int MAX_SORTED = 4096;  // beyond this the batch keeps its own order

__global__ void __launch_bounds__(NUM_THREADS) order_kernel(const int* __restrict__ cu, int n_seq, int* __restrict__ order) {
    __shared__ int len[MAX_SORTED];
    if (n_seq > MAX_SORTED) {
        for (int i = threadIdx.x; i < n_seq; i += NUM_THREADS) order[i] = i;
        return;
    }
    for (int i = threadIdx.x; i < n_seq; i += NUM_THREADS) len[i] = cu[i + 1] - cu[i];
    __syncthreads();
    for (int i = threadIdx.x; i < n_seq; i += NUM_THREADS) {
        const int li = len[i];
        int rank = 0;
        for (int j = 0; j < n_seq; ++j) {
            const int lj = len[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

}  // namespace vorder
}  // namespace lcl

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

// Segments of a packed batch cut into pieces of seg_len tokens (the last piece
// of a sequence may be shorter; an empty sequence keeps one empty piece).  In
// work order (rank r = position in `order`): seg_off[r] = the number of
// segments before rank r, seg_off_nl[r] = the same not counting each
// sequence's last segment; both have n_seq + 1 entries.  One warp scans the
// ranks 32 at a time.
__global__ void __launch_bounds__(32) seg_plan_kernel(const int* __restrict__ cu, const int* __restrict__ order,
                                                     int n_seq, int seg_len, int* __restrict__ seg_off,
                                                     int* __restrict__ seg_off_nl) {
    const int lane = threadIdx.x;
    int carry = 0, carry_nl = 0;
    for (int base = 0; base < n_seq; base += 32) {
        const int r = base + lane;
        int c = 0;
        if (r < n_seq) {
            const int sq = order[r];
            const int len = cu[sq + 1] - cu[sq];
            c = max(1, (len + seg_len - 1) / seg_len);
        }
        const int cnl = r < n_seq ? c - 1 : 0;
        int x = c, y = cnl;  // inclusive scans over the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int xs = __shfl_up_sync(0xffffffffu, x, off), ys = __shfl_up_sync(0xffffffffu, y, off);
            if (lane >= off) {
                x += xs;
                y += ys;
            }
        }
        if (r < n_seq) {
            seg_off[r] = carry + x - c;
            seg_off_nl[r] = carry_nl + y - cnl;
        }
        carry += __shfl_sync(0xffffffffu, x, 31);
        carry_nl += __shfl_sync(0xffffffffu, y, 31);
    }
    if (lane == 0) {
        seg_off[n_seq] = carry;
        seg_off_nl[n_seq] = carry_nl;
    }
}

}  // namespace vorder
}  // namespace lcl

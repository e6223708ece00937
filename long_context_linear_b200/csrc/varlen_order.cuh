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

// Segments of a packed batch: the segment length is chosen here, where the
// lengths are known, as the smallest multiple of `unit` tokens, at least
// min_seg, for which the batch has at most max_segs segments (a sequence of
// len tokens has max(1, ceil(len / seg_len)) of them; the last one may be
// shorter; an empty sequence keeps one empty piece).  max_segs >= n_seq.
// Written: *seg_len, and in work order (rank r = position in `order`):
// seg_off[r] = the number of segments before rank r, seg_off_nl[r] = the same
// not counting each sequence's last segment; both have n_seq + 1 entries.
// One warp: a binary search over the length, then a scan of the ranks 32 at a
// time.
__device__ __forceinline__ int seg_pieces(int len, int seg) {
    return static_cast<int>(max(1L, ((long)len + seg - 1) / seg));
}
__device__ __forceinline__ long seg_count_warp(const int* __restrict__ cu, int n_seq, int seg) {
    long c = 0;
    for (int i = threadIdx.x; i < n_seq; i += 32) c += seg_pieces(cu[i + 1] - cu[i], seg);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    return c;
}

__global__ void __launch_bounds__(32) seg_plan_kernel(const int* __restrict__ cu, const int* __restrict__ order,
                                                     int n_seq, long max_segs, int min_seg, int unit,
                                                     int* __restrict__ seg_len_out, int* __restrict__ seg_off,
                                                     int* __restrict__ seg_off_nl) {
    const int lane = threadIdx.x;
    int max_len = 0;
    for (int i = lane; i < n_seq; i += 32) max_len = max(max_len, cu[i + 1] - cu[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) max_len = max(max_len, __shfl_xor_sync(0xffffffffu, max_len, off));
    // smallest u in [lo, hi] with count(u * unit) <= max_segs; count(hi * unit) = n_seq
    int lo = (min_seg + unit - 1) / unit, hi = max(lo, (max_len + unit - 1) / unit);
    while (lo < hi) {
        const int mid = lo + (hi - lo) / 2;
        if (seg_count_warp(cu, n_seq, mid * unit) <= max_segs) hi = mid;
        else lo = mid + 1;
    }
    const int seg_len = lo * unit;
    if (lane == 0) *seg_len_out = seg_len;
    int carry = 0, carry_nl = 0;
    for (int base = 0; base < n_seq; base += 32) {
        const int r = base + lane;
        int c = 0;
        if (r < n_seq) {
            const int sq = order[r];
            const int len = cu[sq + 1] - cu[sq];
            c = seg_pieces(len, seg_len);
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

// States at segment starts for a prefill whose sequences are cut into segments.
//
// The state after t tokens is S_t = S_0 + sum_{s <= t} k_s v_s^T (page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"), so the
// state before segment p is S_0 plus the K^T V sums of segments 0 .. p-1; the
// sums of the segments (dS_p) come from a state-only pass of the prefill
// kernel over segments 0 .. n_seg-2.  In reverse token order (the backward's
// suffix sums) the state before segment p is S_init plus the sums of segments
// p+1 .. n_seg-1.  Each thread owns 4 consecutive fp32 elements of one unit's
// d_k x d_v state and walks the segments in order.
#pragma once
#include <cuda_runtime.h>

namespace lcl {
namespace segp {

constexpr int NUM_THREADS = 256;

// seg_sums: [U][n_seg-1][elems]; s0: [U][elems] or null; starts: [U][n_seg][elems].
// Forward: seg_sums[p] is the sum of segment p, starts[p] = s0 + sum_{p' < p}.
// Reverse (tokens visited last to first): seg_sums[p] is the sum of segment
// p + 1, starts[p] = s0 + sum_{p' > p}.  s0_transposed: s0 is given as the
// transpose of a d x d state (elems = d * d).
__global__ void __launch_bounds__(NUM_THREADS)
seg_prefix_kernel(const float* __restrict__ seg_sums, const float* __restrict__ s0, float* __restrict__ starts,
                  long U, int n_seg, int elems, int reverse, int s0_transposed, int d) {
    const int per_unit = elems / 4;
    for (long t = (long)blockIdx.x * blockDim.x + threadIdx.x; t < U * per_unit; t += (long)gridDim.x * blockDim.x) {
        const long u = t / per_unit;
        const int e = static_cast<int>(t - u * per_unit) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0 && s0_transposed) {
            const float* b = s0 + u * elems;
            const int i = e / d, j = e % d;
            acc = make_float4(b[j * d + i], b[(j + 1) * d + i], b[(j + 2) * d + i], b[(j + 3) * d + i]);
        } else if (s0) {
            acc = *reinterpret_cast<const float4*>(s0 + u * elems + e);
        }
        float* dst = starts + (u * n_seg) * (long)elems + e;
        const float* src = seg_sums + (u * (n_seg - 1)) * (long)elems + e;
        if (!reverse) {
            *reinterpret_cast<float4*>(dst) = acc;
            for (int p = 1; p < n_seg; ++p) {
                const float4 x = *reinterpret_cast<const float4*>(src + (long)(p - 1) * elems);
                acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
                *reinterpret_cast<float4*>(dst + (long)p * elems) = acc;
            }
        } else {
            *reinterpret_cast<float4*>(dst + (long)(n_seg - 1) * elems) = acc;
            for (int p = n_seg - 2; p >= 0; --p) {
                const float4 x = *reinterpret_cast<const float4*>(src + (long)p * elems);
                acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
                *reinterpret_cast<float4*>(dst + (long)p * elems) = acc;
            }
        }
    }
}

// The same for a packed batch whose sequences have different segment counts
// (seg_off, seg_off_nl from vorder::seg_plan_kernel, in work order): the state
// before segment g of rank r, head h is pool[init_idx[seq]][h] (or zero) plus
// the sums of the sequence's segments before g.
//   seg_sums: [non-last segments][H][elems]   starts: [segments][H][elems]
__global__ void __launch_bounds__(NUM_THREADS)
seg_prefix_varlen_kernel(const float* __restrict__ seg_sums, const float* __restrict__ pool,
                         const int* __restrict__ init_idx, const int* __restrict__ order, const int* __restrict__ seg_off,
                         const int* __restrict__ seg_off_nl, float* __restrict__ starts, int n_seq, int H, int elems) {
    const int per_unit = elems / 4;
    const long total = (long)n_seq * H * per_unit;
    for (long t = (long)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (long)gridDim.x * blockDim.x) {
        const int r = static_cast<int>(t / ((long)H * per_unit));
        const int rem = static_cast<int>(t - (long)r * H * per_unit);
        const int h = rem / per_unit, e = (rem - h * per_unit) * 4;
        const int sq = order[r];
        const int ii = init_idx ? init_idx[sq] : -1;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (pool && ii >= 0) acc = *reinterpret_cast<const float4*>(pool + ((long)ii * H + h) * elems + e);
        const int s0 = seg_off[r], cnt = seg_off[r + 1] - s0, nl0 = seg_off_nl[r];
        *reinterpret_cast<float4*>(starts + ((long)s0 * H + h) * elems + e) = acc;
        for (int g = 1; g < cnt; ++g) {
            const float4 x = *reinterpret_cast<const float4*>(seg_sums + ((long)(nl0 + g - 1) * H + h) * elems + e);
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
            *reinterpret_cast<float4*>(starts + ((long)(s0 + g) * H + h) * elems + e) = acc;
        }
    }
}

}  // namespace segp
}  // namespace lcl

// States at segment starts for a prefill whose sequences are cut into segments.
//
// The state after t tokens is S_t = S_0 + sum_{s <= t} k_s v_s^T (page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"), so the
// state before segment p is S_0 plus the K^T V sums of segments 0 .. p-1; the
// sums of the segments (dS_p) come from a state-only pass of the prefill
// kernel over segments 0 .. n_seg-2.  Each thread owns 4 consecutive fp32
// elements of one unit's d_k x d_v state and walks the segments in order.
#pragma once
#include <cuda_runtime.h>

namespace lcl {
namespace segp {

constexpr int NUM_THREADS = 256;

// seg_sums: [U][n_seg-1][elems]; s0: [U][elems] or null; starts: [U][n_seg][elems].
__global__ void __launch_bounds__(NUM_THREADS)
seg_prefix_kernel(const float* __restrict__ seg_sums, const float* __restrict__ s0, float* __restrict__ starts,
                  long U, int n_seg, int elems) {
    const int per_unit = elems / 4;
    for (long t = (long)blockIdx.x * blockDim.x + threadIdx.x; t < U * per_unit; t += (long)gridDim.x * blockDim.x) {
        const long u = t / per_unit;
        const int e = static_cast<int>(t - u * per_unit) * 4;
        float4 acc = s0 ? *reinterpret_cast<const float4*>(s0 + u * elems + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        float* dst = starts + (u * n_seg) * (long)elems + e;
        const float* src = seg_sums + (u * (n_seg - 1)) * (long)elems + e;
        *reinterpret_cast<float4*>(dst) = acc;
        for (int p = 1; p < n_seg; ++p) {
            const float4 d = *reinterpret_cast<const float4*>(src + (long)(p - 1) * elems);
            acc.x += d.x; acc.y += d.y; acc.z += d.z; acc.w += d.w;
            *reinterpret_cast<float4*>(dst + (long)p * elems) = acc;
        }
    }
}

}  // namespace segp
}  // namespace lcl

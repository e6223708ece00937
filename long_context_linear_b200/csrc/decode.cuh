// One decode step for a batch of independent states (HBM-bound).
//
// Per (sequence, head): S <- S + k v^T, then o = q S (the recurrence of page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎", one token at a
// time; page "MiniMax: «Почему M2 …»", section 4, notes this is a small state
// matrix that is read and written on every step).  One CTA streams one d x d
// fp32 state once: every thread owns 4 consecutive value columns of D/RS rows,
// loads them with 16-byte streaming loads (all loads issued before any use),
// updates, stores them back, and accumulates its share of o; partial sums are
// reduced across row slots in shared memory.
#pragma once
#include <cuda_bf16.h>

namespace lcl {
namespace dec {

constexpr int NUM_THREADS = 256;

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, int D>
__global__ void __launch_bounds__(NUM_THREADS)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
                   float* __restrict__ S) {
    constexpr int TPR = D / 4;             // threads per row
    constexpr int RS = NUM_THREADS / TPR;  // row slots
    constexpr int RPT = D / RS;            // rows per thread
    __shared__ float qs[D], ks[D], vs[D];
    __shared__ float4 red[RS][TPR];

    const long u = blockIdx.x;
    const int tid = threadIdx.x;
    const int c4 = tid % TPR;
    const int slot = tid / TPR;
    float4* Su = reinterpret_cast<float4*>(S + u * D * D);

    float4 x[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) x[m] = __ldcs(&Su[(slot + m * RS) * TPR + c4]);
    if (tid < D) {
        qs[tid] = ld_f(q + u * D + tid);
        ks[tid] = ld_f(k + u * D + tid);
        vs[tid] = ld_f(v + u * D + tid);
    }
    __syncthreads();
    const float4 vj = make_float4(vs[4 * c4], vs[4 * c4 + 1], vs[4 * c4 + 2], vs[4 * c4 + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = slot + m * RS;
        const float ki = ks[i], qi = qs[i];
        float4 y = x[m];
        y.x = fmaf(ki, vj.x, y.x);
        y.y = fmaf(ki, vj.y, y.y);
        y.z = fmaf(ki, vj.z, y.z);
        y.w = fmaf(ki, vj.w, y.w);
        __stcs(&Su[i * TPR + c4], y);
        acc.x = fmaf(qi, y.x, acc.x);
        acc.y = fmaf(qi, y.y, acc.y);
        acc.z = fmaf(qi, y.z, acc.z);
        acc.w = fmaf(qi, y.w, acc.w);
    }
    red[slot][c4] = acc;
    __syncthreads();
    if (tid < D) {
        const float* rf = reinterpret_cast<const float*>(&red[0][0]);
        float sum = 0.f;
#pragma unroll
        for (int s = 0; s < RS; ++s) sum += rf[s * D + tid];
        st_f(o + u * D + tid, sum);
    }
}

}  // namespace dec
}  // namespace lcl

// Speculative decoding over m draft tokens per (sequence, head): verify, then commit.
//
// A draft model proposes m tokens; the target must give o_t = q_t S_t for all
// of them, then keep the state of the accepted prefix only.  The state cannot
// simply be truncated after the fact (page "MiniMax: «Почему M2 …»",
// section 4, and page "MiniMax-M1で理解する…", the infrastructure list: a
// recurrent state has no per-token entries to drop), so the two halves are
// separate:
//
//   verify:  o_t = q_t S_0 + sum_{s <= t} (q_t . k_s) v_s      S_0 is only read
//            (the recurrence S_t = S_0 + sum_{s<=t} k_s v_s^T of page
//            "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎",
//            expanded for the m tokens)
//   commit:  S <- S + sum_{t < a} k_t v_t^T, a = accepted count, in place, one
//            fused multiply-add per token in token order (so the committed
//            state is bit-identical to a single decode steps)
//
// A feature map phi (phi.cuh) is applied to q and k as they are loaded.
// Both read the d x d fp32 state once (commit also writes it): 3 state passes
// for m tokens instead of 2 m with m decode steps.  Layout per unit as in
// decode.cuh: thread = one 16-byte column vector of D/RS rows.
#pragma once
#include <cuda_bf16.h>
#include "decode.cuh"

namespace lcl {
namespace dmulti {

constexpr int NUM_THREADS = 256;
constexpr int MAX_M = 16;

constexpr int G = 4;  // draft tokens per reduction round of verify

// 16 bytes of T -> fp32 (4 fp32 or 8 bf16 values)
__device__ __forceinline__ void unpack16(const uint4 r, float (&f)[4]) {
    f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y); f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void unpack16(const uint4 r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Two CTAs per SM: the bound lets the compiler use up to 128 registers, and
// with them verify keeps more loads in flight (measured: 0.213 ms against
// 0.257 ms at 101 registers for B=256, H=64, m=4).
template <typename T, int D>
__global__ void __launch_bounds__(NUM_THREADS, 2)
verify_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
              const float* __restrict__ S, int m, int phi) {
    constexpr int TPR = D / 4;
    constexpr int RS = NUM_THREADS / TPR;
    constexpr int RPT = D / RS;
    __shared__ __align__(16) float qs[MAX_M][D], ks[MAX_M][D], vs[MAX_M][D];
    __shared__ float A[MAX_M][MAX_M];  // A[t][s] = q_t . k_s, s <= t
    __shared__ __align__(16) float red[G][RS][D];

    const long u = blockIdx.x;
    const int tid = threadIdx.x;
    const int c4 = tid % TPR, slot = tid / TPR;
    const float4* Su = reinterpret_cast<const float4*>(S + u * D * D);
    float4 x[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) x[r] = __ldcs(&Su[(slot + r * RS) * TPR + c4]);
    const long base = u * (long)m * D;
    // the drafts' q, k, v: 16-byte loads (rows are 16-byte aligned: D * sizeof(T) is)
    constexpr int VEC = 16 / (int)sizeof(T);
    for (int e = tid * VEC; e < m * D; e += NUM_THREADS * VEC) {
        const int t = e / D, i = e % D;
        float qv[VEC], kv[VEC], vv[VEC];
        unpack16(*reinterpret_cast<const uint4*>(q + base + e), qv);
        unpack16(*reinterpret_cast<const uint4*>(k + base + e), kv);
        unpack16(*reinterpret_cast<const uint4*>(v + base + e), vv);
#pragma unroll
        for (int j = 0; j < VEC; j += 4) {
            *reinterpret_cast<float4*>(&qs[t][i + j]) = make_float4(apply_phi(qv[j], phi), apply_phi(qv[j + 1], phi),
                                                                    apply_phi(qv[j + 2], phi), apply_phi(qv[j + 3], phi));
            *reinterpret_cast<float4*>(&ks[t][i + j]) = make_float4(apply_phi(kv[j], phi), apply_phi(kv[j + 1], phi),
                                                                    apply_phi(kv[j + 2], phi), apply_phi(kv[j + 3], phi));
            *reinterpret_cast<float4*>(&vs[t][i + j]) = make_float4(vv[j], vv[j + 1], vv[j + 2], vv[j + 3]);
        }
    }
    __syncthreads();
    // intra-draft scores: one warp per pair (t, s), s <= t, lanes split the dim;
    // pairs in row order, warp w taking every 8th from the w-th, (t, s) stepped
    // along without recomputing it from the pair index
    {
        constexpr int NW = NUM_THREADS / 32;
        const int warp = tid >> 5, lane = tid & 31;
        int t = 0, s = warp;
        while (s > t) { s -= t + 1; ++t; }
        for (; t < m;) {
            float a = 0.f;
#pragma unroll
            for (int i = lane; i < D; i += 32) a = fmaf(qs[t][i], ks[s][i], a);
#pragma unroll
            for (int off = 16; off; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
            if (lane == 0) A[t][s] = a;
            s += NW;
            while (s > t) { s -= t + 1; ++t; }
        }
    }
    // q_t S_0 for G draft tokens at a time, reduced over row slots, plus the
    // intra-draft terms (A is complete after the barrier below)
    for (int t0 = 0; t0 < m; t0 += G) {
        const int gn = min(G, m - t0);
        float4 acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float qi = g < gn ? qs[t0 + g][slot + r * RS] : 0.f;
                acc[g].x = fmaf(qi, x[r].x, acc[g].x);
                acc[g].y = fmaf(qi, x[r].y, acc[g].y);
                acc[g].z = fmaf(qi, x[r].z, acc[g].z);
                acc[g].w = fmaf(qi, x[r].w, acc[g].w);
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) *reinterpret_cast<float4*>(&red[g][slot][4 * c4]) = acc[g];
        __syncthreads();
        for (int e = tid; e < gn * D; e += NUM_THREADS) {
            const int g = e / D, col = e % D, t = t0 + g;
            float sum = 0.f;
#pragma unroll
            for (int sl = 0; sl < RS; ++sl) sum += red[g][sl][col];
            for (int s = 0; s <= t; ++s) sum = fmaf(A[t][s], vs[s][col], sum);
            dec::st_f(o + base + (long)t * D + col, sum);
        }
        __syncthreads();
    }
}

// Two CTAs per SM (up to 128 registers, no spills).
template <typename T, int D>
__global__ void __launch_bounds__(NUM_THREADS, 2)
commit_kernel(const T* __restrict__ k, const T* __restrict__ v, float* __restrict__ S,
              const int* __restrict__ accepted, int H, int m, int phi) {
    constexpr int TPR = D / 4;
    constexpr int RS = NUM_THREADS / TPR;
    constexpr int RPT = D / RS;
    __shared__ __align__(16) float ks[MAX_M][D], vs[MAX_M][D];

    const long u = blockIdx.x;
    const int tid = threadIdx.x;
    const int c4 = tid % TPR, slot = tid / TPR;
    // the state loads go out before the accepted count is known, so that the
    // two memory latencies overlap (a unit that accepts nothing reads its
    // state in vain)
    float4* Su = reinterpret_cast<float4*>(S + u * D * D);
    float4 x[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) x[r] = __ldcs(&Su[(slot + r * RS) * TPR + c4]);
    const int a = min(max(accepted[u / H], 0), m);
    if (a == 0) return;
    const long base = u * (long)m * D;
    constexpr int VEC = 16 / (int)sizeof(T);
    for (int e = tid * VEC; e < a * D; e += NUM_THREADS * VEC) {
        const int t = e / D, i = e % D;
        float kv[VEC], vv[VEC];
        unpack16(*reinterpret_cast<const uint4*>(k + base + e), kv);
        unpack16(*reinterpret_cast<const uint4*>(v + base + e), vv);
#pragma unroll
        for (int j = 0; j < VEC; j += 4) {
            *reinterpret_cast<float4*>(&ks[t][i + j]) = make_float4(apply_phi(kv[j], phi), apply_phi(kv[j + 1], phi),
                                                                    apply_phi(kv[j + 2], phi), apply_phi(kv[j + 3], phi));
            *reinterpret_cast<float4*>(&vs[t][i + j]) = make_float4(vv[j], vv[j + 1], vv[j + 2], vv[j + 3]);
        }
    }
    __syncthreads();
    for (int t = 0; t < a; ++t) {
        const float4 vj = *reinterpret_cast<const float4*>(&vs[t][4 * c4]);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float ki = ks[t][slot + r * RS];
            x[r].x = fmaf(ki, vj.x, x[r].x);
            x[r].y = fmaf(ki, vj.y, x[r].y);
            x[r].z = fmaf(ki, vj.z, x[r].z);
            x[r].w = fmaf(ki, vj.w, x[r].w);
        }
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) __stcs(&Su[(slot + r * RS) * TPR + c4], x[r]);
}

}  // namespace dmulti
}  // namespace lcl

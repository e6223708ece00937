// Gradients of chunked causal linear attention (FFMA, fp32 arithmetic).
//
// For S_t = S_{t-1} + k_t v_t^T (S_0 = s0) and o_t = q_t S_t (page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"), a loss with
// dL/do_t = do_t and dL/dS_N = dS_N has, by the chain rule,
//   dq_t = do_t S_t^T,
//   G_t  = sum_{t' >= t} q_t'^T do_t' + dS_N,  dk_t = G_t v_t,  dv_t = G_t^T k_t,
//   dS_0 = G_1.
// Tiled like the forward (masked products inside a chunk of CS tokens, a
// d x d matrix carried between chunks; page "MiniMax: «Почему M2 …»",
// section 1, glossary entry "Lightning Attention"):
//   dQ_c = ((dO_c V_c^T) ⊙ M) K_c + dO_c S_{c-1}^T,       S_c = S_{c-1} + K_c^T V_c
//   dK_c = ((V_c dO_c^T) ⊙ M^T) Q_c + V_c G_{c+1}^T,
//   dV_c = ((K_c Q_c^T) ⊙ M^T) dO_c + K_c G_{c+1},        G_c = G_{c+1} + Q_c^T dO_c
// Grid of 2 U CTAs: CTAs 0 .. U-1 sweep forward for dQ (carrying S), CTAs
// U .. 2U-1 sweep backward for dK and dV (carrying G); both keep their d x d
// fp32 matrix and the chunk tiles in shared memory.
#pragma once
#include <cuda_bf16.h>
#include "prefill_simt.cuh"

namespace lcl {
namespace bwd {

constexpr int NUM_THREADS = 256;

struct Params {
    int U, N;
    const float* s0;    // [U][D][D] or null
    const float* ds_n;  // [U][D][D] or null
    float* ds0;         // [U][D][D] or null
};

template <int D, int CS>
constexpr int smem_bytes() {
    return (D * D + 4 * CS * (D + 1) + 2 * CS * (CS + 1)) * 4;
}

template <typename T, int D, int CS>
__global__ void __launch_bounds__(NUM_THREADS)
backward_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const T* __restrict__ dout, T* __restrict__ dq, T* __restrict__ dk, T* __restrict__ dv,
                     const Params p) {
    extern __shared__ float sf[];
    constexpr int LD = D + 1, LA = CS + 1;
    float* X = sf;                 // [D][D]: S (forward CTAs) or G (backward CTAs)
    float* Qs = X + D * D;         // [CS][LD]
    float* Ks = Qs + CS * LD;
    float* Vs = Ks + CS * LD;
    float* Os = Vs + CS * LD;      // dO tile
    float* A1 = Os + CS * LD;      // [CS][LA]
    float* A2 = A1 + CS * LA;
    const int tid = threadIdx.x;
    const bool fwd = blockIdx.x < p.U;
    const long u = fwd ? blockIdx.x : blockIdx.x - p.U;
    const long row0 = u * (long)p.N;
    const int N = p.N;
    const float* init = fwd ? p.s0 : p.ds_n;
    for (int e = tid; e < D * D; e += NUM_THREADS) X[e] = init ? init[u * D * D + e] : 0.f;
    const int nchunks = (N + CS - 1) / CS;

    for (int ci = 0; ci < nchunks; ++ci) {
        const int c = fwd ? ci : nchunks - 1 - ci;
        const int c0 = c * CS;
        const int rows = min(CS, N - c0);
        __syncthreads();
        for (int e = tid; e < CS * D; e += NUM_THREADS) {
            const int t = e / D, i = e % D;
            float a = 0.f, b = 0.f, cc = 0.f, dd = 0.f;
            if (t < rows) {
                const long g = (row0 + c0 + t) * D + i;
                if (!fwd) a = simt::to_f(q[g]);
                b = simt::to_f(k[g]);
                cc = simt::to_f(v[g]);
                dd = simt::to_f(dout[g]);
            }
            Qs[t * LD + i] = a;
            Ks[t * LD + i] = b;
            Vs[t * LD + i] = cc;
            Os[t * LD + i] = dd;
        }
        __syncthreads();
        if (fwd) {
            // A1[t][s] = dO_t . V_s for s <= t
            for (int e = tid; e < CS * CS; e += NUM_THREADS) {
                const int t = e / CS, s = e % CS;
                float a = 0.f;
                if (s <= t) {
#pragma unroll 8
                    for (int j = 0; j < D; ++j) a = fmaf(Os[t * LD + j], Vs[s * LD + j], a);
                }
                A1[t * LA + s] = a;
            }
            __syncthreads();
            // dq_t[i] = sum_{s<=t} A1[t][s] k_s[i] + sum_j do_t[j] S[i][j]
            for (int e = tid; e < CS * D; e += NUM_THREADS) {
                const int t = e / D, i = e % D;
                if (t < rows) {
                    float acc = 0.f;
                    for (int s = 0; s <= t; ++s) acc = fmaf(A1[t * LA + s], Ks[s * LD + i], acc);
#pragma unroll 8
                    for (int j = 0; j < D; ++j) acc = fmaf(Os[t * LD + j], X[i * D + j], acc);
                    dq[(row0 + c0 + t) * D + i] = simt::from_f<T>(acc);
                }
            }
            __syncthreads();
            // S += K^T V
            for (int e = tid; e < D * D; e += NUM_THREADS) {
                const int i = e / D, j = e % D;
                float acc = X[e];
                for (int s = 0; s < rows; ++s) acc = fmaf(Ks[s * LD + i], Vs[s * LD + j], acc);
                X[e] = acc;
            }
        } else {
            // A1[s][t] = v_s . do_t and A2[s][t] = k_s . q_t for t >= s
            for (int e = tid; e < CS * CS; e += NUM_THREADS) {
                const int s = e / CS, t = e % CS;
                float a1 = 0.f, a2 = 0.f;
                if (t >= s) {
#pragma unroll 8
                    for (int j = 0; j < D; ++j) a1 = fmaf(Vs[s * LD + j], Os[t * LD + j], a1);
#pragma unroll 8
                    for (int i = 0; i < D; ++i) a2 = fmaf(Ks[s * LD + i], Qs[t * LD + i], a2);
                }
                A1[s * LA + t] = a1;
                A2[s * LA + t] = a2;
            }
            __syncthreads();
            // dk_s[i] = sum_{t>=s} A1[s][t] q_t[i] + sum_j v_s[j] G[i][j]
            // dv_s[j] = sum_{t>=s} A2[s][t] do_t[j] + sum_i k_s[i] G[i][j]
            for (int e = tid; e < CS * D; e += NUM_THREADS) {
                const int s = e / D, x = e % D;
                if (s < rows) {
                    float a = 0.f, b = 0.f;
                    for (int t = s; t < rows; ++t) {
                        a = fmaf(A1[s * LA + t], Qs[t * LD + x], a);
                        b = fmaf(A2[s * LA + t], Os[t * LD + x], b);
                    }
#pragma unroll 8
                    for (int y = 0; y < D; ++y) {
                        a = fmaf(Vs[s * LD + y], X[x * D + y], a);
                        b = fmaf(Ks[s * LD + y], X[y * D + x], b);
                    }
                    dk[(row0 + c0 + s) * D + x] = simt::from_f<T>(a);
                    dv[(row0 + c0 + s) * D + x] = simt::from_f<T>(b);
                }
            }
            __syncthreads();
            // G += Q^T dO
            for (int e = tid; e < D * D; e += NUM_THREADS) {
                const int i = e / D, j = e % D;
                float acc = X[e];
                for (int t = 0; t < rows; ++t) acc = fmaf(Qs[t * LD + i], Os[t * LD + j], acc);
                X[e] = acc;
            }
        }
    }
    __syncthreads();
    if (!fwd && p.ds0) {
        float* dst = p.ds0 + u * D * D;
        for (int e = tid; e < D * D; e += NUM_THREADS) dst[e] = X[e];
    }
}

}  // namespace bwd
}  // namespace lcl

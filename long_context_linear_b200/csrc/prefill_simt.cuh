// Chunked causal linear attention on CUDA cores (FFMA, fp32 throughout).
//
// Serves fp32 inputs (where the state must stay within ~1e-4 of the exact
// result, beyond what bf16 tensor-core operands give) and d = 64.  Same tiled
// form as the tensor-core path (page "MiniMax: «Почему M2 в итоге стала моделью
// с полным вниманием?» (конспект)", section 1, glossary entry "Lightning
// Attention"), with chunks of CS tokens:
//   A   = (Q_c K_c^T) ⊙ M        M keeps s <= t
//   O_c = A V_c + Q_c S
//   S  += K_c^T V_c
// One CTA per (unit | sequence, head); the whole d x d fp32 state lives in
// shared memory.  The chunk length CS (32 or 64) is a template parameter.
#pragma once
#include "phi.cuh"
#include <cuda_bf16.h>

namespace lcl {
namespace simt {

constexpr int NUM_THREADS = 256;

struct Params {
    int mode;               // 0 = dense [U][N][d]; 1 = packed [T][H][d]
    int N;                  // dense tokens per unit
    int H;                  // heads (packed)
    const int* cu_seqlens;  // packed
    const float* s0;        // dense: [U][d][d] or null
    const float* pool;      // packed: [n_pool][H][d][d] or null
    const int* init_idx;    // packed: [n_seq] or null
    float* s_out;           // [U | n_seq*H][d][d] or null
    int phi;                // feature map applied to q and k (phi.cuh)
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <int D, int CS>
constexpr int smem_bytes() {
    return (D * D + 3 * CS * (D + 1) + CS * (CS + 1)) * 4;
}

template <typename T, int D, int CS>
__global__ void __launch_bounds__(NUM_THREADS)
prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
                    const Params p) {
    extern __shared__ float sf[];
    float* S = sf;                   // [D][D]
    float* Qs = S + D * D;           // [CS][D+1]
    float* Ks = Qs + CS * (D + 1);
    float* Vs = Ks + CS * (D + 1);
    float* A = Vs + CS * (D + 1);    // [CS][CS+1]
    constexpr int LD = D + 1;
    const int tid = threadIdx.x;

    long row0, row_stride, state;
    int len;
    const float* init = nullptr;
    if (p.mode == 0) {
        const int u = blockIdx.x;
        row0 = (long)u * p.N;
        row_stride = 1;
        len = p.N;
        state = u;
        if (p.s0) init = p.s0 + (long)u * D * D;
    } else {
        const int seq = blockIdx.x / p.H, h = blockIdx.x % p.H;
        const int t0 = p.cu_seqlens[seq];
        len = p.cu_seqlens[seq + 1] - t0;
        row0 = (long)t0 * p.H + h;
        row_stride = p.H;
        state = (long)seq * p.H + h;
        const int ii = p.init_idx ? p.init_idx[seq] : -1;
        if (p.pool && ii >= 0) init = p.pool + ((long)ii * p.H + h) * D * D;
    }
    for (int e = tid; e < D * D; e += NUM_THREADS) S[e] = init ? init[e] : 0.f;

    for (int c0 = 0; c0 < len; c0 += CS) {
        const int rows = min(CS, len - c0);
        __syncthreads();
        for (int e = tid; e < CS * D; e += NUM_THREADS) {
            const int t = e / D, i = e % D;
            float a = 0.f, b = 0.f, cc = 0.f;
            if (t < rows) {
                const long g = (row0 + (long)(c0 + t) * row_stride) * D + i;
                a = apply_phi(to_f(q[g]), p.phi);
                b = apply_phi(to_f(k[g]), p.phi);
                cc = to_f(v[g]);
            }
            Qs[t * LD + i] = a;
            Ks[t * LD + i] = b;
            Vs[t * LD + i] = cc;
        }
        __syncthreads();
        for (int e = tid; e < CS * CS; e += NUM_THREADS) {
            const int t = e / CS, s = e % CS;
            float a = 0.f;
            if (s <= t) {
#pragma unroll 8
                for (int i = 0; i < D; ++i) a = fmaf(Qs[t * LD + i], Ks[s * LD + i], a);
            }
            A[t * (CS + 1) + s] = a;
        }
        __syncthreads();
        for (int e = tid; e < CS * D; e += NUM_THREADS) {
            const int t = e / D, j = e % D;
            if (t < rows) {
                float acc = 0.f;
                for (int s = 0; s <= t; ++s) acc = fmaf(A[t * (CS + 1) + s], Vs[s * LD + j], acc);
#pragma unroll 8
                for (int i = 0; i < D; ++i) acc = fmaf(Qs[t * LD + i], S[i * D + j], acc);
                o[(row0 + (long)(c0 + t) * row_stride) * D + j] = from_f<T>(acc);
            }
        }
        __syncthreads();
        for (int e = tid; e < D * D; e += NUM_THREADS) {
            const int i = e / D, j = e % D;
            float acc = S[e];
            for (int s = 0; s < rows; ++s) acc = fmaf(Ks[s * LD + i], Vs[s * LD + j], acc);
            S[e] = acc;
        }
    }
    __syncthreads();
    if (p.s_out) {
        float* dst = p.s_out + state * D * D;
        for (int e = tid; e < D * D; e += NUM_THREADS) dst[e] = S[e];
    }
}

}  // namespace simt
}  // namespace lcl

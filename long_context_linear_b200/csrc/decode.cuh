// One decode step for a batch of independent states (HBM-bound).
//
// Per (sequence, head): S <- S + k v^T, then o = q S (the recurrence of page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎", one token at a
// time; page "MiniMax: «Почему M2 …»", section 4, notes this is a small state
// matrix that is read and written on every step).  One CTA streams one d x d
// state once: every thread owns one 16-byte vector of E consecutive value
// columns in each of D/RS rows, loads them with streaming loads (all loads
// issued before any use), updates, stores them back, and accumulates its share
// of o; partial sums are reduced across row slots in shared memory.
//
// The state may be stored in fp32, bf16, fp16 or the 8-bit formats e4m3 / e5m2
// (the low-precision state storage the same section warns about).  The update is always computed in
// fp32: S_new = RN_fp32(S_stored + k_i v_j) (one fused multiply-add, the
// product of two bf16 inputs being exact in fp32), then rounded to the storage
// format to nearest even (the 8-bit formats saturate at their largest finite
// value); o uses the stored (rounded) state.  A feature map
// phi (phi.cuh) is applied to q and k as they are loaded.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include "phi.cuh"

namespace lcl {
namespace dec {

constexpr int NUM_THREADS = 256;

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// E values of one 16-byte state vector <-> fp32
template <typename SS> struct Vec;
template <> struct Vec<float> {
    static constexpr int E = 4;
    __device__ __forceinline__ static void unpack(const uint4& r, float (&f)[4]) {
        f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y); f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
    }
    // rounds f to the storage format in place and packs it
    __device__ __forceinline__ static uint4 pack(float (&f)[4]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float (&f)[8]) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(float (&f)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
            f[2 * i] = __low2float(h);
            f[2 * i + 1] = __high2float(h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec<__half> {
    static constexpr int E = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float (&f)[8]) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            f[2 * i] = __low2float(h);
            f[2 * i + 1] = __high2float(h);
        }
    }
    __device__ __forceinline__ static uint4 pack(float (&f)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
            f[2 * i] = __low2float(h);
            f[2 * i + 1] = __high2float(h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// 8-bit formats: 16 values per vector.  fp8 -> half is exact for both formats;
// fp32 -> fp8 is one rounding (to nearest even, saturating).
template <__nv_fp8_interpretation_t I>
struct VecFp8 {
    static constexpr int E = 16;
    __device__ __forceinline__ static float2 dec2(uint32_t pair) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair), I);
        return __half22float2(*reinterpret_cast<const __half2*>(&hr));
    }
    __device__ __forceinline__ static void unpack(const uint4& r, float (&f)[16]) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = dec2(w[i] & 0xffffu), b = dec2(w[i] >> 16);
            f[4 * i] = a.x; f[4 * i + 1] = a.y; f[4 * i + 2] = b.x; f[4 * i + 3] = b.y;
        }
    }
    __device__ __forceinline__ static uint4 pack(float (&f)[16]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t a = __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i], f[4 * i + 1]), __NV_SATFINITE, I);
            const uint32_t b = __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i + 2], f[4 * i + 3]), __NV_SATFINITE, I);
            w[i] = a | (b << 16);
            const float2 da = dec2(a), db = dec2(b);
            f[4 * i] = da.x; f[4 * i + 1] = da.y; f[4 * i + 2] = db.x; f[4 * i + 3] = db.y;
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec<__nv_fp8_e4m3> : VecFp8<__NV_E4M3> {};
template <> struct Vec<__nv_fp8_e5m2> : VecFp8<__NV_E5M2> {};

// Threads per CTA: 16- and 8-bit states are 32 / 16 KB per unit at d = 128,
// so their CTAs are half as wide and twice as many units are in flight per SM
// (measured on B=256, H=64: fp8 5.34 TB/s at 128 threads, 3.34 at 256, 4.46
// at 64; bf16 6.72 TB/s at 128 threads, 6.56 at 256).
template <typename SS>
__host__ __device__ constexpr int decode_threads() { return Vec<SS>::E >= 8 ? NUM_THREADS / 2 : NUM_THREADS; }

// CTAs per SM the register budget is sized for.  8-bit states: 8 (64
// registers, a 60-byte spill) against the 6 that their 80 registers allow
// otherwise; measured 5-7 % faster on B=256, H=64 (e4m3 and e5m2, either
// launch order), with bit-identical states.  16-bit states: 5 (96 registers)
// and fp32: 3 (80): a bound of 1 let the compiler take them to 168 and 96
// registers, which measured 6 % slower (fp32 state 0.338 against 0.319 ms,
// bf16 0.172 against 0.163 ms per step).
template <typename SS>
__host__ __device__ constexpr int decode_min_blocks() {
    return Vec<SS>::E == 16 ? 8 : (Vec<SS>::E == 8 ? 5 : 3);
}

template <typename T, typename SS, int D>
__global__ void __launch_bounds__(decode_threads<SS>(), decode_min_blocks<SS>())
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
                   SS* __restrict__ S, int phi) {
    constexpr int NT = decode_threads<SS>();
    constexpr int E = Vec<SS>::E;          // state values per 16-byte vector
    constexpr int TPR = D / E;             // threads per row
    constexpr int RS = NT / TPR;           // row slots
    constexpr int RPT = D / RS;            // rows per thread
    static_assert(TPR * RS == NT && RS * RPT == D, "thread layout must cover the state exactly");
    __shared__ float qs[D], ks[D], vs[D];
    __shared__ float red[RS][D];

    const long u = blockIdx.x;
    const int tid = threadIdx.x;
    const int cv = tid % TPR;
    const int slot = tid / TPR;
    uint4* Su = reinterpret_cast<uint4*>(S + u * D * D);

    uint4 x[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) x[m] = __ldcs(&Su[(slot + m * RS) * TPR + cv]);
    for (int e = tid; e < D; e += NT) {
        qs[e] = apply_phi(ld_f(q + u * D + e), phi);
        ks[e] = apply_phi(ld_f(k + u * D + e), phi);
        vs[e] = ld_f(v + u * D + e);
    }
    __syncthreads();
    float vj[E], acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        vj[e] = vs[E * cv + e];
        acc[e] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = slot + m * RS;
        const float ki = ks[i], qi = qs[i];
        float y[E];
        Vec<SS>::unpack(x[m], y);
#pragma unroll
        for (int e = 0; e < E; ++e) y[e] = fmaf(ki, vj[e], y[e]);
        __stcs(&Su[i * TPR + cv], Vec<SS>::pack(y));
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(qi, y[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) red[slot][E * cv + e] = acc[e];
    __syncthreads();
    for (int e = tid; e < D; e += NT) {
        float sum = 0.f;
#pragma unroll
        for (int s = 0; s < RS; ++s) sum += red[s][e];
        st_f(o + u * D + e, sum);
    }
}

}  // namespace dec
}  // namespace lcl

// Element-wise feature maps phi for linear attention.
//
// Page "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎", writes
// linear attention as phi(Q) (phi(K)^T V) with a generic element-wise feature
// map phi applied to queries and keys; the recurrence becomes
// S_t = S_{t-1} + phi(k_t) v_t^T, o_t = phi(q_t) S_t.  The library offers the
// identity (the default everywhere), elu(x) + 1 and relu(x), computed in fp32
// (expf for the negative branch of elu + 1).
#pragma once
#include <cuda_bf16.h>

namespace lcl {

enum : int { PHI_IDENTITY = 0, PHI_ELU1 = 1, PHI_RELU = 2 };

__device__ __forceinline__ float apply_phi(float x, int phi) {
    if (phi == PHI_ELU1) return x > 0.f ? x + 1.f : expf(x);
    if (phi == PHI_RELU) return fmaxf(x, 0.f);
    return x;
}

// The same maps for a result that is rounded to bf16 next: exp through the
// hardware ex2 approximation (__expf, relative error far below bf16's 2^-9).
__device__ __forceinline__ float apply_phi_fast(float x, int phi) {
    if (phi == PHI_ELU1) return x > 0.f ? x + 1.f : __expf(x);
    if (phi == PHI_RELU) return fmaxf(x, 0.f);
    return x;
}

// phi on 8 bf16 values packed in 16 bytes, with the result of the fp32
// evaluation above rounded to bf16 (nearest even), in packed bf16 pairs.
// relu is one packed max per pair.  elu + 1 is written as
// exp(min(x, 0)) + max(x, 0): for x <= 0 the bf16 exponential plus zero is
// that exponential, and for x > 0 it is bf16(exp(0)) = 1 plus x, one
// rounding of 1 + x, which is what rounding the fp32 sum gives as well
// (1 + x is exact in fp32 for every bf16 x >= 2^-16, and rounds to 1 either
// way below).
__device__ __forceinline__ uint4 apply_phi_bf16x8(uint4 r, int phi) {
    if (phi != PHI_ELU1 && phi != PHI_RELU) return r;
    const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
    uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        __nv_bfloat162 y = __hmax2(x, zero);
        if (phi == PHI_ELU1) {
            const float2 m = __bfloat1622float2(__hmin2(x, zero));
            y = __hadd2(__floats2bfloat162_rn(__expf(m.x), __expf(m.y)), y);
        }
        w[i] = *reinterpret_cast<const uint32_t*>(&y);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace lcl

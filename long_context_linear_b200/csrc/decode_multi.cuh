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
// for m tokens instead of 2 m with m decode steps.  Commit keeps the layout of
// decode.cuh (thread = one 16-byte column vector of D/RS rows); verify streams
// the rows (below).
#pragma once
#include <cuda_bf16.h>
#include "decode.cuh"
#include "sm100.cuh"

namespace lcl {
namespace dmulti {

constexpr int NUM_THREADS = 256;
constexpr int MAX_M = 16;

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

// 4 values at dst: 16 bytes of fp32 or 8 bytes of bf16 (nearest even)
__device__ __forceinline__ void store4(float* dst, const float4 y) { *reinterpret_cast<float4*>(dst) = y; }
__device__ __forceinline__ void store4(__nv_bfloat16* dst, const float4 y) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(y.x, y.y), b = __floats2bfloat162_rn(y.z, y.w);
    *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

// A piece of S_0: streamed past L1 when one draft group reads it, cached in
// L1 for the other groups when several do.
template <bool kOneGroup>
__device__ __forceinline__ float4 load_s(const float4* p) {
    if constexpr (kOneGroup) return __ldcs(p);
    else return __ldg(p);
}

// verify, one CTA per unit of D / 2 threads per group of DPG drafts (MB / DPG
// groups, MB = 4, 8, 12 or 16 >= m; drafts past m are zero and not stored).
// In each draft group, thread (g, c) owns value columns 4c .. 4c + 3 and rows
// g * D / 2 .. of S_0 in two row groups of D / 4 threads, streams them one
// 16-byte piece per row (8 rows in flight) and updates the q_t S_0 sums of its
// DPG drafts per piece (4 DPG accumulators).  Several draft groups read the
// same pieces (HBM once, L1 or L2 for the others).  q is also stored
// transposed, draft index fastest, so that four drafts' q_i come in one
// broadcast load.  Row group 1 hands its partial sums to row group 0 through
// shared memory; row group 0 adds them and the intra-draft terms and stores o.
// Measured at B=256, H=64 (ms): one group for m <= 12; at m = 16 one group of
// 16 (161 registers, 12 warps per SM) took 0.59, four groups of 4 took 0.77
// (the extra state reads go to L2).
template <typename T, int D, int MB, int DPG>
__global__ void __launch_bounds__(D / 2 * (MB / DPG))
verify_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
              const float* __restrict__ S, int m, int phi) {
    constexpr int LPR = D / 4;     // threads per row group
    constexpr int NG = 2 * LPR;    // threads per draft group
    constexpr int NT = NG * (MB / DPG);
    constexpr int ROWS = D / 2;    // rows per row group
    constexpr int UNR = 8;         // rows in flight per thread
    static_assert(ROWS % UNR == 0 && MB % DPG == 0 && DPG % 4 == 0 && MB <= MAX_M, "verify layout");
    constexpr bool kOne = MB == DPG;
    __shared__ __align__(16) float qT[D][MB];
    __shared__ __align__(16) float qs[MB][D], ks[MB][D], vs[MB][D];
    __shared__ float A[MB][MB];  // A[t][s] = q_t . k_s, s <= t
    float(*red)[D] = qs;         // row group 1's partial sums, once the scores are done with q

    const long u = blockIdx.x;
    const int tid = threadIdx.x, dg = tid / NG, g = (tid % NG) / LPR, c = tid % LPR;
    const int t0 = DPG * dg;  // this thread's drafts t0 .. t0 + DPG - 1
    // the first rows of S_0 are requested before the drafts are read
    const float4* Sg = reinterpret_cast<const float4*>(S + u * D * D) + (long)g * ROWS * LPR + c;
    float4 x[UNR];
#pragma unroll
    for (int j = 0; j < UNR; ++j) x[j] = load_s<kOne>(Sg + (long)j * LPR);
    // the drafts' q, k, v (phi on q and k), zero past m; 16-byte loads
    const long base = u * (long)m * D;
    constexpr int VEC = 16 / (int)sizeof(T);
    for (int e = tid * VEC; e < MB * D; e += NT * VEC) {
        const int t = e / D, i = e % D;
        float qv[VEC], kv[VEC], vv[VEC];
        if (t < m) {
            unpack16(*reinterpret_cast<const uint4*>(q + base + e), qv);
            unpack16(*reinterpret_cast<const uint4*>(k + base + e), kv);
            unpack16(*reinterpret_cast<const uint4*>(v + base + e), vv);
#pragma unroll
            for (int jj = 0; jj < VEC; ++jj) {
                qv[jj] = apply_phi(qv[jj], phi);
                kv[jj] = apply_phi(kv[jj], phi);
            }
        } else {
#pragma unroll
            for (int jj = 0; jj < VEC; ++jj) qv[jj] = kv[jj] = vv[jj] = 0.f;
        }
#pragma unroll
        for (int jj = 0; jj < VEC; jj += 4) {
            *reinterpret_cast<float4*>(&qs[t][i + jj]) = make_float4(qv[jj], qv[jj + 1], qv[jj + 2], qv[jj + 3]);
            *reinterpret_cast<float4*>(&ks[t][i + jj]) = make_float4(kv[jj], kv[jj + 1], kv[jj + 2], kv[jj + 3]);
            *reinterpret_cast<float4*>(&vs[t][i + jj]) = make_float4(vv[jj], vv[jj + 1], vv[jj + 2], vv[jj + 3]);
        }
#pragma unroll
        for (int jj = 0; jj < VEC; ++jj) qT[i + jj][t] = qv[jj];
    }
    __syncthreads();
    // intra-draft scores: one warp per pair (t, s), s <= t, lanes split the dim
    {
        constexpr int NW = NT / 32 > 0 ? NT / 32 : 1;
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
    __syncthreads();  // qs is reused for the partial sums below
    // q_t S_0 over this row group's rows for the thread's drafts
    float4 acc[DPG];
#pragma unroll
    for (int t = 0; t < DPG; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int r0 = 0; r0 < ROWS; r0 += UNR) {
        if (r0 > 0) {
#pragma unroll
            for (int j = 0; j < UNR; ++j) x[j] = load_s<kOne>(Sg + (long)(r0 + j) * LPR);
        }
#pragma unroll
        for (int j = 0; j < UNR; ++j) {
            const float* qrow = qT[g * ROWS + r0 + j] + t0;
#pragma unroll
            for (int t4 = 0; t4 < DPG; t4 += 4) {
                const float4 qq = *reinterpret_cast<const float4*>(qrow + t4);
                const float qa[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    float4& a = acc[t4 + tt];
                    a.x = fmaf(qa[tt], x[j].x, a.x);
                    a.y = fmaf(qa[tt], x[j].y, a.y);
                    a.z = fmaf(qa[tt], x[j].z, a.z);
                    a.w = fmaf(qa[tt], x[j].w, a.w);
                }
            }
        }
    }
    if (g == 1) {
#pragma unroll
        for (int tt = 0; tt < DPG; ++tt) *reinterpret_cast<float4*>(&red[t0 + tt][4 * c]) = acc[tt];
    }
    __syncthreads();
    if (g == 0) {
#pragma unroll
        for (int tt = 0; tt < DPG; ++tt) {
            const int t = t0 + tt;
            if (t < m) {
                const float4 p = *reinterpret_cast<const float4*>(&red[t][4 * c]);
                float4 y = make_float4(acc[tt].x + p.x, acc[tt].y + p.y, acc[tt].z + p.z, acc[tt].w + p.w);
                for (int s = 0; s <= t; ++s) {
                    const float a = A[t][s];
                    const float4 vv = *reinterpret_cast<const float4*>(&vs[s][4 * c]);
                    y.x = fmaf(a, vv.x, y.x);
                    y.y = fmaf(a, vv.y, y.y);
                    y.z = fmaf(a, vv.z, y.z);
                    y.w = fmaf(a, vv.w, y.w);
                }
                store4(o + base + (long)t * D + 4 * c, y);
            }
        }
    }
}

// verify on the tensor cores, bf16 q, k, v at d = 128 (fp32 S_0), one CTA of
// 128 threads per unit.  The inter-draft part is one product per unit,
//   O^T = bf16(S_0)^T Q^T    (M = 128 value columns, N = 16 drafts, K = 128),
// with bf16(S_0) as the operand and fp32 accumulation -- the same reading as
// the prefill's Q S product -- so that the tensor cores, not the FMA pipes,
// carry the m d^2 work whatever m is.  The threads convert S_0 to bf16 in the
// MN-major 128B-swizzled layout (row i of S_0 is K-step row i, two 64-column
// panels), Q (zero past m) to a K-major tile of 16 rows, one thread issues the
// 8 tcgen05.mma, and thread j reads column j of O^T (16 drafts) from TMEM,
// adds the intra-draft terms sum_{s <= t} (q_t . k_s) v_s in fp32 and stores.
// phi(q) and phi(k) are rounded to bf16 (tensor-core operands) for the scores
// too, as on the tensor-core prefill.
constexpr int TC_THREADS = 128;

__global__ void __launch_bounds__(TC_THREADS)
verify_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ o, const float* __restrict__ S,
                 int m, int phi, int* status) {
    constexpr int D = 128, MT = 16;                  // value columns, draft rows of the product
    constexpr int PANEL_S = D * 128;                 // 128 rows x 128 bytes: 64 value columns of bf16(S)
    constexpr int PANEL_Q = MT * 128;                // 16 rows x 128 bytes: 64 key dims of q
    __shared__ __align__(1024) uint8_t s_tile[2 * PANEL_S];
    __shared__ __align__(1024) uint8_t q_tile[2 * PANEL_Q];
    __shared__ __align__(16) __nv_bfloat16 ksb[MT][D];  // bf16(phi(k)) of the drafts, for the scores
    __shared__ __align__(16) __nv_bfloat16 qsb[MT][D];  // bf16(phi(q))
    __shared__ float A[MT][MT];                      // A[t][s] = q_t . k_s, s <= t
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_holder;

    const long u = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float4* Su = reinterpret_cast<const float4*>(S + u * D * D);
    // S_0 -> bf16 tile: warp w converts rows w, w + 4, ...; lane c holds columns 4c .. 4c + 3
    {
        const int c = lane;
        const uint32_t panel = static_cast<uint32_t>(c >> 4) * PANEL_S;
        const uint32_t chunk = static_cast<uint32_t>((c & 15) >> 1), half = static_cast<uint32_t>(c & 1) * 8u;
        const uint32_t sb = smem_u32(s_tile) + panel + half;
#pragma unroll 4
        for (int r0 = 0; r0 < D; r0 += 32) {
            float4 x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = __ldcs(Su + (long)(r0 + 4 * j + warp) * (D / 4) + c);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t row = static_cast<uint32_t>(r0 + 4 * j + warp);
                const uint32_t a = sb + row * 128u + ((chunk ^ (row & 7u)) << 4);
                asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(pack_bf16x2(x[j].x, x[j].y)),
                             "r"(pack_bf16x2(x[j].z, x[j].w))
                             : "memory");
            }
        }
    }
    // the drafts: phi(q) as a K-major bf16 tile and in fp32, phi(k) and v in fp32
    const long base = u * (long)m * D;
    for (int e = tid * 8; e < MT * D; e += TC_THREADS * 8) {
        const int t = e / D, i = e % D;
        float qv[8], kv[8];
        if (t < m) {
            unpack16(*reinterpret_cast<const uint4*>(q + base + e), qv);
            unpack16(*reinterpret_cast<const uint4*>(k + base + e), kv);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                qv[jj] = apply_phi(qv[jj], phi);
                kv[jj] = apply_phi(kv[jj], phi);
            }
        } else {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) qv[jj] = kv[jj] = 0.f;
        }
        const uint4 qp = make_uint4(pack_bf16x2(qv[0], qv[1]), pack_bf16x2(qv[2], qv[3]), pack_bf16x2(qv[4], qv[5]),
                                    pack_bf16x2(qv[6], qv[7]));
        *reinterpret_cast<uint4*>(&qsb[t][i]) = qp;
        *reinterpret_cast<uint4*>(&ksb[t][i]) = make_uint4(pack_bf16x2(kv[0], kv[1]), pack_bf16x2(kv[2], kv[3]),
                                                           pack_bf16x2(kv[4], kv[5]), pack_bf16x2(kv[6], kv[7]));
        // the same 8 bf16 of row t, key dims i .. i + 7, as one 16-byte chunk of the K-major tile
        const uint32_t qa = smem_u32(q_tile) + static_cast<uint32_t>(i >> 6) * PANEL_Q + static_cast<uint32_t>(t) * 128u +
                            ((static_cast<uint32_t>((i & 63) >> 3) ^ static_cast<uint32_t>(t & 7)) << 4);
        st_shared_v4(qa, qp.x, qp.y, qp.z, qp.w);
    }
    fence_proxy_async_smem();
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_holder, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_holder;
    if (tid == 0) {
        constexpr uint32_t id = idesc_bf16(128, MT, 1, 0);  // A = bf16(S_0)^T MN-major, B = Q^T K-major
        const uint64_t da = sw128_desc(smem_u32(s_tile), PANEL_S, 1024);
        const uint64_t db = sw128_desc(smem_u32(q_tile), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a_step = static_cast<uint64_t>(kk) * (2048u >> 4);
            const uint64_t b_step = static_cast<uint64_t>((static_cast<uint32_t>(kk >> 2) * PANEL_Q + static_cast<uint32_t>(kk & 3) * 32u) >> 4);
            mma_ss(tbase, da + a_step, db + b_step, id, kk > 0);
        }
        mma_commit(&bar);
    }
    // intra-draft scores while the product runs: one warp per pair (t, s), s <= t
    {
        int t = 0, s = warp;
        while (s > t) { s -= t + 1; ++t; }
        for (; t < m;) {
            float a = 0.f;
#pragma unroll
            for (int i = lane; i < D; i += 32) a = fmaf(__bfloat162float(qsb[t][i]), __bfloat162float(ksb[s][i]), a);
#pragma unroll
            for (int off = 16; off; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
            if (lane == 0) A[t][s] = a;
            s += TC_THREADS / 32;
            while (s > t) { s -= t + 1; ++t; }
        }
    }
    __syncthreads();
    // O^T column j = tid: 16 drafts from TMEM (lane j), then the intra-draft terms
    bool ok = true;
    {
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(&bar, 0)) {
            if (globaltimer() - t0 > kWaitTimeoutNs) {
                atomicExch(status, kStatusTimeout);
                ok = false;
                break;
            }
        }
    }
    tc_fence_after();
    uint32_t r[16];
    tmem_ld16(tbase + (static_cast<uint32_t>(warp * 32) << 16), r);
    tmem_wait_ld();
    if (ok) {
        const int j = tid;
        float vj[MT];
#pragma unroll
        for (int s = 0; s < MT; ++s) vj[s] = s < m ? __bfloat162float(v[base + (long)s * D + j]) : 0.f;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (t < m) {
                float y = __uint_as_float(r[t]);
#pragma unroll
                for (int s = 0; s <= t; ++s) y = fmaf(A[t][s], vj[s], y);
                o[base + (long)t * D + j] = __float2bfloat16_rn(y);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 32);
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

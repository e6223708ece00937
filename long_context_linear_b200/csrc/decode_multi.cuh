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

// verify on the tensor cores, persistent: bf16 q, k, v at d = 128, fp32 S_0.
// One CTA of 128 threads per SM walks the units u = blockIdx.x + n gridDim.x.
// Thread 32 (lane 0 of warp 1) streams each unit's S_0 (four 32-column fp32 panels by TMA, in the
// 128-byte swizzle of 32-byte atoms: the layout the tensor cores take for an
// MN-major tf32 operand) and its v rows (a plain bulk copy) into one of three
// slots, up to three units ahead of the one being computed, so that about
// 128 KB of state is in flight per SM and the state never passes through
// registers; the threads fetch the next unit's q and k rows into registers
// while the current unit computes.  The inter-draft part is one tcgen05
// product per unit on the fp32 tiles read as tf32,
//   O^T = S_0^T Q^T    (M = 128 value columns, N = 16 drafts, K = 128 key dims),
// with fp32 accumulation in TMEM; meanwhile the threads form the scores
// A[t][s] = phi(q_t) . phi(k_s) in fp32, and thread j then reads column j of
// O^T from TMEM, adds sum_{s <= t} A[t][s] v_s[j] and stores o_t[j].
namespace vtf {
constexpr int THREADS = 128, D = 128, MT = 16, SLOTS = 3;
constexpr uint32_t PANEL_S = 128 * 128;                 // 128 key rows x 128 bytes: 32 value columns of fp32
constexpr uint32_t SLOT_S = 4 * PANEL_S;                // S_0 of one unit, 64 KB
constexpr uint32_t ROWS = MT * D * 2;                   // room for 16 draft rows of bf16 (v)
constexpr uint32_t SLOT = SLOT_S + ROWS;
constexpr uint32_t PANEL_Q = MT * 128;                  // 16 draft rows x 128 bytes: 32 key dims of fp32
constexpr uint32_t OFF_QT = SLOTS * SLOT;               // phi(q), K-major 128B-swizzled B operand
constexpr uint32_t OFF_KF = OFF_QT + 4 * PANEL_Q;       // phi(k) row-major fp32, for the scores
constexpr uint32_t OFF_A = OFF_KF + MT * D * 4;         // A[t][s]
constexpr uint32_t OFF_BAR = OFF_A + MT * MT * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;    // + alignment slack
static_assert(SLOT % 1024 == 0 && OFF_QT % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
}  // namespace vtf

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, int* status) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kWaitTimeoutNs) {
            atomicExch(status, kStatusTimeout);
            return false;
        }
    }
    return true;
}

__global__ void __launch_bounds__(vtf::THREADS, 1)
verify_tf32_kernel(const __grid_constant__ CUtensorMap ms, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                   __nv_bfloat16* __restrict__ o, long U, int m, int phi, int* status) {
    using namespace vtf;
    extern __shared__ uint8_t raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);  // [SLOTS]
    uint64_t* mma_bar = full + SLOTS;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(full + SLOTS + 1);
    float* kf = reinterpret_cast<float*>(sm + OFF_KF);
    float* A = reinterpret_cast<float*>(sm + OFF_A);
    const uint32_t qt = smem_u32(sm + OFF_QT);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t row_bytes = static_cast<uint32_t>(m) * D * 2;

    // thread 32: S_0 and v of unit n of this CTA into slot n % SLOTS
    auto issue = [&](long n) {
        const long u = blockIdx.x + n * gridDim.x;
        if (u >= U) return;
        const int sl = static_cast<int>(n % SLOTS);
        uint8_t* dst = sm + sl * SLOT;
        mbar_arrive_expect_tx(&full[sl], SLOT_S + row_bytes);
#pragma unroll
        for (int p = 0; p < 4; ++p) tma_load_3d(dst + p * PANEL_S, &ms, &full[sl], 32 * p, 0, static_cast<int>(u));
        bulk_load(dst + SLOT_S, v + u * static_cast<long>(m) * D, row_bytes, &full[sl]);
    };
    // every thread: its 8-value pieces of the q and k rows of unit u
    uint4 pq[2], pk[2];
    auto fetch = [&](long u) {
        if (u >= U) return;
        const uint4* q4 = reinterpret_cast<const uint4*>(q + u * static_cast<long>(m) * D);
        const uint4* k4 = reinterpret_cast<const uint4*>(k + u * static_cast<long>(m) * D);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = tid * 8 + r * THREADS * 8;
            if (e < m * D) {
                pq[r] = __ldcs(q4 + e / 8);
                pk[r] = __ldcs(k4 + e / 8);
            }
        }
    };

    if (tid == 0) {
        prefetch_tmap(&ms);
        for (int i = 0; i < SLOTS; ++i) mbar_init(&full[i], 1);
        mbar_init(mma_bar, 1);
        fence_barrier_init();
    }
    // draft rows m .. 15 of the B tile stay zero
    for (uint32_t e = tid * 16; e < 4 * PANEL_Q; e += THREADS * 16) st_shared_v4(qt + e, 0, 0, 0, 0);
    if (warp == 0) {
        tmem_alloc(tmem_holder, 32);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    if (tid == 32)
        for (int i = 0; i < SLOTS; ++i) issue(i);
    fetch(blockIdx.x);
    constexpr uint32_t idesc = idesc_tf32(128, MT, 1, 0);  // A = S_0^T MN-major, B = Q^T K-major
    long n = 0;
    bool ok = true;
    for (;; ++n) {
        const long u = blockIdx.x + n * gridDim.x;
        if (u >= U) break;
        const int sl = static_cast<int>(n % SLOTS);
        // phi(q) into the swizzled B tile, phi(k) into kf (8 values a piece)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = tid * 8 + r * THREADS * 8;
            if (e < m * D) {
                const int t = e >> 7, i = e & (D - 1);
                float x[8], y[8];
                unpack16(pq[r], x);
                unpack16(pk[r], y);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    x[jj] = apply_phi(x[jj], phi);
                    y[jj] = apply_phi(y[jj], phi);
                }
                float4* kr = reinterpret_cast<float4*>(kf + e);
                kr[0] = make_float4(y[0], y[1], y[2], y[3]);
                kr[1] = make_float4(y[4], y[5], y[6], y[7]);
                const uint32_t qa = qt + static_cast<uint32_t>(i >> 5) * PANEL_Q + static_cast<uint32_t>(t) * 128u;
                const uint32_t c0 = static_cast<uint32_t>((i & 31) >> 2), sw = static_cast<uint32_t>(t & 7);
                st_shared_v4(qa + ((c0 ^ sw) << 4), __float_as_uint(x[0]), __float_as_uint(x[1]),
                             __float_as_uint(x[2]), __float_as_uint(x[3]));
                st_shared_v4(qa + (((c0 + 1) ^ sw) << 4), __float_as_uint(x[4]), __float_as_uint(x[5]),
                             __float_as_uint(x[6]), __float_as_uint(x[7]));
            }
        }
        fetch(u + gridDim.x);
        ok = wait_bounded(&full[sl], static_cast<uint32_t>((n / SLOTS) & 1), status);
        fence_proxy_async_smem();
        tc_fence_before();
        if (!__syncthreads_and(ok)) {
            ok = false;
            break;
        }
        tc_fence_after();
        if (tid == 0) {
            // S_0 panels: 32 value columns x 128 key rows, 4-row groups 512 bytes apart
            const uint64_t da = sw128b32_desc(smem_u32(sm + sl * SLOT), PANEL_S, 512);
            const uint64_t db = sw128_desc(qt, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk) {
                // K = 8 per product: 8 key rows (1 KB) of the S_0 panels, 32 bytes of a Q row
                const uint64_t a_step = static_cast<uint64_t>(kk) * (1024u >> 4);
                const uint64_t b_step =
                    static_cast<uint64_t>((static_cast<uint32_t>(kk >> 2) * PANEL_Q + static_cast<uint32_t>(kk & 3) * 32u) >> 4);
                mma_ss_tf32(tbase, da + a_step, db + b_step, idesc, kk > 0);
            }
            mma_commit(mma_bar);
        }
        // intra-draft scores while the product runs, on threads 32 .. 111 (not
        // the one issuing it): the lower triangle of 4 x 4 blocks of (t, s),
        // 8 threads a block, each over the key dims 4 (p + 8 c) .. + 3,
        // c = 0 .. 3 (so the 8 threads of a shared-memory phase read 8
        // different bank groups), summed across the 8 by shuffles
        {
            const int w = tid - 32;
            if (w >= 0 && w < 80) {
                int tb = 0, sb = w >> 3;
                while (sb > tb) {
                    sb -= tb + 1;
                    ++tb;
                }
                const int part = w & 7;
                if (4 * tb < m) {
                    float acc[4][4];
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t cc = static_cast<uint32_t>(part + 8 * c);
                        float4 xa[4], yb[4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const uint32_t t = static_cast<uint32_t>(4 * tb + a);
                            const uint4 x = ld_shared_v4(qt + (cc >> 3) * PANEL_Q + t * 128u + (((cc & 7u) ^ (t & 7u)) << 4));
                            xa[a] = make_float4(__uint_as_float(x.x), __uint_as_float(x.y), __uint_as_float(x.z),
                                                __uint_as_float(x.w));
                        }
#pragma unroll
                        for (int b = 0; b < 4; ++b) yb[b] = reinterpret_cast<const float4*>(kf + (4 * sb + b) * D)[cc];
#pragma unroll
                        for (int a = 0; a < 4; ++a)
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                acc[a][b] = fmaf(xa[a].x, yb[b].x, acc[a][b]);
                                acc[a][b] = fmaf(xa[a].y, yb[b].y, acc[a][b]);
                                acc[a][b] = fmaf(xa[a].z, yb[b].z, acc[a][b]);
                                acc[a][b] = fmaf(xa[a].w, yb[b].w, acc[a][b]);
                            }
                    }
                    const unsigned grp = 0xFFu << (lane & 24);
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            float x = acc[a][b];
                            x += __shfl_xor_sync(grp, x, 4);
                            x += __shfl_xor_sync(grp, x, 2);
                            x += __shfl_xor_sync(grp, x, 1);
                            acc[a][b] = x;
                        }
                    if (part == 0)
#pragma unroll
                        for (int a = 0; a < 4; ++a)
                            *reinterpret_cast<float4*>(A + (4 * tb + a) * MT + 4 * sb) =
                                make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
                }
            }
        }
        __syncthreads();
        ok = wait_bounded(mma_bar, static_cast<uint32_t>(n & 1), status);
        if (!__syncthreads_and(ok)) {
            ok = false;
            break;
        }
        tc_fence_after();
        uint32_t r[16];
        tmem_ld16(tbase + (static_cast<uint32_t>(warp * 32) << 16), r);
        {
            const int j = tid;
            const __nv_bfloat16* vs = reinterpret_cast<const __nv_bfloat16*>(sm + sl * SLOT + SLOT_S);
            float vj[MT];
#pragma unroll
            for (int s = 0; s < MT; ++s) vj[s] = s < m ? __bfloat162float(vs[s * D + j]) : 0.f;
            tmem_wait_ld();
            const long base = u * static_cast<long>(m) * D;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t < m) {
                    float y = __uint_as_float(r[t]);
                    const float4* a4 = reinterpret_cast<const float4*>(A + t * MT);
#pragma unroll
                    for (int s4 = 0; s4 <= t / 4; ++s4) {
                        const float4 a = a4[s4];
                        y = fmaf(a.x, vj[4 * s4], y);
                        if (4 * s4 + 1 <= t) y = fmaf(a.y, vj[4 * s4 + 1], y);
                        if (4 * s4 + 2 <= t) y = fmaf(a.z, vj[4 * s4 + 2], y);
                        if (4 * s4 + 3 <= t) y = fmaf(a.w, vj[4 * s4 + 3], y);
                    }
                    o[base + static_cast<long>(t) * D + j] = __float2bfloat16_rn(y);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 32) issue(n + SLOTS);
    }
    if (!ok && tid == 32) {
        // copies still in flight land before the CTA's shared memory is released
        for (long x = n; x < n + SLOTS; ++x)
            if (blockIdx.x + x * gridDim.x < U)
                if (!wait_bounded(&full[x % SLOTS], static_cast<uint32_t>((x / SLOTS) & 1), status)) break;
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

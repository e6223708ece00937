// Chunked causal linear attention on CUDA cores (FFMA, fp32 throughout).
//
// Serves fp32 inputs (where the state must stay within ~1e-4 of the exact
// result, beyond what bf16 tensor-core operands give).  Same tiled
// form as the tensor-core path (page "MiniMax: «Почему M2 в итоге стала моделью
// с полным вниманием?» (конспект)", section 1, glossary entry "Lightning
// Attention"), with chunks of CS tokens:
//   A   = (Q_c K_c^T) ⊙ M        M keeps s <= t
//   O_c = A V_c + Q_c S
//   S  += K_c^T V_c
// One CTA per (unit | segment of a unit | sequence, head), 256 threads; a
// segment starts from a given state, and a state-only launch sums K^T V over
// its segments without reading Q or writing outputs.  Every product is
// register-tiled (each thread owns a block of outputs and reads 16-byte
// vectors from shared memory), tiles wholly above the causal diagonal are
// skipped, the state S stays in the registers of its owner threads between
// chunks (and in shared memory for Q S), and the next chunk is prefetched into
// L2 while this one is loaded.  The chunk length CS (32 or 64) is a template
// parameter.
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
    // dense only: visit the chunks last to first and keep s >= t inside a
    // chunk, so that o_t = q_t (S_init + sum_{s >= t} k_s v_s^T)
    int reverse;
    int init_transposed;    // the initial state is given as its transpose [d][d]
    // dense only: each unit's sequence cut into segments of seg_len tokens; a
    // launch covers segments seg_base .. seg_base + n_seg - 1 of every unit
    // (CTA = unit * n_seg + j); n_seg = 0 means whole sequences
    int n_seg;
    int seg_len;
    int seg_base;
    const float* seg_init;  // [U][n_seg][d][d]: state before each segment, or null
    int s_out_per_seg;      // 1: s_out is [U][n_seg][d][d], one state per segment
    int state_only;         // 1: only S = (init) + sum K^T V over the segment
    // packed only: segments of *seg_len_dev tokens, CTA = segment * H + head,
    // with the segments numbered in the work order of `order` (the length and
    // the offsets over n_seq sequences from vorder::seg_plan_kernel); a state-only launch numbers
    // only the segments that are not a sequence's last (seg_off_nl).  CTAs past
    // the device-side total (the host launches an upper bound) do nothing.
    const int* order;
    const int* seg_off;
    const int* seg_off_nl;
    const int* seg_len_dev;
    int n_seq;
};

// Shared-memory layout (floats), rows padded by 4 so that 16-byte vectors
// stay aligned and successive rows start in different banks:
//   Qt, Kt [D][CS+4]   Q and K transposed (token index contiguous)
//   Kn, Vn [CS][D+4]   K and V as stored (K twice: the scores read it by key
//                      dimension, the state update by token)
//   At     [CS][CS+4]  masked scores, transposed: At[s][t] = (q_t . k_s) [s <= t]
//   Sm     [D][D+4]    the state before this chunk
template <int D, int CS>
constexpr int smem_bytes() {
    return (2 * D * (CS + 4) + 2 * CS * (D + 4) + CS * (CS + 4) + D * (D + 4)) * 4;
}
static_assert(smem_bytes<128, 64>() <= 232448, "exceeds the 227 KB per-block shared memory limit");

// Register tiles: the 256 threads form a 16 x 16 grid (ty = tid / 16 picks
// the tile row, tx = tid % 16 the tile column); each thread owns TM x TN
// outputs of a product.  Tile rows are a contiguous block (ty*TM ...); tile
// columns come in groups of 4 spread N / (TN/4) apart (tx*4 ... within each
// group), so that the 16 threads of a row read one contiguous stretch per
// 16-byte load.
template <int TN, int N>
__device__ __forceinline__ int col_of(int tx, int c) {
    if constexpr (TN >= 4) return (c / 4) * (N / (TN / 4)) + tx * 4 + (c % 4);
    else return tx * TN + c;
}

// TN values of one row for thread column tx
template <int TN, int N>
__device__ __forceinline__ void ld_cols(const float* row, int tx, float (&x)[TN]) {
    if constexpr (TN >= 4) {
#pragma unroll
        for (int g = 0; g < TN / 4; ++g) {
            const float4 v = *reinterpret_cast<const float4*>(row + g * (N / (TN / 4)) + tx * 4);
            x[4 * g] = v.x; x[4 * g + 1] = v.y; x[4 * g + 2] = v.z; x[4 * g + 3] = v.w;
        }
    } else {
        const float2 v = *reinterpret_cast<const float2*>(row + tx * 2);
        x[0] = v.x; x[1] = v.y;
    }
}
template <int TN, int N>
__device__ __forceinline__ void st_cols(float* row, int tx, const float (&x)[TN]) {
    if constexpr (TN >= 4) {
#pragma unroll
        for (int g = 0; g < TN / 4; ++g)
            *reinterpret_cast<float4*>(row + g * (N / (TN / 4)) + tx * 4) =
                make_float4(x[4 * g], x[4 * g + 1], x[4 * g + 2], x[4 * g + 3]);
    } else {
        *reinterpret_cast<float2*>(row + tx * 2) = make_float2(x[0], x[1]);
    }
}
// TM contiguous values (TM = 2, 4 or 8) at p, 8-byte aligned at least
template <int TM>
__device__ __forceinline__ void ld_run(const float* p, float (&x)[TM]) {
    if constexpr (TM % 4 == 0) {
#pragma unroll
        for (int g = 0; g < TM / 4; ++g) {
            const float4 v = *reinterpret_cast<const float4*>(p + 4 * g);
            x[4 * g] = v.x; x[4 * g + 1] = v.y; x[4 * g + 2] = v.z; x[4 * g + 3] = v.w;
        }
    } else {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    }
}
template <int TM>
__device__ __forceinline__ void st_run(float* p, const float (&x)[TM]) {
    if constexpr (TM % 4 == 0) {
#pragma unroll
        for (int g = 0; g < TM / 4; ++g)
            *reinterpret_cast<float4*>(p + 4 * g) = make_float4(x[4 * g], x[4 * g + 1], x[4 * g + 2], x[4 * g + 3]);
    } else {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    }
}

// 16 bytes of T -> fp32
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
// 4 outputs -> T at p (16 bytes for fp32, 8 for bf16)
__device__ __forceinline__ void store4(float* p, const float* x) { *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]); }
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* x) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}
__device__ __forceinline__ void store2(float* p, const float* x) { *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]); }
__device__ __forceinline__ void store2(__nv_bfloat16* p, const float* x) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    *reinterpret_cast<uint32_t*>(p) = *reinterpret_cast<const uint32_t*>(&a);
}

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

template <typename T, int D, int CS>
__global__ void __launch_bounds__(NUM_THREADS, 1)
prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ o,
                    const Params p) {
    static_assert(CS == 32 || CS == 64, "chunk of 32 or 64 tokens");
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    constexpr int LQ = CS + 4, LV = D + 4;
    constexpr int TM1 = CS / 16, TN1 = CS / 16;   // scores   [CS x CS]
    constexpr int TM2 = CS / 16, TN2 = D / 16;    // outputs  [CS x D]
    constexpr int TM3 = D / 16, TN3 = D / 16;     // state    [D x D]
    constexpr int VEC = 16 / sizeof(T);           // elements per 16-byte global load
    constexpr int VPR = D / VEC;                  // 16-byte vectors per row
    extern __shared__ float sf[];
    float* Qt = sf;
    float* Kt = Qt + D * LQ;
    float* Kn = Kt + D * LQ;
    float* Vn = Kn + CS * LV;
    float* At = Vn + CS * LV;
    float* Sm = At + CS * LQ;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

    long row0, row_stride, state;
    int len;
    bool write_state = true;
    bool init_t = p.init_transposed;
    const float* init = nullptr;
    if (p.mode == 0 && p.n_seg > 0) {
        // segment seg of unit u: tokens seg * seg_len .. (the last one may be shorter)
        const int u = blockIdx.x / p.n_seg, j = blockIdx.x % p.n_seg, seg = p.seg_base + j;
        const int t0 = seg * p.seg_len, n_all = (p.N + p.seg_len - 1) / p.seg_len;
        row0 = (long)u * p.N + t0;
        row_stride = 1;
        len = min(p.seg_len, p.N - t0);
        state = p.s_out_per_seg ? (long)u * p.n_seg + j : u;
        // without one state per segment only the segment visited last writes S
        write_state = p.s_out_per_seg || (p.reverse ? seg == 0 : seg == n_all - 1);
        if (p.seg_init) {
            init = p.seg_init + ((long)u * p.n_seg + j) * D * D;
            init_t = false;
        } else if (p.s0) {
            init = p.s0 + (long)u * D * D;
        }
    } else if (p.mode == 0) {
        const int u = blockIdx.x;
        row0 = (long)u * p.N;
        row_stride = 1;
        len = p.N;
        state = u;
        if (p.s0) init = p.s0 + (long)u * D * D;
    } else if (p.seg_off) {
        const int* off = p.state_only ? p.seg_off_nl : p.seg_off;
        const int sgi = blockIdx.x / p.H, h = blockIdx.x % p.H;
        if (sgi >= off[p.n_seq]) return;  // past the total: the whole CTA leaves before any barrier
        int lo = 0, hi = p.n_seq;         // rank r with off[r] <= sgi < off[r + 1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (off[mid] <= sgi) lo = mid;
            else hi = mid;
        }
        const int seq = p.order[lo], sl = *p.seg_len_dev;
        const int t0 = p.cu_seqlens[seq] + (sgi - off[lo]) * sl;
        len = max(0, min(sl, p.cu_seqlens[seq + 1] - t0));
        row0 = (long)t0 * p.H + h;
        row_stride = p.H;
        if (p.state_only) {
            state = (long)sgi * p.H + h;  // index of this segment's sum
        } else {
            state = (long)seq * p.H + h;
            init = p.seg_init + ((long)sgi * p.H + h) * D * D;
            init_t = false;
            write_state = sgi == off[lo + 1] - 1;  // the sequence's last segment
        }
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
    // the state tile of this thread: rows ty*TM3 + r, columns col_of<TN3, D>(tx, c)
    float accS[TM3][TN3];
#pragma unroll
    for (int r = 0; r < TM3; ++r) {
        const int i = ty * TM3 + r;
#pragma unroll
        for (int c = 0; c < TN3; ++c) {
            const int j = col_of<TN3, D>(tx, c);
            accS[r][c] = init ? init[init_t ? j * D + i : i * D + j] : 0.f;
        }
        st_cols<TN3, D>(Sm + i * LV, tx, accS[r]);
    }

    const bool rev = p.reverse;
    const bool state_only = p.state_only;
    const int nc = (len + CS - 1) / CS;
    for (int ci = 0; ci < nc; ++ci) {
        const int c0 = (rev ? nc - 1 - ci : ci) * CS;
        const int rows = min(CS, len - c0);
        __syncthreads();  // the previous chunk is done with Qt, Kt, Vn, At and Sm
        // ---- next chunk into L2, this chunk into shared memory (phi on q and k)
        if (ci + 1 < nc) {
            constexpr int LINES = D * (int)sizeof(T) / 128;
            const int n0 = (rev ? nc - 2 - ci : ci + 1) * CS;
            const int nrows = min(CS, len - n0);
            const int first = state_only ? 1 : 0;  // q is not read for the state alone
            for (int f = tid + first * nrows * LINES; f < 3 * nrows * LINES; f += NUM_THREADS) {
                const int which = f / (nrows * LINES), rl = f % (nrows * LINES);
                const long g = (row0 + (long)(n0 + rl / LINES) * row_stride) * D;
                const T* src = which == 0 ? q : (which == 1 ? k : v);
                prefetch_l2(src + g + (rl % LINES) * (128 / (int)sizeof(T)));
            }
        }
        for (int f = tid; f < CS * VPR; f += NUM_THREADS) {
            const int t = f / VPR, cc = (f % VPR) * VEC;
            float qv[VEC], kv[VEC], vv[VEC];
            if (t < rows) {
                const long g = (row0 + (long)(c0 + t) * row_stride) * D + cc;
                if (!state_only) {
                    unpack16(*reinterpret_cast<const uint4*>(q + g), qv);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) qv[e] = 0.f;
                }
                unpack16(*reinterpret_cast<const uint4*>(k + g), kv);
                unpack16(*reinterpret_cast<const uint4*>(v + g), vv);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    qv[e] = apply_phi(qv[e], p.phi);
                    kv[e] = apply_phi(kv[e], p.phi);
                }
            } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) qv[e] = kv[e] = vv[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                Qt[(cc + e) * LQ + t] = qv[e];
                Kt[(cc + e) * LQ + t] = kv[e];
            }
#pragma unroll
            for (int e = 0; e < VEC; e += 4) {
                *reinterpret_cast<float4*>(Kn + t * LV + cc + e) = make_float4(kv[e], kv[e + 1], kv[e + 2], kv[e + 3]);
                *reinterpret_cast<float4*>(Vn + t * LV + cc + e) = make_float4(vv[e], vv[e + 1], vv[e + 2], vv[e + 3]);
            }
        }
        __syncthreads();
        // ---- scores: At[s][t] = q_t . k_s for s <= t (s >= t in reverse), else 0
        if (!state_only) {
            const int t0 = ty * TM1, s0 = tx * TN1;
            float acc[TM1][TN1];
#pragma unroll
            for (int r = 0; r < TM1; ++r)
#pragma unroll
                for (int c = 0; c < TN1; ++c) acc[r][c] = 0.f;
            if (rev ? s0 + TN1 - 1 >= t0 : s0 <= t0 + TM1 - 1) {  // the tile holds kept entries
#pragma unroll 4
                for (int i = 0; i < D; ++i) {
                    float a[TM1], b[TN1];
                    ld_run<TM1>(Qt + i * LQ + t0, a);
                    ld_run<TN1>(Kt + i * LQ + s0, b);
#pragma unroll
                    for (int r = 0; r < TM1; ++r)
#pragma unroll
                        for (int c = 0; c < TN1; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
                }
            }
#pragma unroll
            for (int c = 0; c < TN1; ++c) {
                float col[TM1];
#pragma unroll
                for (int r = 0; r < TM1; ++r) col[r] = (rev ? s0 + c >= t0 + r : s0 + c <= t0 + r) ? acc[r][c] : 0.f;
                st_run<TM1>(At + (s0 + c) * LQ + t0, col);
            }
        }
        __syncthreads();
        // ---- outputs: O_t = sum_s At[s][t] v_s + q_t S (s <= t, or s >= t in reverse)
        if (!state_only) {
            const int t0 = ty * TM2;
            float acc[TM2][TN2];
#pragma unroll
            for (int r = 0; r < TM2; ++r)
#pragma unroll
                for (int c = 0; c < TN2; ++c) acc[r][c] = 0.f;
            const int smin = rev ? t0 : 0, smax = rev ? rows : min(rows, t0 + TM2);
#pragma unroll 2
            for (int s = smin; s < smax; ++s) {
                float a[TM2], b[TN2];
                ld_run<TM2>(At + s * LQ + t0, a);
                ld_cols<TN2, D>(Vn + s * LV, tx, b);
#pragma unroll
                for (int r = 0; r < TM2; ++r)
#pragma unroll
                    for (int c = 0; c < TN2; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
            }
#pragma unroll 4
            for (int i = 0; i < D; ++i) {
                float a[TM2], b[TN2];
                ld_run<TM2>(Qt + i * LQ + t0, a);
                ld_cols<TN2, D>(Sm + i * LV, tx, b);
#pragma unroll
                for (int r = 0; r < TM2; ++r)
#pragma unroll
                    for (int c = 0; c < TN2; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
            }
#pragma unroll
            for (int r = 0; r < TM2; ++r) {
                if (t0 + r >= rows) break;
                T* dst = o + (row0 + (long)(c0 + t0 + r) * row_stride) * D;
                if constexpr (TN2 >= 4) {
#pragma unroll
                    for (int g = 0; g < TN2 / 4; ++g) store4(dst + col_of<TN2, D>(tx, 4 * g), &acc[r][4 * g]);
                } else {
                    store2(dst + col_of<TN2, D>(tx, 0), &acc[r][0]);
                }
            }
        }
        __syncthreads();  // every read of Sm for this chunk is done
        // ---- state: S += K^T V over the chunk's valid rows
#pragma unroll 2
        for (int s = 0; s < rows; ++s) {
            float a[TM3], b[TN3];
            ld_run<TM3>(Kn + s * LV + ty * TM3, a);
            ld_cols<TN3, D>(Vn + s * LV, tx, b);
#pragma unroll
            for (int r = 0; r < TM3; ++r)
#pragma unroll
                for (int c = 0; c < TN3; ++c) accS[r][c] = fmaf(a[r], b[c], accS[r][c]);
        }
#pragma unroll
        for (int r = 0; r < TM3; ++r) st_cols<TN3, D>(Sm + (ty * TM3 + r) * LV, tx, accS[r]);
    }
    if (p.s_out && write_state) {
        float* dst = p.s_out + state * D * D;
#pragma unroll
        for (int r = 0; r < TM3; ++r) {
            const int i = ty * TM3 + r;
#pragma unroll
            for (int c = 0; c < TN3; ++c) dst[i * D + col_of<TN3, D>(tx, c)] = accS[r][c];
        }
    }
}

}  // namespace simt
}  // namespace lcl

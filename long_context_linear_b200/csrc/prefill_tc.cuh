// Chunked causal linear attention on tcgen05 tensor cores (bf16 in, fp32 state).
//
// For every chunk c of C = 128 tokens of one (sequence, head) the kernel forms
// the tiled Lightning Attention update (page "MiniMax: «Почему M2 в итоге стала
// моделью с полным вниманием?» (конспект)", section 1, glossary entry
// "Lightning Attention": masked matrix inside the block, K^T V state between
// blocks) of the recurrence S_t = S_{t-1} + k_t v_t^T, o_t = q_t S_t (page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"):
//
//   P_c   = Q_c K_c^T                      tcgen05, fp32 accumulator in TMEM
//   P_c  <- P_c ⊙ M  (keep s <= t), bf16   mask warps, written back into TMEM
//   O_c   = P_c V_c                        tcgen05 with A = P_c read from TMEM
//   O_c  += Q_c S_hi + Q_c S_lo            S_{c-1} split into two bf16 terms
//   dS_c  = K_c^T V_c                      tcgen05 (K, V read MN-major)
//   S_c   = S_{c-1} + dS_c                 fp32, in the state warps' registers
//
// Work item = (sequence or batch*head unit, head, 64-wide slice of d_v).  One
// CTA (persistent over items) holds the item's state slice S[:, slice] in
// fp32 registers of four "state" warps; the tensor cores only ever see it as
// S_hi = bf16(S), S_lo = bf16(S - S_hi), so the Q S product keeps ~16 bits of
// the fp32 state.  Warp roles (14 warps):
//   w0 lane 0 : TMA producer (Q, K, V chunk tiles, 128B-swizzled, 2 stages)
//   w1        : TMEM allocation; lane 0 issues every tcgen05.mma
//   w2..w5    : mask warps   (P: TMEM -> regs -> causal mask -> bf16 -> TMEM)
//   w6..w9    : state warps  (dS: TMEM -> regs, S += dS, S_hi/S_lo -> smem)
//   w10..w13  : output warps (O: TMEM -> regs -> bf16 -> smem -> TMA store)
// Every wait is bounded (see mbar_wait); a timeout stops the CTA cleanly.
#pragma once
#include "sm100.cuh"

namespace lcl {
namespace tc {

constexpr int C = 128;         // chunk length (tokens)
constexpr int DK = 128;        // key dim
constexpr int DVS = 64;        // value columns per CTA
constexpr int STAGES = 2;
constexpr int PANEL = 128 * 128;  // one 128-row x 128-byte swizzled panel
constexpr int OFF_Q = 0;
constexpr int OFF_K = 2 * PANEL;
constexpr int OFF_V = 4 * PANEL;
constexpr int STAGE_BYTES = 5 * PANEL;
constexpr int OFF_SHI = STAGES * STAGE_BYTES;
constexpr int OFF_SLO = OFF_SHI + PANEL;
constexpr int OFF_OST = OFF_SLO + PANEL;   // 2 output staging panels
constexpr int OFF_BAR = OFF_OST + 2 * PANEL;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
constexpr int NUM_THREADS = 448;

constexpr uint32_t TM_P = 0;     // 2 buffers x 128 columns
constexpr uint32_t TM_O = 256;   // 2 buffers x 64 columns
constexpr uint32_t TM_DS = 384;  // 2 buffers x 64 columns
constexpr uint32_t TMEM_COLS = 512;

struct Params {
    int mode;              // 0 = dense [U][N][d]; 1 = packed [T][H][d]
    int n_items;           // work items
    int n_vs;              // value slices per head (dv / 64)
    int H;                 // heads (packed layout)
    int N;                 // tokens per unit (dense)
    int dv;                // full value dim
    const int* cu_seqlens; // packed: [n_seq + 1]
    const int* order;      // packed: sequence indices, longest first
    const float* s0;       // dense: [U][DK][dv] or null
    const float* pool;     // packed: [n_pool][H][DK][dv] or null
    const int* init_idx;   // packed: [n_seq] or null
    float* s_out;          // [U or n_seq*H][DK][dv] or null
    __nv_bfloat16* o;      // output base, for direct stores of ragged tails
    int* status;           // device status word
};

struct Item {
    int t0;         // first token (packed: absolute row; dense: 0)
    int len;        // tokens
    int c1, c2;     // TMA coordinates (dense: unit in c2; packed: head in c1)
    int vs;         // value slice
    long state;     // index of the (unit | sequence*H + head) state
    const float* init;  // initial state row block or null
};

__device__ __forceinline__ int item_index(int round, int cta, int grid) {
    // boustrophedon order over CTAs keeps per-CTA totals balanced when items
    // arrive longest first
    return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

__device__ __forceinline__ Item decode_item(const Params& p, int idx) {
    Item it;
    it.vs = idx % p.n_vs;
    if (p.mode == 0) {
        const int u = idx / p.n_vs;
        it.t0 = 0;
        it.len = p.N;
        it.c1 = 0;
        it.c2 = u;
        it.state = u;
        it.init = p.s0 ? p.s0 + (long)u * DK * p.dv : nullptr;
    } else {
        const int per_seq = p.H * p.n_vs;
        const int r = idx / per_seq;
        const int h = (idx % per_seq) / p.n_vs;
        const int seq = p.order ? p.order[r] : r;
        it.t0 = p.cu_seqlens[seq];
        it.len = p.cu_seqlens[seq + 1] - it.t0;
        it.c1 = h;
        it.c2 = 0;
        it.state = (long)seq * p.H + h;
        const int ii = p.init_idx ? p.init_idx[seq] : -1;
        it.init = (p.pool && ii >= 0) ? p.pool + ((long)ii * p.H + h) * DK * p.dv : nullptr;
    }
    return it;
}

// Wait on an mbarrier from a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
    const bool ok = mbar_wait(bar, parity, abort, status);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait used only while draining on the way out (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > 200000000ull) break;
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* full = bars + 0;      // [2] TMA -> MMA
    uint64_t* empty = bars + 2;     // [2] MMA -> TMA
    uint64_t* p_full = bars + 4;    // [2] MMA -> mask
    uint64_t* p_ready = bars + 6;   // [2] mask -> MMA
    uint64_t* ds_full = bars + 8;   // [2] MMA -> state
    uint64_t* ds_empty = bars + 10; // [2] state -> MMA
    uint64_t* o_full = bars + 12;   // [2] MMA -> output
    uint64_t* o_empty = bars + 14;  // [2] output -> MMA
    uint64_t* s_full = bars + 16;   // state -> MMA (S_hi/S_lo written)
    uint64_t* s_empty = bars + 17;  // MMA -> state (Q S products done)
    uint64_t* drain = bars + 18;    // MMA drain on exit
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 19);
    volatile int* abort = reinterpret_cast<volatile int*>(bars + 20);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
            mbar_init(&p_full[i], 1);
            mbar_init(&p_ready[i], 4);
            mbar_init(&ds_full[i], 1);
            mbar_init(&ds_empty[i], 4);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 4);
        }
        mbar_init(s_full, 4);
        mbar_init(s_empty, 1);
        mbar_init(drain, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
        prefetch_tmap(&map_o);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int g = 0;
            for (int r = 0;; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const Item it = decode_item(p, idx);
                const int nc = (it.len + C - 1) / C;
                bool stop = false;
                for (int c = 0; c < nc; ++c, ++g) {
                    const int st = g & 1, k = g >> 1;
                    if (k > 0 && !mbar_wait(&empty[st], (k - 1) & 1, abort, p.status)) { stop = true; break; }
                    mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
                    uint8_t* sb = sm + st * STAGE_BYTES;
                    int y, z;
                    if (p.mode == 0) { y = c * C; z = it.c2; }
                    else { y = it.c1; z = it.t0 + c * C; }
                    tma_load_3d(sb + OFF_Q, &map_q, &full[st], 0, y, z);
                    tma_load_3d(sb + OFF_Q + PANEL, &map_q, &full[st], 64, y, z);
                    tma_load_3d(sb + OFF_K, &map_k, &full[st], 0, y, z);
                    tma_load_3d(sb + OFF_K + PANEL, &map_k, &full[st], 64, y, z);
                    tma_load_3d(sb + OFF_V, &map_v, &full[st], DVS * it.vs, y, z);
                }
                if (stop) break;
            }
            // make sure no copy into shared memory is still in flight at exit
            for (int x = (g >= 2 ? g - 2 : 0); x < g; ++x) drain_wait(&full[x & 1], (x >> 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        const uint32_t id_p = idesc_bf16(128, 128, 0, 0);
        const uint32_t id_ds = idesc_bf16(128, DVS, 1, 1);
        const uint32_t id_pv = idesc_bf16(128, DVS, 0, 1);
        const uint32_t id_qs = idesc_bf16(128, DVS, 0, 1);
        const uint32_t s_hi = smem_u32(sm + OFF_SHI), s_lo = smem_u32(sm + OFF_SLO);
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item(p, idx);
            const int nc = (it.len + C - 1) / C;
            for (int c = 0; c < nc; ++c, ++g) {
                const int st = g & 1, b = g & 1, k = g >> 1;
                if (!warp_wait(&full[st], k & 1, abort, p.status)) { stop = true; break; }
                uint8_t* sb = sm + st * STAGE_BYTES;
                const int rows = it.len - c * C;
                if (p.mode == 1 && rows < C) {
                    // ragged tail inside a packed batch: rows past the end belong to
                    // the next sequence; clear them in K and V before any product
                    const int first = rows * 128;
                    const int n16 = (PANEL - first) >> 4;
                    for (int pnl = 0; pnl < 3; ++pnl) {
                        uint8_t* base = sb + (pnl < 2 ? OFF_K + pnl * PANEL : OFF_V) + first;
                        for (int e = lane; e < n16; e += 32)
                            *reinterpret_cast<uint4*>(base + e * 16) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                tc_fence_after();
                const uint32_t qa = smem_u32(sb + OFF_Q), ka = smem_u32(sb + OFF_K), va = smem_u32(sb + OFF_V);
                const uint32_t tp = tbase + TM_P + 128u * b, to = tbase + TM_O + 64u * b,
                               tds = tbase + TM_DS + 64u * b;
                if (lane == 0) {
                    // P = Q K^T   (A: Q K-major, B: K K-major)
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
                        mma_ss(tp, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), id_p, kk > 0);
                    }
                    mma_commit(&p_full[b]);
                }
                __syncwarp();
                // dS = K^T V   (A: K MN-major over 2 panels, B: V MN-major)
                if (k > 0 && !warp_wait(&ds_empty[b], (k - 1) & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_ss(tds, sw128_desc(ka + kk * 2048, PANEL, 1024), sw128_desc(va + kk * 2048, PANEL, 1024),
                               id_ds, kk > 0);
                    mma_commit(&ds_full[b]);
                }
                __syncwarp();
                // O = P V   (A: masked bf16 P in TMEM)
                if (!warp_wait(&p_ready[b], k & 1, abort, p.status)) { stop = true; break; }
                if (k > 0 && !warp_wait(&o_empty[b], (k - 1) & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_ts(to, tp + kk * 8, sw128_desc(va + kk * 2048, PANEL, 1024), id_pv, kk > 0);
                }
                __syncwarp();
                // O += Q S_hi + Q S_lo   (B: S slices MN-major)
                if (!warp_wait(s_full, g & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
                        mma_ss(to, sw128_desc(qa + off, 16, 1024), sw128_desc(s_hi + kk * 2048, PANEL, 1024), id_qs, 1);
                    }
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
                        mma_ss(to, sw128_desc(qa + off, 16, 1024), sw128_desc(s_lo + kk * 2048, PANEL, 1024), id_qs, 1);
                    }
                    mma_commit(&o_full[b]);
                    mma_commit(s_empty);
                    mma_commit(&empty[st]);
                }
                __syncwarp();
            }
        }
        // every MMA issued by this thread must be finished before TMEM is freed
        if (lane == 0) {
            mma_commit(drain);
            drain_wait(drain, 0);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------ mask warps
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item(p, idx);
            const int nc = (it.len + C - 1) / C;
            for (int c = 0; c < nc; ++c, ++g) {
                const int b = g & 1, k = g >> 1;
                if (!warp_wait(&p_full[b], k & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_P + 128u * b;
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    uint32_t packed[16];
                    if (pc > q4) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) packed[i] = 0u;
                    } else {
                        uint32_t v[32];
                        tmem_ld32(ta + 32 * pc, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int s = 32 * pc + 2 * i;
                            const float a0 = (s <= row) ? __uint_as_float(v[2 * i]) : 0.f;
                            const float a1 = (s + 1 <= row) ? __uint_as_float(v[2 * i + 1]) : 0.f;
                            packed[i] = pack_bf16x2(a0, a1);
                        }
                    }
                    tmem_st16(ta + 16 * pc, packed);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_ready[b]);
            }
        }
    } else if (warp < 10) {
        // ------------------------------------------------------ state warps
        const int q4 = warp & 3;
        const int i = q4 * 32 + lane;  // key-dim row of S owned by this thread
        const uint32_t s_hi = smem_u32(sm + OFF_SHI), s_lo = smem_u32(sm + OFF_SLO);
        const uint32_t row_off = static_cast<uint32_t>(i) * 128u;
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item(p, idx);
            const int nc = (it.len + C - 1) / C;
            float S[DVS];
            if (it.init) {
                const float4* src = reinterpret_cast<const float4*>(it.init + (long)i * p.dv + DVS * it.vs);
#pragma unroll
                for (int j = 0; j < DVS / 4; ++j) {
                    const float4 x = src[j];
                    S[4 * j] = x.x; S[4 * j + 1] = x.y; S[4 * j + 2] = x.z; S[4 * j + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < DVS; ++j) S[j] = 0.f;
            }
            for (int c = 0; c < nc; ++c, ++g) {
                const int b = g & 1, k = g >> 1;
                // publish S_{c-1} as S_hi + S_lo (bf16, MN-major swizzled rows)
                if (g > 0 && !warp_wait(s_empty, (g - 1) & 1, abort, p.status)) { stop = true; break; }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a0 = S[ch * 8 + 2 * e], a1 = S[ch * 8 + 2 * e + 1];
                        const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
                        hi[e] = *reinterpret_cast<const uint32_t*>(&h);
                        lo[e] = pack_bf16x2(a0 - __low2float(h), a1 - __high2float(h));
                    }
                    const uint32_t off = row_off + ((static_cast<uint32_t>(ch) ^ (i & 7)) << 4);
                    st_shared_v4(s_hi + off, hi[0], hi[1], hi[2], hi[3]);
                    st_shared_v4(s_lo + off, lo[0], lo[1], lo[2], lo[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_full);
                // absorb dS_c
                if (!warp_wait(&ds_full[b], k & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_DS + 64u * b;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[32];
                    tmem_ld32(ta + 32 * h2, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * h2 + j] += __uint_as_float(v[j]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ds_empty[b]);
            }
            if (stop) break;
            if (p.s_out) {
                float4* dst = reinterpret_cast<float4*>(p.s_out + (it.state * DK + i) * p.dv + DVS * it.vs);
#pragma unroll
                for (int j = 0; j < DVS / 4; ++j)
                    dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            }
        }
    } else {
        // ------------------------------------------------------ output warps
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item(p, idx);
            const int nc = (it.len + C - 1) / C;
            for (int c = 0; c < nc; ++c, ++g) {
                const int b = g & 1, k = g >> 1;
                if (!warp_wait(&o_full[b], k & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_O + 64u * b;
                uint32_t hp[32];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[32];
                    tmem_ld32(ta + 32 * h2, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        hp[16 * h2 + e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_empty[b]);
                const int rows = it.len - c * C;
                if (p.mode == 0 && q4 * 32 >= rows) {
                    // this warp's rows all lie past the end of the sequence
                } else if (p.mode == 0 || rows >= C) {
                    // each warp stages its 32 rows and stores them with one TMA copy
                    uint8_t* stg = sm + OFF_OST + (g & 1) * PANEL + q4 * 32 * 128;
                    if (lane == 0) bulk_wait_read<1>();
                    __syncwarp();
                    const uint32_t sa = smem_u32(stg) + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        st_shared_v4(sa + ((static_cast<uint32_t>(ch) ^ (row & 7)) << 4), hp[4 * ch], hp[4 * ch + 1],
                                     hp[4 * ch + 2], hp[4 * ch + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (p.mode == 0) tma_store_3d(&map_o, stg, DVS * it.vs, c * C + q4 * 32, it.c2);
                        else tma_store_3d(&map_o, stg, DVS * it.vs, it.c1, it.t0 + c * C + q4 * 32);
                        bulk_commit();
                    }
                } else if (row < rows) {
                    uint4* dst = reinterpret_cast<uint4*>(
                        p.o + ((long)(it.t0 + c * C + row) * p.H + it.c1) * p.dv + DVS * it.vs);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        dst[ch] = make_uint4(hp[4 * ch], hp[4 * ch + 1], hp[4 * ch + 2], hp[4 * ch + 3]);
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace lcl

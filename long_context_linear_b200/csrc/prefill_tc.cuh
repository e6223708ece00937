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
//   [O|O']= Q_c [S_hi | S_lo]              one N=128 product; S_{c-1} split
//                                          into two bf16 terms, summed on output
//   dS_c  = K_c^T V_c                      tcgen05 (K, V read MN-major)
//   O    += P_c V_c                        tcgen05 with A = P_c read from TMEM
//   S_c   = S_{c-1} + dS_c                 fp32, in the state warps' registers
//
// Work item = (sequence or batch*head unit, head, 64-wide slice of d_v).  One
// CTA (persistent over items) holds the item's state slice S[:, slice] in
// fp32 registers of four "state" warps; the tensor cores only ever see it as
// S_hi = bf16(S), S_lo = bf16(S - S_hi), so the Q S product keeps ~16 bits of
// the fp32 state.  Warp roles (14 warps):
//   w0 lane 0 : TMA producer (Q,K tiles in 2 slots, V tiles in 3 slots,
//               128B-swizzled; L2 prefetch a few chunks ahead)
//   w1        : TMEM allocation; lane 0 issues every tcgen05.mma
//   w2..w5    : mask warps   (P: TMEM -> regs -> causal mask -> bf16 -> TMEM)
//   w6..w9    : state warps  (dS: TMEM -> regs, S += dS, S_hi/S_lo -> smem)
//   w10..w13  : output warps (O + O': TMEM -> regs -> bf16 -> smem -> TMA store)
// The issue order per chunk (P, dS, Q S, P V) lets the tensor cores run dS and
// Q S while the mask warps work on P, and gives the state warps Q S, P V and
// the next chunk's P and dS to fold dS_c into S before it is needed.  Q/K
// slots are released after Q S, V slots after P V.
// Every wait is bounded (see mbar_wait); a timeout stops the CTA cleanly.
#pragma once
#include "sm100.cuh"

namespace lcl {
namespace tc {

constexpr int C = 128;         // chunk length (tokens)
constexpr int DK = 128;        // key dim
constexpr int DVS = 64;        // value columns per CTA
constexpr int QK_SLOTS = 2;    // Q,K chunk tiles in flight (held until Q S)
constexpr int V_SLOTS = 3;     // V chunk tiles in flight (held until P V)
constexpr int PREFETCH = 3;    // chunks brought into L2 ahead of their load
constexpr int PANEL = 128 * 128;  // one 128-row x 128-byte swizzled panel
constexpr int QK_BYTES = 4 * PANEL;                   // Q (2 panels) + K (2 panels)
constexpr int OFF_QK = 0;                             // QK_SLOTS x [Q0 Q1 K0 K1]
constexpr int OFF_V = OFF_QK + QK_SLOTS * QK_BYTES;   // V_SLOTS x [V]
constexpr int OFF_SHI = OFF_V + V_SLOTS * PANEL;      // S_hi panel, S_lo panel right after
constexpr int OFF_SLO = OFF_SHI + PANEL;
constexpr int OFF_OST = OFF_SLO + PANEL;              // output staging panel
constexpr int OFF_BAR = OFF_OST + PANEL;
// mbarrier slots (8 bytes each) at OFF_BAR, then the TMEM base and the abort flag
constexpr int BAR_QK_FULL = 0;
constexpr int BAR_QK_EMPTY = BAR_QK_FULL + QK_SLOTS;
constexpr int BAR_V_FULL = BAR_QK_EMPTY + QK_SLOTS;
constexpr int BAR_V_EMPTY = BAR_V_FULL + V_SLOTS;
constexpr int BAR_P_FULL = BAR_V_EMPTY + V_SLOTS;
constexpr int BAR_P_READY = BAR_P_FULL + 1;
constexpr int BAR_DS_FULL = BAR_P_READY + 1;
constexpr int BAR_DS_EMPTY = BAR_DS_FULL + 2;
constexpr int BAR_O_FULL = BAR_DS_EMPTY + 2;
constexpr int BAR_O_EMPTY = BAR_O_FULL + 2;
constexpr int BAR_S_FULL = BAR_O_EMPTY + 2;
constexpr int BAR_S_EMPTY = BAR_S_FULL + 1;
constexpr int BAR_DRAIN = BAR_S_EMPTY + 1;
constexpr int BAR_COUNT = BAR_DRAIN + 1;
constexpr int BAR_BYTES = 256;
static_assert((BAR_COUNT + 2) * 8 <= BAR_BYTES, "barrier area too small");
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB per-block shared memory limit");
constexpr int NUM_THREADS = 448;

constexpr uint32_t TM_P = 0;     // 128 columns: P (fp32), then bf16 P in columns 0..63
constexpr uint32_t TM_O = 128;   // 2 buffers x 128 columns: [Q S_hi + P V | Q S_lo]
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
    uint64_t* qk_full = bars + BAR_QK_FULL;    // [QK_SLOTS] TMA -> MMA
    uint64_t* qk_empty = bars + BAR_QK_EMPTY;  // [QK_SLOTS] MMA -> TMA (after Q S)
    uint64_t* v_full = bars + BAR_V_FULL;      // [V_SLOTS]
    uint64_t* v_empty = bars + BAR_V_EMPTY;    // [V_SLOTS] (after P V)
    uint64_t* p_full = bars + BAR_P_FULL;      // MMA -> mask
    uint64_t* p_ready = bars + BAR_P_READY;    // mask -> MMA
    uint64_t* ds_full = bars + BAR_DS_FULL;    // [2] MMA -> state
    uint64_t* ds_empty = bars + BAR_DS_EMPTY;  // [2] state -> MMA
    uint64_t* o_full = bars + BAR_O_FULL;      // [2] MMA -> output
    uint64_t* o_empty = bars + BAR_O_EMPTY;    // [2] output -> MMA
    uint64_t* s_full = bars + BAR_S_FULL;      // state -> MMA (S_hi/S_lo written)
    uint64_t* s_empty = bars + BAR_S_EMPTY;    // MMA -> state (Q S product done)
    uint64_t* drain = bars + BAR_DRAIN;        // MMA drain on exit
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + BAR_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(bars + BAR_COUNT + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < QK_SLOTS; ++i) {
            mbar_init(&qk_full[i], 1);
            mbar_init(&qk_empty[i], 1);
        }
        for (int i = 0; i < V_SLOTS; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ds_full[i], 1);
            mbar_init(&ds_empty[i], 4);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 4);
        }
        mbar_init(p_full, 1);
        mbar_init(p_ready, 4);
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
                auto coords = [&](int c, int& y, int& z) {
                    if (p.mode == 0) { y = c * C; z = it.c2; }
                    else { y = it.c1; z = it.t0 + c * C; }
                };
                auto prefetch = [&](int c) {
                    int y, z;
                    coords(c, y, z);
                    tma_prefetch_3d(&map_q, 0, y, z);
                    tma_prefetch_3d(&map_q, 64, y, z);
                    tma_prefetch_3d(&map_k, 0, y, z);
                    tma_prefetch_3d(&map_k, 64, y, z);
                    tma_prefetch_3d(&map_v, DVS * it.vs, y, z);
                };
                for (int c = 0; c < PREFETCH && c < nc; ++c) prefetch(c);
                bool stop = false;
                for (int c = 0; c < nc; ++c, ++g) {
                    if (c + PREFETCH < nc) prefetch(c + PREFETCH);
                    int y, z;
                    coords(c, y, z);
                    const int a = g % QK_SLOTS, ka = g / QK_SLOTS;
                    if (ka > 0 && !mbar_wait(&qk_empty[a], (ka - 1) & 1, abort, p.status)) { stop = true; break; }
                    uint8_t* qk = sm + OFF_QK + a * QK_BYTES;
                    mbar_arrive_expect_tx(&qk_full[a], QK_BYTES);
                    tma_load_3d(qk, &map_q, &qk_full[a], 0, y, z);
                    tma_load_3d(qk + PANEL, &map_q, &qk_full[a], 64, y, z);
                    tma_load_3d(qk + 2 * PANEL, &map_k, &qk_full[a], 0, y, z);
                    tma_load_3d(qk + 3 * PANEL, &map_k, &qk_full[a], 64, y, z);
                    const int vc = g % V_SLOTS, kv = g / V_SLOTS;
                    if (kv > 0 && !mbar_wait(&v_empty[vc], (kv - 1) & 1, abort, p.status)) { stop = true; break; }
                    mbar_arrive_expect_tx(&v_full[vc], PANEL);
                    tma_load_3d(sm + OFF_V + vc * PANEL, &map_v, &v_full[vc], DVS * it.vs, y, z);
                }
                if (stop) break;
            }
            // make sure no copy into shared memory is still in flight at exit
            for (int x = (g >= QK_SLOTS ? g - QK_SLOTS : 0); x < g; ++x)
                drain_wait(&qk_full[x % QK_SLOTS], (x / QK_SLOTS) & 1);
            for (int x = (g >= V_SLOTS ? g - V_SLOTS : 0); x < g; ++x)
                drain_wait(&v_full[x % V_SLOTS], (x / V_SLOTS) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        // One thread issues every product; the other lanes of this warp only
        // take part in TMEM allocation.  The tensor pipe is fed from this single
        // thread, so each group of products is issued from fully unrolled code
        // with its descriptors computed up front (a rolled loop only for the
        // ragged last chunk of a packed sequence).  Completions of this thread's
        // own tcgen05.commit need no fence; TMEM written or read by other warps is
        // ordered by tcgen05.fence::after_thread_sync after the barrier.
        if (lane == 0) {
            constexpr uint32_t id_p = idesc_bf16(128, 128, 0, 0);   // Q K^T
            constexpr uint32_t id_qs = idesc_bf16(128, 128, 0, 1);  // Q [S_hi | S_lo]
            constexpr uint32_t id_ds = idesc_bf16(128, DVS, 1, 1);  // K^T V
            constexpr uint32_t id_pv = idesc_bf16(128, DVS, 0, 1);  // P V (P from TMEM)
            const uint64_t d_qk0 = sw128_desc(smem_u32(sm + OFF_QK), 16, 1024);
            const uint64_t d_kt0 = sw128_desc(smem_u32(sm + OFF_QK + 2 * PANEL), PANEL, 1024);
            const uint64_t d_v0 = sw128_desc(smem_u32(sm + OFF_V), PANEL, 1024);
            const uint64_t d_s = sw128_desc(smem_u32(sm + OFF_SHI), PANEL, 1024);
            const uint32_t tp = tbase + TM_P;
            // K-step offsets (16-byte units): K-major tiles step 32 B inside a
            // 64-column panel, MN-major tiles step 16 rows (2048 B)
            auto kmaj = [](int kk) { return static_cast<uint64_t>(((kk >> 2) * PANEL + (kk & 3) * 32) >> 4); };
            auto mnmaj = [](int kk) { return static_cast<uint64_t>((kk * 2048) >> 4); };
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const Item it = decode_item(p, idx);
                const int nc = (it.len + C - 1) / C;
                for (int c = 0; c < nc; ++c, ++g) {
                    const int a = g % QK_SLOTS, ka = g / QK_SLOTS;
                    const int vc = g % V_SLOTS, kv = g / V_SLOTS;
                    const int b = g & 1, kb = g >> 1;
                    const uint64_t d_q = d_qk0 + static_cast<uint64_t>((a * QK_BYTES) >> 4);
                    const uint64_t d_k = d_q + static_cast<uint64_t>((2 * PANEL) >> 4);
                    const uint64_t d_kt = d_kt0 + static_cast<uint64_t>((a * QK_BYTES) >> 4);
                    const uint64_t d_v = d_v0 + static_cast<uint64_t>((vc * PANEL) >> 4);
                    const uint32_t to = tbase + TM_O + 128u * b, tds = tbase + TM_DS + 64u * b;
                    // a ragged tail inside a packed batch: rows past the end belong to
                    // the next sequence.  Products over the token dim (K^T V, P V) stop
                    // at the last 16-row step holding valid rows, whose invalid rows are
                    // cleared; Q K^T columns past the end are removed by the causal mask.
                    const int rows = it.len - c * C;
                    const bool ragged = p.mode == 1 && rows < C;
                    const int ksteps = ragged ? (rows + 15) >> 4 : C / 16;
                    if (!mbar_wait(&qk_full[a], ka & 1, abort, p.status)) { stop = true; break; }
                    if (ragged && (rows & 15)) {
                        uint8_t* kb0 = sm + OFF_QK + a * QK_BYTES + 2 * PANEL;
                        for (int pnl = 0; pnl < 2; ++pnl)
                            for (int e = rows * 128; e < ksteps * 16 * 128; e += 16)
                                *reinterpret_cast<uint4*>(kb0 + pnl * PANEL + e) = make_uint4(0u, 0u, 0u, 0u);
                        fence_proxy_async_smem();
                    }
                    // P = Q K^T   (A: Q K-major, B: K K-major)
                    {
                        uint64_t da[8], db[8];
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) { da[kk] = d_q + kmaj(kk); db[kk] = d_k + kmaj(kk); }
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) mma_ss(tp, da[kk], db[kk], id_p, kk > 0);
                    }
                    mma_commit(p_full);
                    // dS = K^T V   (A: K MN-major over 2 panels, B: V MN-major); issued
                    // early so the state warps have the rest of this chunk and the
                    // next chunk's P to fold it into S before the next Q S product
                    if (!mbar_wait(&v_full[vc], kv & 1, abort, p.status)) { stop = true; break; }
                    if (ragged && (rows & 15)) {
                        uint8_t* vb = sm + OFF_V + vc * PANEL;
                        for (int e = rows * 128; e < ksteps * 16 * 128; e += 16)
                            *reinterpret_cast<uint4*>(vb + e) = make_uint4(0u, 0u, 0u, 0u);
                        fence_proxy_async_smem();
                    }
                    if (kb > 0 && !mbar_wait(&ds_empty[b], (kb - 1) & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    if (!ragged) {
                        uint64_t da[8], db[8];
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) { da[kk] = d_kt + mnmaj(kk); db[kk] = d_v + mnmaj(kk); }
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) mma_ss(tds, da[kk], db[kk], id_ds, kk > 0);
                    } else {
                        for (int kk = 0; kk < ksteps; ++kk) mma_ss(tds, d_kt + mnmaj(kk), d_v + mnmaj(kk), id_ds, kk > 0);
                    }
                    mma_commit(&ds_full[b]);
                    // [O | O'] = Q [S_hi | S_lo]   (B: the two S panels, MN-major, N = 128)
                    if (kb > 0 && !mbar_wait(&o_empty[b], (kb - 1) & 1, abort, p.status)) { stop = true; break; }
                    if (!mbar_wait(s_full, g & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    {
                        uint64_t da[8], db[8];
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) { da[kk] = d_q + kmaj(kk); db[kk] = d_s + mnmaj(kk); }
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) mma_ss(to, da[kk], db[kk], id_qs, kk > 0);
                    }
                    mma_commit(s_empty);
                    mma_commit(&qk_empty[a]);
                    // O += P V   (A: masked bf16 P in TMEM, B: V MN-major)
                    if (!mbar_wait(p_ready, g & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    if (!ragged) {
                        uint64_t db[8];
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) db[kk] = d_v + mnmaj(kk);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) mma_ts(to, tp + kk * 8, db[kk], id_pv, 1);
                    } else {
                        for (int kk = 0; kk < ksteps; ++kk) mma_ts(to, tp + kk * 8, d_v + mnmaj(kk), id_pv, 1);
                    }
                    mma_commit(&o_full[b]);
                    mma_commit(&v_empty[vc]);
                }
            }
            // every MMA issued by this thread must be finished before TMEM is freed
            mma_commit(drain);
            drain_wait(drain, 0);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------ mask warps
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_P;
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item(p, idx);
            const int nc = (it.len + C - 1) / C;
            for (int c = 0; c < nc; ++c, ++g) {
                if (!warp_wait(p_full, g & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                // columns s of 32-wide pieces 2h, 2h+1; pieces above this warp's rows are zero
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v0[32], v1[32];
                    const int p0 = 2 * h, p1 = 2 * h + 1;
                    if (p0 <= q4) tmem_ld32(ta + 32 * p0, v0);
                    if (p1 <= q4) tmem_ld32(ta + 32 * p1, v1);
                    if (p0 <= q4) tmem_wait_ld();
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int s0 = 32 * p0 + 2 * i, s1 = 32 * p1 + 2 * i;
                        pk[i] = (p0 <= q4) ? pack_bf16x2(s0 <= row ? __uint_as_float(v0[2 * i]) : 0.f,
                                                         s0 + 1 <= row ? __uint_as_float(v0[2 * i + 1]) : 0.f)
                                           : 0u;
                        pk[16 + i] = (p1 <= q4) ? pack_bf16x2(s1 <= row ? __uint_as_float(v1[2 * i]) : 0.f,
                                                              s1 + 1 <= row ? __uint_as_float(v1[2 * i + 1]) : 0.f)
                                                : 0u;
                    }
                    tmem_st32(ta + 32 * h, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_ready);
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
                const int b = g & 1, kb = g >> 1;
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
                if (!warp_wait(&ds_full[b], kb & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_DS + 64u * b;
                uint32_t v0[32], v1[32];
                tmem_ld32(ta, v0);
                tmem_ld32(ta + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ds_empty[b]);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    S[j] += __uint_as_float(v0[j]);
                    S[32 + j] += __uint_as_float(v1[j]);
                }
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
        uint8_t* stg = sm + OFF_OST + q4 * 32 * 128;  // this warp's 32 staging rows
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item(p, idx);
            const int nc = (it.len + C - 1) / C;
            for (int c = 0; c < nc; ++c, ++g) {
                const int b = g & 1, kb = g >> 1;
                if (!warp_wait(&o_full[b], kb & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_O + 128u * b;
                uint32_t hp[32];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(ta + 32 * h, v0);       // Q S_hi + P V
                    tmem_ld32(ta + 64 + 32 * h, v1);  // Q S_lo
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        hp[16 * h + e] = pack_bf16x2(__uint_as_float(v0[2 * e]) + __uint_as_float(v1[2 * e]),
                                                     __uint_as_float(v0[2 * e + 1]) + __uint_as_float(v1[2 * e + 1]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_empty[b]);
                const int rows = it.len - c * C;
                if (p.mode == 0 && q4 * 32 >= rows) {
                    // this warp's rows all lie past the end of the sequence
                } else if (p.mode == 0 || rows >= C) {
                    // each warp stages its 32 rows and stores them with one TMA copy
                    if (lane == 0) bulk_wait_read<0>();
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
                    // ragged tail of a packed sequence: plain row stores
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

// Chunked causal linear attention on tcgen05 tensor cores, one CTA per head
// over the whole value width (d_k = d_v = 128, bf16 in, fp32 state).
//
// The same tiled update as prefill_tc.cuh (page "MiniMax: «Почему M2 в итоге
// стала моделью с полным вниманием?» (конспект)", section 1, glossary entry
// "Lightning Attention": a masked matrix inside the block and a K^T V state
// between blocks, of the recurrence S_t = S_{t-1} + k_t v_t^T, o_t = q_t S_t
// of page "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"), for
// batches whose heads alone fill the GPU.  A work item is a whole head (unit,
// or sequence and head), so Q K^T is formed once per head instead of once per
// 64-column value slice, and every product is N = 128 wide:
//
//   P_c  = Q_c K_c^T               8 x N=128, fp32 in TMEM (two P buffers)
//   O_c  = Q_c bf16(S_{c-1})       8 x N=128 (S^T staged in shared memory)
//   P_c <- P_c ⊙ M  (keep s <= t)  mask, bf16, back into TMEM
//   O_c += P_c V_c                 8 x N=128, A = P_c from TMEM
//   dS_c = K_c^T V_c               8 x N=128 (K, V read MN-major)
//   S_c  = S_{c-1} + dS_c          fp32 registers of eight state warps
//
// Q K^T of chunk c+1 needs neither the state nor O, so it is issued right
// after P V of chunk c and its mask overlaps chunk c's output; the chain from
// chunk to chunk is Q S, P V and reading O out of TMEM.  TMEM: P buffers at
// columns 0 and 128 (bf16 P in the first 64 of each), O at 256, dS at 384.
//
// Shared memory: Q, K and V tiles of 128 tokens x 128 columns, two slots each,
// and one bf16(S)^T tile: 224 KB.  There is no room left for a separate output
// staging area, so each chunk's O is staged in that chunk's V slot: P V, the
// product that makes O, is V's last reader, so the slot is free exactly when O
// is ready; it goes back to the V producer once the TMA store has read it.
//
// Warp roles (16 warps):
//   w0 lane 0  : TMA producer for Q
//   w15 lane 0 : TMA producer for K and V
//   w1 lane 0  : MMA thread A: Q S and P V of chunk c, then Q K^T of chunk c+1
//   w14 lane 0 : MMA thread B: K^T V
//   w2..w5     : P/O warps: causal mask of P, then O -> bf16 -> V slot -> TMA store
//   w6..w13    : state warps: two per TMEM lane quarter, 64 value columns each
// Every wait is bounded (mbar_wait); a timeout stops the CTA cleanly.
#pragma once
#include "prefill_tc.cuh"

namespace lcl {
namespace tcw {

using tc::C;
using tc::PANEL;
// No L2 prefetch ahead of the loads: with 128 CTAs each streaming Q, K and V,
// prefetches three chunks ahead queued ahead of the demand loads and took
// the 8K batch (B=4, H=32) from 0.200 to 0.251 ms (one chunk ahead: 0.203).
constexpr int KD = 128;                 // key dim = value dim
constexpr int SLOTS = 2;                // Q, K, V ring depth
constexpr int TILE = 2 * PANEL;         // 128 rows x 128 bf16 columns: two 64-column panels
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + SLOTS * TILE;
constexpr int OFF_V = OFF_K + SLOTS * TILE;
constexpr int OFF_ST = OFF_V + SLOTS * TILE;  // bf16(S)^T: row j = value column j, key dims along the panels
constexpr int OFF_BAR = OFF_ST + TILE;
// mbarriers (8 bytes each) at OFF_BAR, then the TMEM base and the abort flag
constexpr int BAR_Q_FULL = 0;                       // [2] TMA -> A, state warps
constexpr int BAR_Q_EMPTY = BAR_Q_FULL + SLOTS;     // [2] A (Q K^T, Q S) -> TMA
constexpr int BAR_K_FULL = BAR_Q_EMPTY + SLOTS;     // [2] TMA -> A, B, state warps
constexpr int BAR_K_EMPTY = BAR_K_FULL + SLOTS;     // [2] A (Q K^T) + B (K^T V) -> TMA
constexpr int BAR_V_FULL = BAR_K_EMPTY + SLOTS;     // [2] TMA -> P/O warps, B
constexpr int BAR_V_EMPTY = BAR_V_FULL + SLOTS;     // [2] P/O warps (O stored from the slot) -> TMA
constexpr int BAR_V_KV = BAR_V_EMPTY + SLOTS;       // [2] B (K^T V done with the tile) -> P/O warps
constexpr int BAR_KPHI_FULL = BAR_V_KV + SLOTS;     // [2] state warps (phi(K) written) -> B
constexpr int BAR_QK_MAPPED = BAR_KPHI_FULL + SLOTS;  // [2] state warps (phi(K), phi(Q) written) -> A
constexpr int BAR_P_FULL = BAR_QK_MAPPED + SLOTS;   // [2] A (Q K^T done) -> P/O warps
constexpr int BAR_P_READY = BAR_P_FULL + 2;         // [2] P/O warps (bf16 P written, V landed) -> A
constexpr int BAR_DS_FULL = BAR_P_READY + 2;        // B -> state warps
constexpr int BAR_DS_EMPTY = BAR_DS_FULL + 1;       // state warps -> B
constexpr int BAR_S_FULL = BAR_DS_EMPTY + 1;        // state warps (S^T written) -> A
constexpr int BAR_ST_FREE = BAR_S_FULL + 1;         // A (Q S done) -> state warps: S^T may be rewritten
constexpr int BAR_O_FULL = BAR_ST_FREE + 1;         // A (P V done) -> P/O warps, A
constexpr int BAR_O_EMPTY = BAR_O_FULL + 1;         // P/O warps (O read out of TMEM) -> A
constexpr int BAR_DRAIN_A = BAR_O_EMPTY + 1;
constexpr int BAR_DRAIN_B = BAR_DRAIN_A + 1;
constexpr int BAR_COUNT = BAR_DRAIN_B + 1;
constexpr int BAR_BYTES = 512;
static_assert((BAR_COUNT + 2) * 8 <= BAR_BYTES, "barrier area too small");
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_ST % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB per-block shared memory limit");
constexpr int NUM_THREADS = 512;
constexpr int WARP_MMA_A = 1;
constexpr int WARP_MMA_B = 14;
constexpr int WARP_LOAD_V = 15;
constexpr int STATE_WARPS = 8;
constexpr int PO_WARPS = 4;

constexpr uint32_t TM_P = 0;     // P buffer b at TM_P + 128 b
constexpr uint32_t TM_O = 256;
constexpr uint32_t TM_DS = 384;
constexpr uint32_t TMEM_COLS = 512;

// Rows past the end of a packed sequence inside its last 16-row step belong to
// the next sequence; clear them in both panels of a V tile before a product
// over the token dim (both issuing threads write the same zeros).
__device__ __noinline__ void clear_tail_rows2(uint8_t* tile, int rows, int ksteps) {
    for (int e = rows * 128; e < ksteps * 16 * 128; e += 16) {
        *reinterpret_cast<uint4*>(tile + e) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(tile + PANEL + e) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
}

// phi in place on the 128 rows of both panels of a Q or K tile by the 256
// state-warp threads t = 0 .. 255, 16-byte vectors, four loads in flight.
__device__ __forceinline__ void phi_tile2(uint32_t base, int t, int phi) {
    constexpr int PER_THREAD = TILE / 16 / (STATE_WARPS * 32);  // 8
#pragma unroll
    for (int j0 = 0; j0 < PER_THREAD; j0 += 4) {
        uint4 r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = ld_shared_v4(base + static_cast<uint32_t>(t + (j0 + j) * 256) * 16u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 y = apply_phi_bf16x8(r[j], phi);
            st_shared_v4(base + static_cast<uint32_t>(t + (j0 + j) * 256) * 16u, y.x, y.y, y.z, y.w);
        }
    }
    fence_proxy_async_smem();
}

// kGeneral = false: feature map identity, chunks in order, initial state as
// given (the common forward case).  kGeneral = true adds the feature map on
// the Q and K tiles, the reverse chunk order and the transposed initial state
// of the backward passes.  Items are whole sequences (no segments).
// kAhead (with kGeneral, for elu + 1): the state warps map each chunk's
// tiles a chunk ahead (below); a separate instance, so that the others keep a
// single mapping site in their loop.
template <bool kGeneral, bool kAhead = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
prefill_wide_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                    const __grid_constant__ tc::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* q_full = bars + BAR_Q_FULL;
    uint64_t* q_empty = bars + BAR_Q_EMPTY;
    uint64_t* k_full = bars + BAR_K_FULL;
    uint64_t* k_empty = bars + BAR_K_EMPTY;
    uint64_t* v_full = bars + BAR_V_FULL;
    uint64_t* v_empty = bars + BAR_V_EMPTY;
    uint64_t* v_kv = bars + BAR_V_KV;
    uint64_t* kphi_full = bars + BAR_KPHI_FULL;
    uint64_t* qk_mapped = bars + BAR_QK_MAPPED;
    uint64_t* p_full = bars + BAR_P_FULL;
    uint64_t* p_ready = bars + BAR_P_READY;
    uint64_t* ds_full = bars + BAR_DS_FULL;
    uint64_t* ds_empty = bars + BAR_DS_EMPTY;
    uint64_t* s_full = bars + BAR_S_FULL;
    uint64_t* st_free = bars + BAR_ST_FREE;
    uint64_t* o_full = bars + BAR_O_FULL;
    uint64_t* o_empty = bars + BAR_O_EMPTY;
    uint64_t* drain_a = bars + BAR_DRAIN_A;
    uint64_t* drain_b = bars + BAR_DRAIN_B;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + BAR_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(bars + BAR_COUNT + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int cta = blockIdx.x;
    const int phi = kGeneral ? p.phi : static_cast<int>(PHI_IDENTITY);
    const bool rev = kGeneral && p.reverse;
    const bool init_t = kGeneral && p.init_transposed;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SLOTS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 2);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], PO_WARPS);
            mbar_init(&v_kv[i], 1);
            mbar_init(&kphi_full[i], STATE_WARPS);
            mbar_init(&qk_mapped[i], STATE_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&p_full[i], 1);
            mbar_init(&p_ready[i], PO_WARPS);
        }
        mbar_init(ds_full, 1);
        mbar_init(ds_empty, STATE_WARPS);
        mbar_init(s_full, STATE_WARPS);
        mbar_init(st_free, 1);
        mbar_init(o_full, 1);
        mbar_init(o_empty, PO_WARPS);
        mbar_init(drain_a, 1);
        mbar_init(drain_b, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
        prefetch_tmap(&map_o);
    }
    if (warp == WARP_MMA_A) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer: Q
        if (lane == 0) {
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = tc::item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const tc::Item it = tc::decode_item<kGeneral, KD, 1>(p, idx);
                const int nc = (it.len + C - 1) / C;
                for (int c = 0; c < nc; ++c) {
                    const int t = it.t0 + tc::chunk_row(rev, c, nc);
                    const int y = p.mode == 0 ? t : it.c1, z = p.mode == 0 ? it.c2 : t;
                    const int s = g % SLOTS, n = g / SLOTS;
                    if (n > 0 && !mbar_wait(&q_empty[s], (n - 1) & 1, abort, p.status)) { stop = true; break; }
                    uint8_t* qb = sm + OFF_Q + s * TILE;
                    mbar_arrive_expect_tx(&q_full[s], TILE);
                    tma_load_3d(qb, &map_q, &q_full[s], 0, y, z);
                    tma_load_3d(qb + PANEL, &map_q, &q_full[s], 64, y, z);
                    ++g;
                }
            }
            // no copy into shared memory may still be in flight at exit
            for (int x = (g >= SLOTS ? g - SLOTS : 0); x < g; ++x) tc::drain_wait(&q_full[x % SLOTS], (x / SLOTS) & 1);
        }
    } else if (warp == WARP_LOAD_V) {
        // ------------------------------------------------------ TMA producer: K, V
        if (lane == 0) {
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = tc::item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const tc::Item it = tc::decode_item<kGeneral, KD, 1>(p, idx);
                const int nc = (it.len + C - 1) / C;
                for (int c = 0; c < nc; ++c, ++g) {
                    const int t = it.t0 + tc::chunk_row(rev, c, nc);
                    const int y = p.mode == 0 ? t : it.c1, z = p.mode == 0 ? it.c2 : t;
                    const int s = g % SLOTS, n = g / SLOTS;
                    if (n > 0 && !mbar_wait(&k_empty[s], (n - 1) & 1, abort, p.status)) { stop = true; break; }
                    uint8_t* kb = sm + OFF_K + s * TILE;
                    mbar_arrive_expect_tx(&k_full[s], TILE);
                    tma_load_3d(kb, &map_k, &k_full[s], 0, y, z);
                    tma_load_3d(kb + PANEL, &map_k, &k_full[s], 64, y, z);
                    if (n > 0 && !mbar_wait(&v_empty[s], (n - 1) & 1, abort, p.status)) {
                        tc::drain_wait(&k_full[s], n & 1);  // the K copy just issued
                        stop = true;
                        break;
                    }
                    uint8_t* vb = sm + OFF_V + s * TILE;
                    mbar_arrive_expect_tx(&v_full[s], TILE);
                    tma_load_3d(vb, &map_v, &v_full[s], 0, y, z);
                    tma_load_3d(vb + PANEL, &map_v, &v_full[s], 64, y, z);
                }
            }
            for (int x = (g >= SLOTS ? g - SLOTS : 0); x < g; ++x) {
                tc::drain_wait(&k_full[x % SLOTS], (x / SLOTS) & 1);
                tc::drain_wait(&v_full[x % SLOTS], (x / SLOTS) & 1);
            }
        }
    } else if (warp == WARP_MMA_A) {
        // ------------------------------------------------------ MMA thread A
        // Chunk g: Q S (once S^T_{g-1} is written and O_{g-1} read out), P V
        // (once P_g is masked), then Q K^T of chunk g+1 into the other P buffer.
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);  // Q K^T   (A: Q, B: K, both K-major)
            constexpr uint32_t id_qs = idesc_bf16(128, 128, 0, 0);  // Q S     (B: S^T, K-major)
            constexpr uint32_t id_pv = idesc_bf16(128, 128, 0, 1);  // P V     (A: P in TMEM, B: V MN-major)
            const uint32_t sq = smem_u32(sm + OFF_Q), sk = smem_u32(sm + OFF_K), sv = smem_u32(sm + OFF_V);
            const uint64_t dst = tc::kmaj_desc(smem_u32(sm + OFF_ST), 0, PANEL);
            const bool mapped = phi != PHI_IDENTITY;
            // Q K^T of chunk x (Q_x and K_x landed, or mapped by the state warps)
            auto issue_qk = [&](int x) -> bool {
                const int s = x % SLOTS;
                if (mapped) {
                    if (!mbar_wait(&qk_mapped[s], (x / SLOTS) & 1, abort, p.status)) return false;
                } else {
                    if (!mbar_wait(&q_full[s], (x / SLOTS) & 1, abort, p.status)) return false;
                    if (!mbar_wait(&k_full[s], (x / SLOTS) & 1, abort, p.status)) return false;
                }
                tc_fence_after();
                const uint32_t tp = tbase + TM_P + 128u * (x & 1);
                const uint64_t da = tc::kmaj_desc(sq + s * TILE, 0, PANEL);
                const uint64_t dk = tc::kmaj_desc(sk + s * TILE, 0, PANEL);
#pragma unroll
                for (int kk = 0; kk < KD / 16; ++kk)
                    mma_ss(tp, da + tc::kmaj_step(kk, PANEL), dk + tc::kmaj_step(kk, PANEL), id_qk, kk > 0);
                mma_commit(&p_full[x & 1]);
                mma_commit(&k_empty[s]);
                return true;
            };
            int total = 0;  // this CTA's chunks
            for (int r = 0;; ++r) {
                const int idx = tc::item_index(r, cta, G);
                if (idx >= p.n_items) break;
                total += (tc::decode_item<kGeneral, KD, 1>(p, idx).len + C - 1) / C;
            }
            int g = 0;
            bool stop = total > 0 && !issue_qk(0);
            for (int r = 0; !stop; ++r) {
                const int idx = tc::item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const int len = tc::decode_item<kGeneral, KD, 1>(p, idx).len;
                for (int c0 = 0; c0 < len; c0 += C, ++g) {
                    const int s = g % SLOTS;
                    // O = Q S_{g-1}
                    if (!mbar_wait(s_full, g & 1, abort, p.status)) { stop = true; break; }
                    if (g > 0 && !mbar_wait(o_empty, (g - 1) & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    const uint64_t da = tc::kmaj_desc(sq + s * TILE, 0, PANEL);
#pragma unroll
                    for (int kk = 0; kk < KD / 16; ++kk)
                        mma_ss(tbase + TM_O, da + tc::kmaj_step(kk, PANEL), dst + tc::kmaj_step(kk, PANEL), id_qs, kk > 0);
                    mma_commit(st_free);
                    mma_commit(&q_empty[s]);
                    // O += P V; on the ragged tail of a packed sequence the product
                    // stops at the last 16-row step with valid rows (the rest cleared)
                    const int rows = len - c0;
                    const int ksteps = (p.mode == 1 && rows < C) ? (rows + 15) >> 4 : C / 16;
                    if (!mbar_wait(&p_ready[g & 1], (g >> 1) & 1, abort, p.status)) { stop = true; break; }
                    if (p.mode == 1 && ksteps * 16 > rows) clear_tail_rows2(sm + OFF_V + s * TILE, rows, ksteps);
                    tc_fence_after();
                    const uint32_t tp = tbase + TM_P + 128u * (g & 1);
                    const uint64_t dv = tc::mnmaj_desc(sv + s * TILE, 0, PANEL);
                    if (ksteps == C / 16) {
#pragma unroll
                        for (int kk = 0; kk < C / 16; ++kk)
                            mma_ts(tbase + TM_O, tp + kk * 8, dv + tc::mnmaj_step(kk), id_pv, 1);
                    } else {
#pragma unroll 1
                        for (int kk = 0; kk < ksteps; ++kk)
                            mma_ts(tbase + TM_O, tp + kk * 8, dv + tc::mnmaj_step(kk), id_pv, 1);
                    }
                    mma_commit(o_full);
                    // Q K^T of the next chunk into the other P buffer, whose last
                    // reader (P V of chunk g-1) finished before O_{g-1} was read out
                    if (g + 1 < total && !issue_qk(g + 1)) { stop = true; break; }
                }
            }
            // every MMA issued by this thread must be finished before TMEM is freed
            mma_commit(drain_a);
            tc::drain_wait(drain_a, 0);
        }
        __syncwarp();
    } else if (warp == WARP_MMA_B) {
        // ------------------------------------------------------ MMA thread B
        if (lane == 0) {
            constexpr uint32_t id_ds = idesc_bf16(128, 128, 1, 1);  // K^T V (both MN-major)
            const uint32_t sk = smem_u32(sm + OFF_K), sv = smem_u32(sm + OFF_V);
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = tc::item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const int len = tc::decode_item<kGeneral, KD, 1>(p, idx).len;
                for (int c0 = 0; c0 < len; c0 += C, ++g) {
                    const int s = g % SLOTS;
                    const int rows = len - c0;
                    const int ksteps = (p.mode == 1 && rows < C) ? (rows + 15) >> 4 : C / 16;
                    uint64_t* kready = phi != PHI_IDENTITY ? &kphi_full[s] : &k_full[s];
                    if (!mbar_wait(kready, (g / SLOTS) & 1, abort, p.status)) { stop = true; break; }
                    if (!mbar_wait(&v_full[s], (g / SLOTS) & 1, abort, p.status)) { stop = true; break; }
                    if (p.mode == 1 && ksteps * 16 > rows) clear_tail_rows2(sm + OFF_V + s * TILE, rows, ksteps);
                    // the state warps have absorbed dS_{g-1}
                    if (g > 0 && !mbar_wait(ds_empty, (g - 1) & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    const uint64_t dk = tc::mnmaj_desc(sk + s * TILE, 0, PANEL), dv = tc::mnmaj_desc(sv + s * TILE, 0, PANEL);
                    if (ksteps == C / 16) {
#pragma unroll
                        for (int kk = 0; kk < C / 16; ++kk)
                            mma_ss(tbase + TM_DS, dk + tc::mnmaj_step(kk), dv + tc::mnmaj_step(kk), id_ds, kk > 0);
                    } else {
#pragma unroll 1
                        for (int kk = 0; kk < ksteps; ++kk)
                            mma_ss(tbase + TM_DS, dk + tc::mnmaj_step(kk), dv + tc::mnmaj_step(kk), id_ds, kk > 0);
                    }
                    mma_commit(ds_full);
                    mma_commit(&k_empty[s]);
                    mma_commit(&v_kv[s]);
                }
            }
            mma_commit(drain_b);
            tc::drain_wait(drain_b, 0);
        }
        __syncwarp();
    } else if (warp < 2 + PO_WARPS) {
        // ------------------------------------------------------ P/O warps
        // Row t = 32 q4 + lane of P and O.  Mask: 32-column pieces below the
        // diagonal piece kept, the diagonal piece keeps s <= t, pieces above it
        // are zero (reverse order: above kept, s >= t, below zero); bf16 piece
        // pc goes to columns 16 pc .. 16 pc + 15 of the chunk's P buffer.
        // Output: the chunk's O rows (bf16) are staged in its V slot and stored
        // with TMA; the slot is handed back after the next chunk's mask, by
        // when the store has long read it.
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        int g = 0;
        int pending = -1;  // V slot whose O store may still be reading it
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = tc::item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const tc::Item it = tc::decode_item<kGeneral, KD, 1>(p, idx);
            const int nc = (it.len + C - 1) / C;
            for (int c = 0; c < nc; ++c, ++g) {
                const int c0 = tc::chunk_row(rev, c, nc);
                const int s = g % SLOTS;
                // --- causal mask of P_c
                if (!tc::warp_wait(&p_full[g & 1], (g >> 1) & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const uint32_t ta = tbase + lane_off + TM_P + 128u * (g & 1);
#pragma unroll 1
                for (int pc = 0; pc < 4; ++pc) {
                    uint32_t pk[16];
                    if (rev ? pc >= q4 : pc <= q4) {
                        uint32_t v[32];
                        tmem_ld32(ta + 32 * pc, v);
                        tmem_wait_ld();
                        const uint32_t keep = pc != q4 ? 0xffffffffu
                                                       : (rev ? 0xffffffffu << lane : 0xffffffffu >> (31 - lane));
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = pack_bf16x2((keep & (1u << (2 * i))) ? __uint_as_float(v[2 * i]) : 0.f,
                                                (keep & (2u << (2 * i))) ? __uint_as_float(v[2 * i + 1]) : 0.f);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[i] = 0u;
                    }
                    tmem_st16(ta + 16 * pc, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                // the previous chunk's O store has read its V slot by now: hand
                // the slot back before anything waits on a V tile
                if (pending >= 0) {
                    if (lane == 0) {
                        bulk_wait_read<0>();
                        mbar_arrive(&v_empty[pending]);
                    }
                    __syncwarp();
                    pending = -1;
                }
                // P V also needs V_c
                if (!tc::warp_wait(&v_full[s], (g / SLOTS) & 1, abort, p.status)) { stop = true; break; }
                if (lane == 0) mbar_arrive(&p_ready[g & 1]);
                // --- O_c: TMEM -> bf16 -> the V slot of chunk c -> TMA store, one
                // 64-column half at a time (TMEM is released after the second load);
                // P V (o_full) and K^T V (v_kv) are then done with the V tile
                if (!tc::warp_wait(o_full, g & 1, abort, p.status)) { stop = true; break; }
                if (!tc::warp_wait(&v_kv[s], (g / SLOTS) & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
                const int rows = it.len - c0;
                // 0: this warp's rows all lie past the end of the sequence; 1: the
                // 32 rows go through the staging tile (a dense tensor clips rows
                // past N itself); 2: ragged tail of a packed sequence, whose next
                // rows belong to another sequence: plain row stores
                const int how = q4 * 32 >= rows ? 0 : (p.mode == 0 || q4 * 32 + 32 <= rows) ? 1 : 2;
                uint8_t* stg = sm + OFF_V + s * TILE + q4 * 4096;  // this warp's 32 rows of each panel
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tbase + lane_off + TM_O + 64 * h, v0);
                    tmem_ld32(tbase + lane_off + TM_O + 64 * h + 32, v1);
                    tmem_wait_ld();
                    if (h == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(o_empty);
                    }
                    uint32_t hp[32];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        hp[e] = pack_bf16x2(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
                        hp[16 + e] = pack_bf16x2(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
                    }
                    if (how == 1) {
                        const uint32_t sa = smem_u32(stg + h * PANEL) + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            st_shared_v4(sa + ((static_cast<uint32_t>(ch) ^ (row & 7)) << 4), hp[4 * ch], hp[4 * ch + 1],
                                         hp[4 * ch + 2], hp[4 * ch + 3]);
                    } else if (how == 2 && row < rows) {
                        uint4* dst = reinterpret_cast<uint4*>(p.o + ((long)(it.t0 + c0 + row) * p.H + it.c1) * p.dv);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            dst[8 * h + ch] = make_uint4(hp[4 * ch], hp[4 * ch + 1], hp[4 * ch + 2], hp[4 * ch + 3]);
                    }
                }
                if (how == 1) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (p.mode == 0) tma_store_3d(&map_o, stg + h * PANEL, 64 * h, it.t0 + c0 + q4 * 32, it.c2);
                            else tma_store_3d(&map_o, stg + h * PANEL, 64 * h, it.c1, it.t0 + c0 + q4 * 32);
                        }
                        bulk_commit();
                    }
                }
                __syncwarp();
                pending = s;
            }
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ------------------------------------------------------ state warps
        // Warp w holds S[i][64 h + j], j < 64, for key dim i = 32 (w & 3) + lane
        // (the TMEM lane quarter it may read) and h = (w - 6) / 4.
        const int sw = warp - (2 + PO_WARPS);     // 0 .. 7
        const int h = sw >> 2;
        const int q4 = warp & 3;
        const int i = q4 * 32 + lane;
        const int tid = sw * 32 + lane;           // 0 .. 255, for the feature map
        const uint32_t ta0 = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_DS + 64u * h;
        // bf16(S[i][64 h + j]) goes to row 64 h + j, key dim i, of the S^T tile;
        // a warp's 32 two-byte stores of one row fill 4 distinct 16-byte chunks
        const uint32_t colchunk = static_cast<uint32_t>((i & 63) >> 3);
        uint8_t* st_base = sm + OFF_ST + (i >> 6) * PANEL + 64 * h * 128 + (i & 7) * 2;
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = tc::item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const tc::Item it = tc::decode_item<kGeneral, KD, 1>(p, idx);
            float S[64];
            if (it.init && init_t) {
                const float* src = it.init + (long)64 * h * KD + i;  // column i of the transposed block
#pragma unroll
                for (int j = 0; j < 64; ++j) S[j] = src[(long)j * KD];
            } else if (it.init) {
                const float4* src = reinterpret_cast<const float4*>(it.init + (long)i * p.dv + 64 * h);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 x = src[j];
                    S[4 * j] = x.x; S[4 * j + 1] = x.y; S[4 * j + 2] = x.z; S[4 * j + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) S[j] = 0.f;
            }
            // phi(K), then phi(Q), of the chunk with global index gg (slot gg %
            // SLOTS), in place, before the tensor cores read them
            auto map_chunk = [&](long gg) -> bool {
                const int sg = static_cast<int>(gg % SLOTS);
                const uint32_t par = static_cast<uint32_t>((gg / SLOTS) & 1);
                if (!tc::warp_wait(&k_full[sg], par, abort, p.status)) return false;
                phi_tile2(smem_u32(sm + OFF_K + sg * TILE), tid, phi);
                __syncwarp();
                if (lane == 0) mbar_arrive(&kphi_full[sg]);
                if (!tc::warp_wait(&q_full[sg], par, abort, p.status)) return false;
                phi_tile2(smem_u32(sm + OFF_Q + sg * TILE), tid, phi);
                __syncwarp();
                if (lane == 0) mbar_arrive(&qk_mapped[sg]);
                return true;
            };
            // with kAhead (elu + 1: exponentials) an item's later chunks are
            // mapped a chunk ahead (below), so that the mapping is not queued
            // behind the state update on the way to the next chunk's Q K^T;
            // relu's packed max is cheap enough to map each chunk at its start
            constexpr bool ahead = kAhead;
            for (int c0 = 0; c0 < it.len; c0 += C, ++g) {
                if (kGeneral && phi != PHI_IDENTITY && (c0 == 0 || !ahead) && !map_chunk(g)) { stop = true; break; }
                // publish bf16(S_{c-1})^T once Q S of the previous chunk has read the old one
                if (g > 0 && !tc::warp_wait(st_free, (g - 1) & 1, abort, p.status)) { stop = true; break; }
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    reinterpret_cast<__nv_bfloat16*>(st_base + j * 128 + ((colchunk ^ static_cast<uint32_t>(j & 7)) << 4))[0] =
                        __float2bfloat16_rn(S[j]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_full);
                if (kGeneral && ahead && c0 + C < it.len && !map_chunk(g + 1)) { stop = true; break; }
                // absorb dS_c
                if (!tc::warp_wait(ds_full, g & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[32];
                    tmem_ld32(ta0 + 32 * h2, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * h2 + j] += __uint_as_float(v[j]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(ds_empty);
            }
            if (stop) break;
            if (p.s_out && it.write_state) {
                float4* dst = reinterpret_cast<float4*>(p.s_out + (it.state * KD + i) * p.dv + 64 * h);
#pragma unroll
                for (int j = 0; j < 16; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA_A) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

}  // namespace tcw
}  // namespace lcl

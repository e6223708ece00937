// Chunked causal linear attention on tcgen05 tensor cores (bf16 in, fp32 state).
//
// For every chunk c of C = 128 tokens of one (sequence, head) the kernel forms
// the tiled Lightning Attention update (page "MiniMax: «Почему M2 в итоге стала
// моделью с полным вниманием?» (конспект)", section 1, glossary entry
// "Lightning Attention": masked matrix inside the block, K^T V state between
// blocks) of the recurrence S_t = S_{t-1} + k_t v_t^T, o_t = q_t S_t (page
// "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"):
//
//   [P_c | O_c] = Q_c [K_c ; S_{c-1}^T]^T  one N = 192 tcgen05 product, fp32 in TMEM
//   P_c  <- P_c ⊙ M  (keep s <= t), bf16   mask warps, written back into TMEM
//   O_c  += P_c V_c                        tcgen05 with A = P_c read from TMEM
//   dS_c  = K_c^T V_c                      tcgen05 (K, V read MN-major)
//   S_c   = S_{c-1} + dS_c                 fp32, in the state warps' registers
//
// Work item = (sequence or batch*head unit, head, 64-wide slice of d_v).  One
// CTA (persistent over items) holds the item's state slice S[:, slice] in
// fp32 registers of four "state" warps; the tensor cores see it as bf16(S)^T,
// written by those warps right behind the chunk's K rows, so Q is read once for
// both Q K^T and Q S.  Warp roles (16 warps):
//   w0 lane 0  : TMA producer for Q and K (2 slots each)
//   w15 lane 0 : TMA producer for V (3 slots)
//   w1 lane 0  : MMA thread A: [P|O] of the NEXT chunk, then P V of this chunk
//   w14 lane 0 : MMA thread B: K^T V (depends only on the loaded tiles, runs ahead)
//   w2..w5     : mask warps   (P: TMEM -> regs -> causal mask -> bf16 -> TMEM)
//   w6..w9     : state warps  (dS: TMEM -> regs, S += dS, bf16(S)^T -> smem)
//   w10..w13   : output warps (O: TMEM -> regs -> bf16 -> smem -> TMA store)
// [P|O] is double-buffered in TMEM, so chunk c+1's product and mask overlap
// chunk c's P V and output.  A Q slot is released after the [P|O] product, a K
// slot (with its S^T rows) after both that product and K^T V, a V slot after
// both P V and K^T V.  Every wait is bounded (see mbar_wait); a timeout stops
// the CTA cleanly.
#pragma once
#include "sm100.cuh"
#include "phi.cuh"

namespace lcl {
namespace tc {

constexpr int C = 128;         // chunk length (tokens)
constexpr int DK = 128;        // largest key dim (the shared-memory layout is sized for it)
constexpr int DVS = 64;        // value columns per CTA
constexpr int Q_SLOTS = 2;
constexpr int K_SLOTS = 2;
constexpr int V_SLOTS = 3;
// No L2 prefetch ahead of the TMA loads: measured on the long prefill and the
// 8K batch, prefetching three chunks ahead was 2-6 % slower than none (the
// prefetches queue in front of the demand loads).
constexpr int PANEL = 128 * 128;       // 128 rows x 128 bytes, 128B-swizzled
constexpr int KPANEL = PANEL + DVS * 128;  // K rows 0..127, then S^T rows (one per value column)
constexpr int TILE_Q = 2 * PANEL;          // Q: two 64-column panels
constexpr int TILE_K = 2 * KPANEL;         // K with S^T: two 64-column panels
constexpr int OST_WARP = 32 * 128;         // output staging: 32 rows x 128 bytes per warp
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_SLOTS * TILE_Q;
constexpr int OFF_V = OFF_K + K_SLOTS * TILE_K;
constexpr int OFF_OST = OFF_V + V_SLOTS * PANEL;
constexpr int OFF_BAR = OFF_OST + 4 * OST_WARP;
static_assert(KPANEL % 1024 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_OST % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
// mbarrier slots (8 bytes each) at OFF_BAR, then the TMEM base and the abort flag
constexpr int BAR_Q_FULL = 0;
constexpr int BAR_Q_EMPTY = BAR_Q_FULL + Q_SLOTS;
constexpr int BAR_K_FULL = BAR_Q_EMPTY + Q_SLOTS;
constexpr int BAR_K_EMPTY = BAR_K_FULL + K_SLOTS;
constexpr int BAR_S_FULL = BAR_K_EMPTY + K_SLOTS;   // per K slot: S^T rows written
constexpr int BAR_V_FULL = BAR_S_FULL + K_SLOTS;
constexpr int BAR_V_EMPTY = BAR_V_FULL + V_SLOTS;
constexpr int BAR_P_FULL = BAR_V_EMPTY + V_SLOTS;   // [2]
constexpr int BAR_P_READY = BAR_P_FULL + 2;         // [2]
constexpr int BAR_O_FULL = BAR_P_READY + 2;         // [2]
constexpr int BAR_O_EMPTY = BAR_O_FULL + 2;         // [2]
constexpr int BAR_DS_FULL = BAR_O_EMPTY + 2;        // [2]
constexpr int BAR_DS_EMPTY = BAR_DS_FULL + 2;       // [2]
constexpr int BAR_KPHI_FULL = BAR_DS_EMPTY + 2;     // [K_SLOTS] state (phi applied to K) -> B
constexpr int BAR_DRAIN_A = BAR_KPHI_FULL + K_SLOTS;
constexpr int BAR_DRAIN_B = BAR_DRAIN_A + 1;
constexpr int BAR_COUNT = BAR_DRAIN_B + 1;
constexpr int BAR_BYTES = 512;
static_assert((BAR_COUNT + 2) * 8 <= BAR_BYTES, "barrier area too small");
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB per-block shared memory limit");
constexpr int NUM_THREADS = 512;
// value slices per head: d_v / DVS (2 at d = 128, 1 at d = 64; d_k = d_v)
constexpr int WARP_MMA_A = 1;
constexpr int WARP_MMA_B = 14;
constexpr int WARP_LOAD_V = 15;

// TMEM columns: buffer b of [P (128, fp32; bf16 P later in its first 64) | O (64)]
// starts at 256 b; dS buffer b (64) at 192 + 256 b.
constexpr uint32_t TM_PO_STRIDE = 256;
constexpr uint32_t TM_O_OFF = 128;
constexpr uint32_t TM_DS = 192;
constexpr uint32_t TMEM_COLS = 512;

struct Params {
    int mode;              // 0 = dense [U][N][d]; 1 = packed [T][H][d]
    int n_items;           // work items
    int H;                 // heads (packed layout)
    int N;                 // tokens per unit (dense)
    int dv;                // full value dim (= slices * DVS), equal to the key dim
    const int* cu_seqlens; // packed: [n_seq + 1]
    const int* order;      // packed: sequence indices, longest first
    const float* s0;       // dense: [U][DK][dv] or null
    const float* pool;     // packed: [n_pool][H][DK][dv] or null
    const int* init_idx;   // packed: [n_seq] or null
    float* s_out;          // [U or n_seq*H or U*n_seg][DK][dv] or null
    __nv_bfloat16* o;      // output base, for direct stores of ragged tails
    int* status;           // device status word
    // dense only: the sequence of each unit cut into n_seg segments of seg_len
    // tokens (a multiple of C; the last one may be shorter)
    int n_seg;
    int seg_len;
    const float* seg_init; // [U][n_seg][DK][dv]: state before each segment, or null (then s0)
    int s_out_per_seg;     // 1: s_out holds the state after every segment, [U][n_seg][DK][dv]
    int state_only;        // 1: only the state is computed (no Q, no outputs)
    int phi;               // feature map on q and k (phi.cuh); applied to the tiles in smem
    // dense, one segment only: visit the chunks last to first and keep s >= t
    // inside a chunk, so that o_t = q_t (S_init + sum_{s >= t} k_s v_s^T)
    int reverse;
    int init_transposed;   // the initial state is given as its transpose [dv][DK]
    int seg_base;          // dense: the items' segments are seg_base .. seg_base + n_seg - 1
    int dk;                // key dim = value dim: 128 or 64 (selects the kernel instance)
    // packed only: segments of *seg_len_dev tokens (the length and the offsets
    // in work order over n_seq sequences from vorder::seg_plan_kernel), or null
    const int* seg_off;
    const int* seg_off_nl;
    const int* seg_len_dev;
    int n_seq;
};

struct Item {
    int t0;         // first token (packed: absolute row; dense: segment start)
    int len;        // tokens
    int c1, c2;     // TMA coordinates (dense: unit in c2; packed: head in c1)
    int vs;         // value slice
    long state;     // index of the (unit | sequence*H + head | unit*n_seg + segment) state
    const float* init;  // initial state row block or null
    bool write_state;   // the item's final state goes to s_out
};

__device__ __forceinline__ int item_index(int round, int cta, int grid) {
    // boustrophedon order over CTAs keeps per-CTA totals balanced when items
    // arrive longest first
    return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// First token (relative to the item's start) of the c-th chunk in visiting order.
__device__ __forceinline__ int chunk_row(bool rev, int c, int nc) { return (rev ? nc - 1 - c : c) * C; }

// kGeneral = false: dense items are whole sequences (n_seg = 1).  KD: key dim.
// NV: value slices per unit (KD / DVS here; 1 for the full-width kernel).
template <bool kGeneral, int KD, int NV = KD / DVS>
__device__ __forceinline__ Item decode_item(const Params& p, int idx) {
    Item it;
    it.vs = idx % NV;
    if (!kGeneral && p.mode == 0) {
        const int u = idx / NV;
        it.t0 = 0;
        it.len = p.N;
        it.c1 = 0;
        it.c2 = u;
        it.state = u;
        it.init = p.s0 ? p.s0 + (long)u * KD * p.dv : nullptr;
        it.write_state = true;
    } else if (p.mode == 0) {
        const int us = idx / NV;  // unit * n_seg + segment
        const int u = us / p.n_seg, sg = us - u * p.n_seg;
        // the segment visited first starts from s0; the one visited last ends the sequence
        const int first = p.reverse ? p.n_seg - 1 : 0, last = p.reverse ? 0 : p.n_seg - 1;
        it.t0 = (sg + p.seg_base) * p.seg_len;
        it.len = min(p.seg_len, p.N - it.t0);
        it.c1 = 0;
        it.c2 = u;
        it.state = p.s_out_per_seg ? us : u;
        it.init = p.seg_init ? p.seg_init + (long)us * KD * p.dv
                             : ((sg == first && p.s0) ? p.s0 + (long)u * KD * p.dv : nullptr);
        it.write_state = p.s_out_per_seg || sg == last;
    } else if (kGeneral && p.seg_off) {
        // packed batch cut into segments of seg_len tokens: item = (segment in
        // work order, head, slice); the state-only pass numbers only the
        // segments that are not a sequence's last.  Items past the device-side
        // total (the host launches an upper bound) are empty.
        const int* off = p.state_only ? p.seg_off_nl : p.seg_off;
        const int hs = idx / NV;    // segment * H + head
        const int sgi = hs / p.H;
        const int h = hs - sgi * p.H;
        it.c1 = h;
        it.c2 = 0;
        if (sgi >= off[p.n_seq]) {
            it.t0 = 0;
            it.len = 0;
            it.state = 0;
            it.init = nullptr;
            it.write_state = false;
        } else {
            int lo = 0, hi = p.n_seq;  // rank r with off[r] <= sgi < off[r + 1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (off[mid] <= sgi) lo = mid;
                else hi = mid;
            }
            const int r = lo, sg = sgi - off[r];
            const int seq = p.order[r];
            const int end = p.cu_seqlens[seq + 1], sl = *p.seg_len_dev;
            it.t0 = p.cu_seqlens[seq] + sg * sl;
            it.len = max(0, min(sl, end - it.t0));
            if (p.state_only) {
                it.state = (long)sgi * p.H + h;  // index of this segment's sum
                it.init = nullptr;
                it.write_state = true;
            } else {
                it.state = (long)seq * p.H + h;
                it.init = p.seg_init + ((long)sgi * p.H + h) * KD * p.dv;
                it.write_state = sgi == off[r + 1] - 1;  // the sequence's last segment
            }
        }
    } else {
        const int hs = idx / NV;    // sequence rank * H + head
        const int r = hs / p.H;
        const int h = hs - r * p.H;
        const int seq = p.order ? p.order[r] : r;
        it.t0 = p.cu_seqlens[seq];
        it.len = p.cu_seqlens[seq + 1] - it.t0;
        it.c1 = h;
        it.c2 = 0;
        it.state = (long)seq * p.H + h;
        const int ii = p.init_idx ? p.init_idx[seq] : -1;
        it.init = (p.pool && ii >= 0) ? p.pool + ((long)ii * p.H + h) * KD * p.dv : nullptr;
        it.write_state = true;
    }
    return it;
}

// Wait on an mbarrier from a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
    const bool ok = mbar_wait(bar, parity, abort, status);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait used only while draining on the way out (ignores the abort flag).
__device__ __noinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > 200000000ull) break;
    }
}

// Rows past the end of a packed sequence inside its last 16-row step belong to
// the next sequence; clear them in a V tile before a product over the token
// dim.  Both issuing threads clear the same rows (identical zero writes), each
// before its own product, so neither has to wait for the other.
__device__ __noinline__ void clear_tail_rows(uint8_t* tile, int rows, int ksteps) {
    for (int e = rows * 128; e < ksteps * 16 * 128; e += 16)
        *reinterpret_cast<uint4*>(tile + e) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
}

// phi in place on the 128 token rows of the NP 64-column panels of a Q or K
// tile (panels `stride` bytes apart; the S^T rows behind K are left alone),
// by the 128 state-warp threads t = 0 .. 127, in 16-byte vectors with four
// loads in flight.  Only the feature-map instance carries this code.
template <int NP>
__device__ __forceinline__ void phi_tile(uint32_t base, uint32_t stride, int t, int phi) {
    constexpr int PER_PANEL = PANEL / 16;
    constexpr int PER_THREAD = NP * PER_PANEL / 128;
#pragma unroll 1
    for (int j0 = 0; j0 < PER_THREAD; j0 += 4) {
        uint32_t a[4];
        uint4 r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = t + (j0 + j) * 128;
            a[j] = base + static_cast<uint32_t>(e / PER_PANEL) * stride + static_cast<uint32_t>(e % PER_PANEL) * 16u;
            r[j] = ld_shared_v4(a[j]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 y = apply_phi_bf16x8(r[j], phi);
            st_shared_v4(a[j], y.x, y.y, y.z, y.w);
        }
    }
    fence_proxy_async_smem();
}

// Shared-memory descriptor of K-step kk (16 along the contraction dim):
// K-major tiles step 32 B inside a 64-column panel (panels `panel` bytes
// apart), MN-major tiles step 16 rows of 128 B.
__device__ __forceinline__ uint64_t kmaj_desc(uint32_t base, int kk, uint32_t panel) {
    return sw128_desc(base + static_cast<uint32_t>(kk >> 2) * panel + static_cast<uint32_t>(kk & 3) * 32u, 16, 1024);
}
__device__ __forceinline__ uint64_t mnmaj_desc(uint32_t base, int kk, uint32_t lbo) {
    return sw128_desc(base + static_cast<uint32_t>(kk) * 2048u, lbo, 1024);
}

// The same descriptors as K-step offsets (16-byte units) from the K-step-0
// descriptor, for unrolled issue loops: the tcgen05.mma operands then need no
// per-instruction address arithmetic in the issuing thread.
__device__ __forceinline__ constexpr uint64_t kmaj_step(int kk, uint32_t panel) {
    return static_cast<uint64_t>((static_cast<uint32_t>(kk >> 2) * panel + static_cast<uint32_t>(kk & 3) * 32u) >> 4);
}
__device__ __forceinline__ constexpr uint64_t mnmaj_step(int kk) { return static_cast<uint64_t>(kk) * (2048u >> 4); }

// The code below is kept compact on purpose: all warps of all SMs run their
// roles' loops at once, so the kernel's instruction footprint (not only its
// instruction count) decides how often warps stall on instruction fetch.
// kGeneral = false is the lean instance for the common case (feature map
// identity, chunks in order, outputs computed, initial state as given, whole
// sequences): the options below are then compile-time constants and their
// code is left out.  kPhi (with kGeneral) adds the feature map on Q and K
// tiles; without it the general instance keeps the identity and stays
// smaller.  KD = d_k = d_v: 128 (two 64-column panels per Q and K tile, two
// value slices per head) or 64 (one panel, one slice).
template <bool kGeneral, bool kPhi, int KD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                  const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* q_full = bars + BAR_Q_FULL;      // [Q_SLOTS] TMA -> state warps
    uint64_t* q_empty = bars + BAR_Q_EMPTY;    // [Q_SLOTS] A (after [P|O]) -> TMA
    uint64_t* k_full = bars + BAR_K_FULL;      // [K_SLOTS] TMA -> state warps, B
    uint64_t* k_empty = bars + BAR_K_EMPTY;    // [K_SLOTS] A ([P|O]) + B (K^T V) -> TMA, state
    uint64_t* s_full = bars + BAR_S_FULL;      // [K_SLOTS] state -> A: S^T written, Q and K landed
    uint64_t* v_full = bars + BAR_V_FULL;      // [V_SLOTS] TMA -> mask warps, B
    uint64_t* v_empty = bars + BAR_V_EMPTY;    // [V_SLOTS] A (P V) + B (K^T V) -> TMA
    uint64_t* p_full = bars + BAR_P_FULL;      // [2] A -> mask
    uint64_t* p_ready = bars + BAR_P_READY;    // [2] mask -> A: bf16 P written, V landed
    uint64_t* o_full = bars + BAR_O_FULL;      // [2] A (after P V) -> output
    uint64_t* o_empty = bars + BAR_O_EMPTY;    // [2] output -> A
    uint64_t* ds_full = bars + BAR_DS_FULL;    // [2] B -> state
    uint64_t* ds_empty = bars + BAR_DS_EMPTY;  // [2] state -> B
    uint64_t* kphi_full = bars + BAR_KPHI_FULL;  // [K_SLOTS] state (phi(K) written) -> B, when phi is not the identity
    uint64_t* drain_a = bars + BAR_DRAIN_A;
    uint64_t* drain_b = bars + BAR_DRAIN_B;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + BAR_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(bars + BAR_COUNT + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int cta = blockIdx.x;
    const bool state_only = kGeneral && p.state_only;
    const int phi = kGeneral && kPhi ? p.phi : static_cast<int>(PHI_IDENTITY);
    const bool rev = kGeneral && p.reverse;
    const bool init_t = kGeneral && p.init_transposed;
    constexpr int NP = KD / 64;  // 64-column panels per Q / K tile

    if (threadIdx.x == 0) {
        for (int i = 0; i < Q_SLOTS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < K_SLOTS; ++i) {
            mbar_init(&kphi_full[i], 4);
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], state_only ? 1 : 2);
            mbar_init(&s_full[i], 4);
        }
        for (int i = 0; i < V_SLOTS; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], state_only ? 1 : 2);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&p_full[i], 1);
            mbar_init(&p_ready[i], 4);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 4);
            mbar_init(&ds_full[i], 1);
            mbar_init(&ds_empty[i], 4);
        }
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
        // ------------------------------------------------------ TMA producer: Q, K
        if (lane == 0) {
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const Item it = decode_item<kGeneral, KD>(p, idx);
                const int nc = (it.len + C - 1) / C;
                for (int c = 0; c < nc; ++c) {
                    const int t = it.t0 + chunk_row(rev, c, nc);
                    const int y = p.mode == 0 ? t : it.c1, z = p.mode == 0 ? it.c2 : t;
                    const int qs = g % Q_SLOTS, kq = g / Q_SLOTS;
                    if (!state_only) {
                        if (kq > 0 && !mbar_wait(&q_empty[qs], (kq - 1) & 1, abort, p.status)) { stop = true; break; }
                        uint8_t* qb = sm + OFF_Q + qs * TILE_Q;
                        mbar_arrive_expect_tx(&q_full[qs], NP * PANEL);
#pragma unroll
                        for (int pn = 0; pn < NP; ++pn) tma_load_3d(qb + pn * PANEL, &map_q, &q_full[qs], 64 * pn, y, z);
                    }
                    const int ks = g % K_SLOTS, kk_ = g / K_SLOTS;
                    if (kk_ > 0 && !mbar_wait(&k_empty[ks], (kk_ - 1) & 1, abort, p.status)) { stop = true; break; }
                    uint8_t* kb = sm + OFF_K + ks * TILE_K;
                    mbar_arrive_expect_tx(&k_full[ks], NP * PANEL);
#pragma unroll
                    for (int pn = 0; pn < NP; ++pn) tma_load_3d(kb + pn * KPANEL, &map_k, &k_full[ks], 64 * pn, y, z);
                    ++g;
                }
            }
            // make sure no copy into shared memory is still in flight at exit
            for (int x = (g >= Q_SLOTS ? g - Q_SLOTS : 0); x < g; ++x) {
                if (!state_only) drain_wait(&q_full[x % Q_SLOTS], (x / Q_SLOTS) & 1);
                drain_wait(&k_full[x % K_SLOTS], (x / K_SLOTS) & 1);
            }
        }
    } else if (warp == WARP_LOAD_V) {
        // ------------------------------------------------------ TMA producer: V
        if (lane == 0) {
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const Item it = decode_item<kGeneral, KD>(p, idx);
                const int nc = (it.len + C - 1) / C;
                for (int c = 0; c < nc; ++c, ++g) {
                    const int t = it.t0 + chunk_row(rev, c, nc);
                    const int y = p.mode == 0 ? t : it.c1, z = p.mode == 0 ? it.c2 : t;
                    const int vc = g % V_SLOTS, kv = g / V_SLOTS;
                    if (kv > 0 && !mbar_wait(&v_empty[vc], (kv - 1) & 1, abort, p.status)) { stop = true; break; }
                    mbar_arrive_expect_tx(&v_full[vc], PANEL);
                    tma_load_3d(sm + OFF_V + vc * PANEL, &map_v, &v_full[vc], DVS * it.vs, y, z);
                }
            }
            for (int x = (g >= V_SLOTS ? g - V_SLOTS : 0); x < g; ++x)
                drain_wait(&v_full[x % V_SLOTS], (x / V_SLOTS) & 1);
        }
    } else if (warp == WARP_MMA_A) {
        // ------------------------------------------------------ MMA thread A
        // Software-pipelined by one chunk: [P|O] of chunk g+1 is issued before
        // P V of chunk g, so its mask runs while P V and the next product are
        // queued.  TMEM written or read by other warps is ordered by
        // tcgen05.fence::after_thread_sync after the barrier.
        if (lane == 0 && !state_only) {
            constexpr uint32_t id_f = idesc_bf16(128, C + DVS, 0, 0);  // Q [K ; S^T]^T
            constexpr uint32_t id_pv = idesc_bf16(128, DVS, 0, 1);     // P V (P from TMEM)
            const uint32_t sq = smem_u32(sm + OFF_Q), sk = smem_u32(sm + OFF_K), sv = smem_u32(sm + OFF_V);
            int total = 0;  // this CTA's chunks
            for (int r = 0;; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                total += (decode_item<kGeneral, KD>(p, idx).len + C - 1) / C;
            }
            int k = 0;  // next chunk whose [P|O] is to be issued
            int g = 0;  // chunk whose P V is issued next
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const int len = decode_item<kGeneral, KD>(p, idx).len;
                for (int c0 = 0; c0 < len; c0 += C, ++g) {
                    // [P | O] = Q [K ; S^T]^T for chunks up to g + 1  (A: Q, B: K rows then S^T rows)
                    for (; k <= g + 1 && k < total; ++k) {
                        const int qs = k % Q_SLOTS, ks = k % K_SLOTS, b = k & 1;
                        if (!mbar_wait(&s_full[ks], (k / K_SLOTS) & 1, abort, p.status)) { stop = true; break; }
                        // the O buffer it writes, last used by chunk k - 2, has been read out
                        if (k >= 2 && !mbar_wait(&o_empty[b], ((k - 2) >> 1) & 1, abort, p.status)) { stop = true; break; }
                        tc_fence_after();
                        const uint32_t tpo = tbase + TM_PO_STRIDE * b;
                        const uint64_t da = kmaj_desc(sq + qs * TILE_Q, 0, PANEL);
                        const uint64_t db = kmaj_desc(sk + ks * TILE_K, 0, KPANEL);
#pragma unroll
                        for (int kk = 0; kk < KD / 16; ++kk)
                            mma_ss(tpo, da + kmaj_step(kk, PANEL), db + kmaj_step(kk, KPANEL), id_f, kk > 0);
                        mma_commit(&p_full[b]);
                        mma_commit(&q_empty[qs]);
                        mma_commit(&k_empty[ks]);
                    }
                    if (stop) break;
                    // O += P V   (A: masked bf16 P in TMEM, B: V MN-major).  On the
                    // ragged tail of a packed sequence the product stops at the last
                    // 16-row step with valid rows, whose invalid V rows are cleared.
                    const int vc = g % V_SLOTS, b = g & 1;
                    const int rows = len - c0;
                    const int ksteps = (p.mode == 1 && rows < C) ? (rows + 15) >> 4 : C / 16;
                    if (!mbar_wait(&p_ready[b], (g >> 1) & 1, abort, p.status)) { stop = true; break; }
                    if (p.mode == 1 && ksteps * 16 > rows) clear_tail_rows(sm + OFF_V + vc * PANEL, rows, ksteps);
                    tc_fence_after();
                    const uint32_t tpo = tbase + TM_PO_STRIDE * b;
                    const uint64_t dv = mnmaj_desc(sv + vc * PANEL, 0, PANEL);
                    if (ksteps == C / 16) {
#pragma unroll
                        for (int kk = 0; kk < C / 16; ++kk) mma_ts(tpo + TM_O_OFF, tpo + kk * 8, dv + mnmaj_step(kk), id_pv, 1);
                    } else {
#pragma unroll 1
                        for (int kk = 0; kk < ksteps; ++kk) mma_ts(tpo + TM_O_OFF, tpo + kk * 8, dv + mnmaj_step(kk), id_pv, 1);
                    }
                    mma_commit(&o_full[b]);
                    mma_commit(&v_empty[vc]);
                }
            }
            // every MMA issued by this thread must be finished before TMEM is freed
            mma_commit(drain_a);
            drain_wait(drain_a, 0);
        }
        __syncwarp();
    } else if (warp == WARP_MMA_B) {
        // ------------------------------------------------------ MMA thread B
        // K^T V, which only depends on the loaded tiles: this thread runs ahead
        // and hands each dS_c to the state warps early.
        if (lane == 0) {
            constexpr uint32_t id_ds = idesc_bf16(128, DVS, 1, 1);  // K^T V
            const uint32_t sk = smem_u32(sm + OFF_K), sv = smem_u32(sm + OFF_V);
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const int len = decode_item<kGeneral, KD>(p, idx).len;
                for (int c0 = 0; c0 < len; c0 += C, ++g) {
                    const int ks = g % K_SLOTS, vc = g % V_SLOTS, b = g & 1;
                    const int rows = len - c0;
                    const int ksteps = (p.mode == 1 && rows < C) ? (rows + 15) >> 4 : C / 16;
                    // dS = K^T V   (A: K MN-major over 2 panels, B: V MN-major)
                    uint64_t* kready = phi != PHI_IDENTITY ? &kphi_full[ks] : &k_full[ks];
                    if (!mbar_wait(kready, (g / K_SLOTS) & 1, abort, p.status)) { stop = true; break; }
                    if (!mbar_wait(&v_full[vc], (g / V_SLOTS) & 1, abort, p.status)) { stop = true; break; }
                    if (p.mode == 1 && ksteps * 16 > rows) clear_tail_rows(sm + OFF_V + vc * PANEL, rows, ksteps);
                    if (g >= 2 && !mbar_wait(&ds_empty[b], ((g - 2) >> 1) & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t tds = tbase + TM_DS + TM_PO_STRIDE * b;
                    // A = K^T, 128 rows of key dims: at d = 64 the second 64-row half reads
                    // the same panel again (leading offset 0), so dS rows 64..127 repeat
                    // rows 0..63 and are ignored
                    const uint64_t dk = mnmaj_desc(sk + ks * TILE_K, 0, KD == 128 ? KPANEL : 0),
                                   dv = mnmaj_desc(sv + vc * PANEL, 0, PANEL);
                    if (ksteps == C / 16) {
#pragma unroll
                        for (int kk = 0; kk < C / 16; ++kk) mma_ss(tds, dk + mnmaj_step(kk), dv + mnmaj_step(kk), id_ds, kk > 0);
                    } else {
#pragma unroll 1
                        for (int kk = 0; kk < ksteps; ++kk) mma_ss(tds, dk + mnmaj_step(kk), dv + mnmaj_step(kk), id_ds, kk > 0);
                    }
                    mma_commit(&ds_full[b]);
                    mma_commit(&k_empty[ks]);
                    mma_commit(&v_empty[vc]);
                }
            }
            mma_commit(drain_b);
            drain_wait(drain_b, 0);
        }
        __syncwarp();
    } else if (warp < 6) {
        if (!state_only) {
            // ------------------------------------------------------ mask warps
            // Row t = 32 q4 + lane of P; 32-column piece pc holds keys 32 pc ...
            // Pieces below the diagonal piece are kept whole, the diagonal piece
            // keeps s <= t, pieces above it are zero (in reverse order: pieces
            // above kept, s >= t on the diagonal, pieces below zero).  bf16
            // piece pc goes to columns 16 pc .. 16 pc + 15, which only overlap
            // fp32 pieces already read.
            const int q4 = warp & 3;
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const int len = decode_item<kGeneral, KD>(p, idx).len;
                for (int c0 = 0; c0 < len; c0 += C, ++g) {
                    const int b = g & 1;
                    if (!warp_wait(&p_full[b], (g >> 1) & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_PO_STRIDE * b;
#pragma unroll 1
                    for (int pc = 0; pc < 4; ++pc) {
                        uint32_t pk[16];
                        if (rev ? pc >= q4 : pc <= q4) {
                            uint32_t v[32];
                            tmem_ld32(ta + 32 * pc, v);
                            tmem_wait_ld();
                            // bit j: column j of the piece is kept
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
                    // the P V product of this chunk also needs V_c
                    if (!warp_wait(&v_full[g % V_SLOTS], (g / V_SLOTS) & 1, abort, p.status)) { stop = true; break; }
                    if (lane == 0) mbar_arrive(&p_ready[b]);
                }
            }
        }
    } else if (warp < 10) {
        // ------------------------------------------------------ state warps
        const int q4 = warp & 3;
        const int i = q4 * 32 + lane;  // key-dim row of S owned by this thread
        const bool own = KD == 128 || q4 < KD / 32;  // warp-uniform; at d = 64 warps 8, 9 only follow along
        const uint32_t ta0 = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_DS;
        // S^T row j (value column j) sits at row C + j of each K panel; this
        // thread writes the bf16 of S[i][j] at dk column i of every row.  A
        // warp's 32 two-byte stores of one row fill 4 distinct 16-byte chunks.
        const uint32_t colchunk = static_cast<uint32_t>((i & 63) >> 3);
        const uint32_t col_off = static_cast<uint32_t>((i >> 6) * KPANEL + C * 128 + (i & 7) * 2);
        int g = 0;
        bool stop = false;
        for (int r = 0; !stop; ++r) {
            const int idx = item_index(r, cta, G);
            if (idx >= p.n_items) break;
            const Item it = decode_item<kGeneral, KD>(p, idx);
            float S[DVS];
            if (it.init && init_t && own) {
                // column i of rows DVS vs .. DVS vs + DVS - 1 of the transposed block
                const float* src = it.init + (long)DVS * it.vs * KD + i;
#pragma unroll
                for (int j = 0; j < DVS; ++j) S[j] = src[j * KD];
            } else if (it.init && own) {
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
            for (int c0 = 0; c0 < it.len; c0 += C, ++g) {
                // publish bf16(S_{c-1})^T next to K_c, once the slot's previous product is done
                const int ks = g % K_SLOTS;
                if (!state_only) {
                    if (g >= K_SLOTS && !warp_wait(&k_empty[ks], ((g / K_SLOTS) - 1) & 1, abort, p.status)) { stop = true; break; }
                    if (own) {
                        uint8_t* base = sm + OFF_K + ks * TILE_K + col_off;
                        __nv_bfloat16* rowp[8];
#pragma unroll
                        for (int m = 0; m < 8; ++m)
                            rowp[m] = reinterpret_cast<__nv_bfloat16*>(base + ((colchunk ^ static_cast<uint32_t>(m)) << 4));
#pragma unroll
                        for (int j = 0; j < DVS; ++j) rowp[j & 7][j * 64] = __float2bfloat16_rn(S[j]);
                    }
                    fence_proxy_async_smem();
                    // the [P|O] product of this chunk also needs Q_c and K_c (thread A
                    // checks the O buffer it writes itself)
                    if (!warp_wait(&q_full[g % Q_SLOTS], (g / Q_SLOTS) & 1, abort, p.status)) { stop = true; break; }
                }
                if (phi != PHI_IDENTITY || !state_only) {
                    if (!warp_wait(&k_full[ks], (g / K_SLOTS) & 1, abort, p.status)) { stop = true; break; }
                }
                if (phi != PHI_IDENTITY) {
                    // phi(K_c), then phi(Q_c), in place, before the tensor cores read
                    // them; K first, so that K^T V can start while Q is mapped
#pragma unroll 1
                    for (int reg = 0; reg < (state_only ? 1 : 2); ++reg) {
                        phi_tile<NP>(reg == 0 ? smem_u32(sm + OFF_K + ks * TILE_K)
                                              : smem_u32(sm + OFF_Q + (g % Q_SLOTS) * TILE_Q),
                                     reg == 0 ? KPANEL : PANEL, i, phi);
                        if (reg == 0) {
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&kphi_full[ks]);
                        }
                    }
                }
                if (!state_only) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_full[ks]);
                }
                // absorb dS_c
                const int b = g & 1;
                if (!warp_wait(&ds_full[b], (g >> 1) & 1, abort, p.status)) { stop = true; break; }
                tc_fence_after();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[32];
                    tmem_ld32(ta0 + TM_PO_STRIDE * b + 32 * h2, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) S[32 * h2 + j] += __uint_as_float(v[j]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ds_empty[b]);
            }
            if (stop) break;
            if (p.s_out && it.write_state && own) {
                float4* dst = reinterpret_cast<float4*>(p.s_out + (it.state * KD + i) * p.dv + DVS * it.vs);
#pragma unroll
                for (int j = 0; j < DVS / 4; ++j)
                    dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            }
        }
    } else if (warp < 14) {
        if (!state_only) {
            // ------------------------------------------------------ output warps
            const int q4 = warp & 3;
            const int row = q4 * 32 + lane;
            uint8_t* stg = sm + OFF_OST + q4 * OST_WARP;  // this warp's 32 staging rows
            int g = 0;
            bool stop = false;
            for (int r = 0; !stop; ++r) {
                const int idx = item_index(r, cta, G);
                if (idx >= p.n_items) break;
                const Item it = decode_item<kGeneral, KD>(p, idx);
                const int nc = (it.len + C - 1) / C;
                for (int c = 0; c < nc; ++c, ++g) {
                    const int c0 = chunk_row(rev, c, nc);
                    const int b = g & 1;
                    if (!warp_wait(&o_full[b], (g >> 1) & 1, abort, p.status)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t ta = tbase + (static_cast<uint32_t>(q4 * 32) << 16) + TM_PO_STRIDE * b + TM_O_OFF;
                    uint32_t hp[32];
                    {
                        uint32_t v0[32], v1[32];
                        tmem_ld32(ta, v0);
                        tmem_ld32(ta + 32, v1);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            hp[e] = pack_bf16x2(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
                            hp[16 + e] = pack_bf16x2(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&o_empty[b]);
                    const int rows = it.len - c0;
                    if (q4 * 32 >= rows) {
                        // this warp's rows all lie past the end of the sequence
                    } else if (p.mode == 0 || q4 * 32 + 32 <= rows) {
                        // each warp stages its 32 rows and stores them with one TMA copy
                        // (a dense tensor clips rows past N itself)
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
                            if (p.mode == 0) tma_store_3d(&map_o, stg, DVS * it.vs, it.t0 + c0 + q4 * 32, it.c2);
                            else tma_store_3d(&map_o, stg, DVS * it.vs, it.c1, it.t0 + c0 + q4 * 32);
                            bulk_commit();
                        }
                    } else if (row < rows) {
                        // ragged tail of a packed sequence (the next rows belong to
                        // another sequence): plain row stores
                        uint4* dst = reinterpret_cast<uint4*>(
                            p.o + ((long)(it.t0 + c0 + row) * p.H + it.c1) * p.dv + DVS * it.vs);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            dst[ch] = make_uint4(hp[4 * ch], hp[4 * ch + 1], hp[4 * ch + 2], hp[4 * ch + 3]);
                    }
                }
            }
            if (lane == 0) bulk_wait<0>();
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA_A) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace lcl

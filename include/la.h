/*
 * la.h — C ABI of the B200 (sm_100a) causal linear attention library.
 *
 * The operation (page "MiniMax-M1で理解する：大規模言語モデルのコンテキスト長
 * 限界を突破する革新的アーキテクチャ" (zenn.dev), section "線形アテンションの
 * 数学的基礎"), with the feature map phi = identity, no decay, no normaliser and
 * no 1/sqrt(d) scale (the pages fix none of them):
 *
 *     S_t = S_{t-1} + k_t (x) v_t        (outer product; S is d_k x d_v, fp32)
 *     o_t = q_t S_t                      (q_t a row vector; inclusive of token t)
 *
 * computed in tiles as Lightning Attention (page "MiniMax: «Почему M2 в итоге
 * стала моделью с полным вниманием?» (конспект)" (ai.flicky.cc), section 1,
 * glossary entry "Lightning Attention"): for each chunk c of C tokens,
 *
 *     O_c = (Q_c K_c^T ⊙ M) V_c + Q_c S_{c-1},   S_c = S_{c-1} + K_c^T V_c
 *
 * where M keeps s <= t (diagonal included).  The running state is the
 * prefix-cache object of page "MiniMax: «Почему M2 …»", section 4
 * (prefix caching and state precision): it is exported in fp32 and can be
 * fed back to resume a sequence.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Ownership: the caller allocates and owns every buffer; the library never
 *    allocates device memory.  All pointers are DEVICE pointers unless noted.
 *  - Streams: work is enqueued on `stream` (NULL = the legacy default stream)
 *    and the call returns without waiting; errors found on the host come back
 *    as la_status, launch errors as LA_ERR_CUDA (see la_last_error()).
 *  - Alignment: every tensor pointer must be 16-byte aligned.
 *  - Aliasing: no input may alias an output, except the in-place state of
 *    la_decode_step.
 *  - Dimensions: d_k = d_v = d with d in {64, 128}.  bf16 inputs run on the
 *    tcgen05 tensor-core path; fp32 inputs run on a CUDA-core FFMA path.
 *    Anything else returns LA_ERR_UNSUPPORTED.
 *  - Output dtype equals the input dtype; states are always fp32.
 *  - Device-side waits are bounded; a wait that runs out records
 *    LA_ERR_TIMEOUT in a device status word read by la_device_status().
 */
#ifndef LA_H_
#define LA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative size, bad cu_seqlens ... */
    LA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (dtype, d, chunk)             */
    LA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed             */
    LA_ERR_TIMEOUT = 4       /* a bounded device-side wait ran out                      */
} la_status;

typedef enum { LA_BF16 = 0, LA_FP32 = 1 } la_dtype;

/* Storage format of a decode state (see la_decode_step_ex). */
typedef enum {
    LA_STATE_FP32 = 0,
    LA_STATE_BF16 = 1,
    LA_STATE_FP16 = 2,
    LA_STATE_FP8_E4M3 = 3, /* 8-bit, 3 mantissa bits, largest finite 448 (no infinities) */
    LA_STATE_FP8_E5M2 = 4  /* 8-bit, 2 mantissa bits, largest finite 57344 */
} la_state_dtype;

/*
 * Element-wise feature map phi on queries and keys.  Page "MiniMax-M1で理解す
 * る…", section "線形アテンションの数学的基礎", writes linear attention as
 * phi(Q) (phi(K)^T V) with a generic phi: S_t = S_{t-1} + phi(k_t) v_t^T,
 * o_t = phi(q_t) S_t.  LA_PHI_ELU1 is elu(x) + 1 (x + 1 for x > 0, exp(x)
 * otherwise), LA_PHI_RELU is max(x, 0).  phi is evaluated in fp32; on the bf16
 * tensor-core prefill path its result is rounded to bf16 before the products.
 * Every entry point without a phi argument uses the identity.
 */
typedef enum { LA_PHI_IDENTITY = 0, LA_PHI_ELU1 = 1, LA_PHI_RELU = 2 } la_phi;

/* Same type as cudaStream_t (an opaque CUDA stream handle). */
typedef struct CUstream_st* la_stream_t;

/* Static description of a status code. Never NULL. */
LA_API const char* la_status_string(la_status s);

/* Text of the last error raised on the calling host thread ("" if none). */
LA_API const char* la_last_error(void);

/* Library ABI version (major*10000 + minor*100 + patch). */
LA_API int la_version(void);

/*
 * Dense prefill.
 *   q, k : [B, H, N, d]  dtype `dt`, contiguous (d fastest)
 *   v, o : [B, H, N, d]  dtype `dt`; o is written
 *   s0   : [B, H, d, d]  fp32 state before token 1, or NULL for zero
 *   s_out: [B, H, d, d]  fp32 state after token N, or NULL (not written)
 *   chunk: tile length C (0 = library choice).  Tensor-core path (bf16):
 *          128; FFMA path: 32 or 64 (default 64), for fp32 and also for bf16
 *          when a bf16 call asks for 32 or 64.  C does not change the result
 *          beyond rounding; other values return LA_ERR_UNSUPPORTED.
 *   workspace/ws_bytes: scratch of at least la_prefill_workspace_size(...)
 *          bytes, 16-byte aligned (may be NULL when that size is 0).  The size
 *          is non-zero when B*H units are too few to fill the GPU and N is
 *          long: both paths (tensor cores and FFMA) then cut each sequence
 *          into segments of whole chunks (a segment split of the tiled form on page "MiniMax:
 *          «Почему M2 в итоге стала моделью с полным вниманием?»", section 1,
 *          glossary entry "Lightning Attention": the K^T V sums of the
 *          segments give every segment its starting state).  The workspace
 *          holds those fp32 states; with a NULL or smaller workspace the call
 *          runs unsplit and still returns the same result.  The environment
 *          variable LA_PREFILL_SEGMENTS=<n> forces n segments (1 = unsplit).
 * N = 0 writes s_out = s0 (or zero).  Returns LA_OK once enqueued.
 */
LA_API size_t la_prefill_workspace_size(int B, int H, int N, int dk, int dv, la_dtype dt);
/* The same for la_prefill_ex with feature map `phi`.  When the (batch, head)
 * units fill fewer than half of the SMs (two CTAs per head on the tensor-core
 * path), elu + 1 adds room for phi(q) and phi(k) (2 x B*H*N*dk bf16, each
 * rounded up to 256 bytes) after the segment states; given that room the call
 * maps q and k in one bandwidth-bound pass first, otherwise the prefill kernel
 * maps the tiles in shared memory (same results, slower there).  With more
 * units (one CTA per head) the kernel maps elu + 1 itself, a chunk ahead, and
 * nothing is added (environment variable LA_PHI_PREPASS=1 keeps the pass and
 * its room there too).  relu is always mapped in the kernel and adds nothing. */
LA_API size_t la_prefill_workspace_size_ex(int B, int H, int N, int dk, int dv, la_dtype dt, la_phi phi);
LA_API la_status la_prefill(const void* q, const void* k, const void* v, void* o,
                     const float* s0, float* s_out,
                     int B, int H, int N, int dk, int dv, la_dtype dt, int chunk,
                     void* workspace, size_t ws_bytes, la_stream_t stream);
/* la_prefill with a feature map phi on q and k (see la_phi). */
LA_API la_status la_prefill_ex(const void* q, const void* k, const void* v, void* o,
                        const float* s0, float* s_out,
                        int B, int H, int N, int dk, int dv, la_dtype dt, int chunk, la_phi phi,
                        void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * Ragged (packed) prefill with prefix resume.
 *   q, k : [T, H, d], v, o : [T, H, d]  dtype `dt` (token-major packing)
 *   cu_seqlens: int32 device [n_seq+1]; sequence n covers tokens
 *          [cu_seqlens[n], cu_seqlens[n+1]); cu_seqlens[0] = 0, non-decreasing,
 *          cu_seqlens[n_seq] <= T.  Contents are a precondition; they are
 *          checked (with a device-to-host copy and a stream sync) only when the
 *          environment variable LA_VALIDATE=1 is set.
 *   state_pool: fp32 [n_pool, H, d, d] or NULL; init_idx: int32 device [n_seq]
 *          or NULL.  Sequence n starts from state_pool[init_idx[n]] when
 *          init_idx[n] >= 0, else from zero.  (Prefix caching: a shared prompt
 *          prefix is absorbed once and its state resumed by many sequences.)
 *   s_out: fp32 [n_seq, H, d, d] final state per sequence, or NULL.
 *   A sequence of length 0 writes its initial state to s_out.
 *   workspace: at least la_prefill_varlen_workspace_size(...) bytes (device).
 */
LA_API size_t la_prefill_varlen_workspace_size(int n_seq, int T, int H, int dk, int dv, la_dtype dt);
/* The same for la_prefill_varlen_ex with feature map `phi`: with elu + 1 adds
 * room for phi(q) and phi(k) (2 x T*H*dk bf16) after the order array, on the
 * same terms as the dense call (n_seq x H units). */
LA_API size_t la_prefill_varlen_workspace_size_ex(int n_seq, int T, int H, int dk, int dv, la_dtype dt,
                                                  la_phi phi);
LA_API la_status la_prefill_varlen(const void* q, const void* k, const void* v, void* o,
                            const int32_t* cu_seqlens, int n_seq, int T,
                            const float* state_pool, int n_pool, const int32_t* init_idx,
                            float* s_out, int H, int dk, int dv, la_dtype dt, int chunk,
                            void* workspace, size_t ws_bytes, la_stream_t stream);
/* la_prefill_varlen with a feature map phi on q and k (see la_phi). */
LA_API la_status la_prefill_varlen_ex(const void* q, const void* k, const void* v, void* o,
                               const int32_t* cu_seqlens, int n_seq, int T,
                               const float* state_pool, int n_pool, const int32_t* init_idx,
                               float* s_out, int H, int dk, int dv, la_dtype dt, int chunk, la_phi phi,
                               void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * One decode step for B*H independent states (page "MiniMax: «Почему M2 …»",
 * section 4: a small state matrix read and written on every step).
 *   q, k : [B, H, d], v, o : [B, H, d]  dtype `dt`
 *   S    : [B, H, d, d] fp32, updated IN PLACE: S <- S + k (x) v, then o = q S.
 */
LA_API la_status la_decode_step(const void* q, const void* k, const void* v, void* o, float* S,
                         int B, int H, int dk, int dv, la_dtype dt, la_stream_t stream);

/*
 * la_decode_step with the state stored in a chosen format and a feature map phi, for the study of
 * low-precision state storage that page "MiniMax: «Почему M2 …»", section 4,
 * and page "ノーフリーランチ：MiniMax M2が高効率アテンション機構を解体",
 * infrastructure section, warn about (the state is rewritten at every token,
 * so its rounding errors accumulate).
 *   S: [B, H, d, d] in `sdt` (fp32, bf16, fp16, fp8 e4m3 or fp8 e5m2),
 *   updated IN PLACE.  Each element is updated in fp32 as RN_fp32(S + k_i v_j)
 *   (one fused multiply-add) and rounded to `sdt` to nearest even (the 8-bit
 *   formats saturate at their largest finite value); o = q S uses the stored,
 *   rounded state.  LA_STATE_FP32 is exactly la_decode_step.
 *   Low-precision storage needs bf16 q, k, v (LA_ERR_UNSUPPORTED otherwise).
 *   phi (see la_phi) is applied to q and k as they are loaded.
 */
LA_API la_status la_decode_step_ex(const void* q, const void* k, const void* v, void* o, void* S,
                                   int B, int H, int dk, int dv, la_dtype dt, la_state_dtype sdt, la_phi phi,
                                   la_stream_t stream);

/*
 * Speculative decoding over m draft tokens per sequence (1 <= m <= 16): the
 * state of a recurrent layer cannot be truncated after the fact (page
 * "MiniMax: «Почему M2 …»", section 4), so verifying drafts and advancing the
 * state are two calls.
 *
 * la_decode_verify: o_t = q_t S_t for every draft t = 1..m, where
 *   S_t = S + sum_{s<=t} k_s (x) v_s; S itself is only read.
 *   q, k : [B, H, m, d], v, o : [B, H, m, d]  dtype `dt`;  S : [B, H, d, d] fp32.
 * la_decode_commit: S <- S + sum_{t < accepted[b]} k_t (x) v_t, IN PLACE, for
 *   every head of sequence b; accepted: int32 device [B], values outside
 *   [0, m] are clamped (checked on the host under LA_VALIDATE=1).  The
 *   committed state is bit-identical to accepted[b] calls of la_decode_step.
 * Each call reads the state once (commit also writes it back).  phi (see
 * la_phi) is applied to q and k as they are loaded; use the same phi for both.
 */
LA_API la_status la_decode_verify(const void* q, const void* k, const void* v, void* o, const float* S,
                                  int B, int H, int m, int dk, int dv, la_dtype dt, la_phi phi,
                                  la_stream_t stream);
LA_API la_status la_decode_commit(const void* k, const void* v, float* S, const int32_t* accepted,
                                  int B, int H, int m, int dk, int dv, la_dtype dt, la_phi phi,
                                  la_stream_t stream);

/*
 * la_prefill on host-resident data: q, k, v, o (and s0, s_out) are HOST
 * buffers in the la_prefill layout; page-locked memory lets the copies run
 * asynchronously and overlap (pageable memory works, slower).  The (batch,
 * head) units are processed in groups of `group`: while group i is computed
 * on `stream`, group i + 1 is copied in and group i - 1 copied out on two
 * internal copy streams, so host-to-device and device-to-host traffic run at
 * the same time and the prefill itself hides under them.  Each group runs
 * the single-pass kernel (no segment split), so the results equal those of
 * la_prefill without a workspace bit for bit.
 *   workspace: device scratch of at least la_prefill_host_workspace_size(...)
 *   bytes (two staging buffers of `group` units each), 16-byte aligned.
 * Asynchronous like every other call: `stream` is ordered after the last
 * copy out, so synchronising it (or any later work on it) sees o and s_out.
 * Errors: LA_ERR_INVALID_ARG (null, negative, group <= 0, workspace too
 * small), LA_ERR_UNSUPPORTED (dims), LA_ERR_CUDA (copy or launch).
 */
LA_API size_t la_prefill_host_workspace_size(int B, int H, int N, int dk, int dv, la_dtype dt, int group);
LA_API la_status la_prefill_host(const void* q, const void* k, const void* v, void* o,
                                 const float* s0, float* s_out, int B, int H, int N, int dk, int dv,
                                 la_dtype dt, int group, void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * Gradients of la_prefill (dense layout, feature map identity): for a loss L
 * with dL/dO = dout and dL/dS_N = ds_n, the chain rule through
 * S_t = S_{t-1} + k_t (x) v_t, o_t = q_t S_t (page "MiniMax-M1で理解する…",
 * section "線形アテンションの数学的基礎") gives
 *   dq_t = dout_t S_t^T,   G_t = sum_{t' >= t} q_t'^T dout_t' + ds_n,
 *   dk_t = G_t v_t,   dv_t = G_t^T k_t,   ds0 = G_1,
 * computed chunk by chunk like the forward (masked products inside a chunk,
 * S carried forward for dq and G carried backward for dk, dv).
 *   q, k, dq, dk : [B, H, N, d_k];  v, dout, dv : [B, H, N, d_v]   dtype `dt`
 *   s0, ds_n     : fp32 [B, H, d_k, d_v] or NULL (zero);  ds0: fp32 or NULL.
 * bf16 (d = 128 or 64): three tensor-core passes of the prefill kernel
 * (dq = prefill(dout, v, k) from s0^T; dk = prefill(v, dout, q) from ds_n^T
 * and dv = prefill(k, q, dout) from ds_n, both with time reversed), with the
 * prefill's precision.  fp32: the same three passes on the FFMA
 * prefill kernel, fp32 arithmetic.  LA_BACKWARD_SIMT=1 in the environment
 * sends bf16 to the FFMA passes too (for testing).
 * d_k = d_v in {64, 128}.  All pointers 16-byte aligned; the caller owns every
 * buffer; no host synchronisation.  Errors: LA_ERR_INVALID_ARG (null, negative,
 * misaligned), LA_ERR_UNSUPPORTED (dims), LA_ERR_CUDA (launch).
 */
LA_API la_status la_prefill_backward(const void* q, const void* k, const void* v, const void* dout,
                                     const float* s0, const float* ds_n,
                                     void* dq, void* dk, void* dv, float* ds0,
                                     int B, int H, int N, int d_k, int d_v, la_dtype dt,
                                     la_stream_t stream);
/* la_prefill_backward with a workspace (device, 16-byte aligned) of at least
 * la_prefill_backward_workspace_size(...) bytes: when the (batch, head) units
 * fill less than half of the SMs, each pass (tensor-core or FFMA) cuts the
 * sequences into segments as la_prefill does (in reverse order the segment
 * starts are suffix sums).  With a smaller workspace (or none) the passes run
 * unsplit. */
LA_API size_t la_prefill_backward_workspace_size(int B, int H, int N, int d_k, int d_v, la_dtype dt);
LA_API la_status la_prefill_backward_ex(const void* q, const void* k, const void* v, const void* dout,
                                        const float* s0, const float* ds_n, void* dq, void* dk, void* dv, float* ds0,
                                        int B, int H, int N, int d_k, int d_v, la_dtype dt, void* workspace,
                                        size_t ws_bytes, la_stream_t stream);

/*
 * Reads the device status word of the current device (synchronizes the
 * device).  *out receives LA_OK or LA_ERR_TIMEOUT; clear != 0 resets it.
 */
LA_API la_status la_device_status(int* out, int clear);

/*
 * Self-test of device-side failure detection: launches one small kernel whose
 * bounded wait can never be satisfied; after `timeout_us` microseconds
 * (1 ..= 1,000,000) it gives up and records LA_ERR_TIMEOUT in the device status
 * word (read it with la_device_status).  The context stays usable.  This is
 * the same bounded-wait path every compute kernel takes when a wait runs out.
 */
LA_API la_status la_selftest_wait_timeout(int timeout_us, la_stream_t stream);

/*
 * Ragged prefill for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call; it exists for library users.
 * la_prefill_varlen needs a caller-provided device workspace (it sorts the
 * sequences by length on the GPU).  Some callers cannot obtain one at call
 * time: code embedded in a host framework that owns all device memory and
 * offers no allocator at that point, or latency-critical serving loops where
 * cudaMalloc/cudaFree (which may synchronize the device) are not allowed.
 * This entry point takes the same arguments minus the workspace and uses a
 * scratch array built into the library instead: a file-scope device array of
 * LA_NOALLOC_MAX_SEQS 32-bit entries that every GPU loading the library holds
 * until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 *  - n_seq > LA_NOALLOC_MAX_SEQS returns LA_ERR_INVALID_ARG (use
 *    la_prefill_varlen with a workspace for larger batches).
 *  - All calls on a device share the one scratch array and it keeps the last
 *    call's contents (every call rewrites the part it reads).  Calls whose
 *    work overlaps on the GPU (different streams, or different host threads,
 *    without ordering between them) race on it: order them on one stream.
 *  - The first call on each device performs a one-time set-up on the host
 *    (it looks up the device address of the scratch array for the current
 *    device); make that first call before any stream capture.  The set-up is
 *    redone when the device's context has changed since (after
 *    cudaDeviceReset, for instance).
 *  - Without a workspace the call never takes the segment split or the
 *    separate feature-map pass of la_prefill_varlen_ex (there is no room for
 *    their states), and the feature map is the identity.  Batches of a few
 *    long sequences therefore run unsplit, on fewer SMs and slower than
 *    la_prefill_varlen with the workspace it asks for; the results are the
 *    same within the parity tolerances.
 * Everything else (arguments, layouts, errors) is as for la_prefill_varlen.
 */
#define LA_NOALLOC_MAX_SEQS 4096
LA_API la_status la_prefill_varlen_noalloc(const void* q, const void* k, const void* v, void* o,
                                           const int32_t* cu_seqlens, int n_seq, int T,
                                           const float* state_pool, int n_pool, const int32_t* init_idx,
                                           float* s_out, int H, int dk, int dv, la_dtype dt, int chunk,
                                           la_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LA_H_ */

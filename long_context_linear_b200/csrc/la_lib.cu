// C ABI of the causal linear attention library (see include/la.h): argument
// validation, launch planning, TMA descriptor encoding and kernel launches.
// The library allocates no device memory; TMA descriptors are encoded per call
// on the host and passed by value as kernel parameters.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "la.h"
#include "sm100.cuh"
#include "prefill_tc.cuh"
#include "prefill_wide.cuh"
#include "prefill_simt.cuh"
#include "decode.cuh"
#include "varlen_order.cuh"
#include "selftest.cuh"
#include "seg_prefix.cuh"
#include "decode_multi.cuh"
#include "phi_map.cuh"

namespace lcl {

// Device status word: 0, or LA_ERR_TIMEOUT after a bounded wait ran out.
__device__ int g_status_word = 0;

// Scratch used by la_prefill_varlen_noalloc in place of a caller workspace:
// the longest-first sequence order of one packed batch.  One copy per device,
// alive for the whole process; host code must look up its device address
// (the array's name is only a host-side stand-in).
static __device__ __align__(256) int g_noalloc_order[LA_NOALLOC_MAX_SEQS];

namespace {

constexpr int kMaxDevices = 64;
thread_local char g_last_error[512] = "";

la_status fail(la_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

la_status cuda_fail(cudaError_t e, const char* what) {
    return fail(LA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
    int sms = 0;
    int* status = nullptr;       // device address of g_status_word
    bool attrs_set = false;
    unsigned long long ctx = 0;  // id of the context the set-up above was made in
    // copy streams of la_prefill_host, created on first use and kept for the
    // life of the process (like a library handle)
    cudaStream_t h2d = nullptr, d2h = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

template <typename T>
cudaError_t set_simt_attrs() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(simt::prefill_simt_kernel<T, 128, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  simt::smem_bytes<128, 64>())) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(simt::prefill_simt_kernel<T, 128, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  simt::smem_bytes<128, 32>())) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(simt::prefill_simt_kernel<T, 64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  simt::smem_bytes<64, 64>())) != cudaSuccess)
        return e;
    return cudaFuncSetAttribute(simt::prefill_simt_kernel<T, 64, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                simt::smem_bytes<64, 32>());
}

// Unique id of the calling thread's current CUDA context, 0 when none is
// current.  Device addresses and function attributes belong to a context: one
// destroyed and re-created (cudaDeviceReset) gets a new id, so per-device
// set-up cached under the old id is redone.
typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);
PFN_ctx_get_current g_ctx_current = nullptr;
PFN_ctx_get_id g_ctx_id = nullptr;
std::once_flag g_ctx_once;

unsigned long long current_ctx_id() {
    std::call_once(g_ctx_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<PFN_ctx_get_current>(fn);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_id = reinterpret_cast<PFN_ctx_get_id>(fn);
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!g_ctx_current || !g_ctx_id || g_ctx_current(&c) != CUDA_SUCCESS || !c || g_ctx_id(c, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

la_status device_info(DeviceInfo** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(LA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    // set-up made in another context (one that is gone, or none is current on
    // this thread yet): redo it
    if (d.attrs_set && current_ctx_id() != d.ctx) d.attrs_set = false;
    if (!d.attrs_set) {
        int major = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        if (major != 10) return fail(LA_ERR_UNSUPPORTED, "device %d is sm_%d x; the library is compiled for sm_100a", dev, major);
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        if ((e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_status_word)) != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress");
        const void* tc_kernels[6] = {reinterpret_cast<const void*>(tc::prefill_tc_kernel<false, false, 128>),
                                     reinterpret_cast<const void*>(tc::prefill_tc_kernel<true, false, 128>),
                                     reinterpret_cast<const void*>(tc::prefill_tc_kernel<true, true, 128>),
                                     reinterpret_cast<const void*>(tc::prefill_tc_kernel<false, false, 64>),
                                     reinterpret_cast<const void*>(tc::prefill_tc_kernel<true, false, 64>),
                                     reinterpret_cast<const void*>(tc::prefill_tc_kernel<true, true, 64>)};
        for (const void* kern : tc_kernels)
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES)) !=
                cudaSuccess)
                return cuda_fail(e, "cudaFuncSetAttribute(prefill_tc)");
        const void* wide_kernels[3] = {reinterpret_cast<const void*>(tcw::prefill_wide_kernel<false>),
                                       reinterpret_cast<const void*>(tcw::prefill_wide_kernel<true>),
                                       reinterpret_cast<const void*>(tcw::prefill_wide_kernel<true, true>)};
        for (const void* kern : wide_kernels)
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tcw::SMEM_BYTES)) !=
                cudaSuccess)
                return cuda_fail(e, "cudaFuncSetAttribute(prefill_wide)");
        if ((e = cudaFuncSetAttribute(dmulti::verify_tf32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      dmulti::vtf::SMEM_BYTES)) != cudaSuccess)
            return cuda_fail(e, "cudaFuncSetAttribute(verify_tf32)");
        if ((e = set_simt_attrs<float>()) != cudaSuccess || (e = set_simt_attrs<__nv_bfloat16>()) != cudaSuccess)
            return cuda_fail(e, "cudaFuncSetAttribute(prefill_simt)");
        const unsigned long long id = current_ctx_id();
        if (id != d.ctx) d.h2d = d.d2h = nullptr;  // copy streams of a context that is gone
        d.ctx = id;
        d.attrs_set = true;
    }
    *out = &d;
    return LA_OK;
}

la_status encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return fail(LA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    *out = g_encode;
    return LA_OK;
}

// 3-D bf16 tensor map with a 64-element (128-byte) inner box and 128B swizzle.
la_status make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                   uint64_t stride2_bytes, uint32_t b1, uint32_t b2) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    la_status s = encoder(&enc);
    if (s != LA_OK) return s;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {64, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return LA_OK;
}

// U fp32 d x d states, row-major and back to back, as a 3-D map {d, d, U} with
// boxes of 32 columns x d rows x 1 unit (128 bytes a row, 128-byte swizzle of
// 32-byte atoms: the MN-major tf32 operand layout).
la_status make_state_map(CUtensorMap* m, const float* S, uint64_t d, uint64_t U) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    la_status s = encoder(&enc);
    if (s != LA_OK) return s;
    cuuint64_t dims[3] = {d, d, U};
    cuuint64_t strides[2] = {d * 4, d * d * 4};
    cuuint32_t box[3] = {32, static_cast<cuuint32_t>(d), 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(S), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LA_ERR_CUDA, "cuTensorMapEncodeTiled (state) failed (%d)", (int)r);
    return LA_OK;
}

bool env_flag(const char* name) {
    const char* v = getenv(name);
    return v && v[0] == '1';
}

bool env_validate() { return env_flag("LA_VALIDATE"); }

la_status check_phi(la_phi phi) {
    if (phi != LA_PHI_IDENTITY && phi != LA_PHI_ELU1 && phi != LA_PHI_RELU)
        return fail(LA_ERR_INVALID_ARG, "unknown feature map %d", (int)phi);
    return LA_OK;
}

la_status check_dims(int dk, int dv, la_dtype dt) {
    if (dt != LA_BF16 && dt != LA_FP32) return fail(LA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    if (dk <= 0 || dv <= 0) return fail(LA_ERR_INVALID_ARG, "dk=%d dv=%d must be positive", dk, dv);
    if (dk != dv || (dk != 64 && dk != 128))
        return fail(LA_ERR_UNSUPPORTED, "only dk = dv in {64, 128} is supported (got %d, %d)", dk, dv);
    return LA_OK;
}

bool use_tensor_cores(int d, la_dtype dt) { return dt == LA_BF16 && (d == 128 || d == 64); }

constexpr int kSimtDefaultChunk = 64;

la_status check_chunk(int chunk, bool tcpath) {
    if (chunk == 0) return LA_OK;
    if (tcpath && chunk == tc::C) return LA_OK;
    if (!tcpath && (chunk == 32 || chunk == 64)) return LA_OK;
    return fail(LA_ERR_UNSUPPORTED,
                "chunk %d is not available: 0 (library choice), 128 (bf16 on the tensor cores), "
                "32 or 64 (FFMA kernel, bf16 or fp32)", chunk);
}

// The tensor-core kernels tile 128 tokens per chunk (one M = 128 tcgen05 tile
// of rows); a bf16 call that asks for 32- or 64-token chunks runs on the FFMA
// kernel, which has those tile lengths.  The result does not depend on the
// chunk length beyond rounding.
bool tensor_core_path(int d, la_dtype dt, int chunk) {
    return use_tensor_cores(d, dt) && (chunk == 0 || chunk == tc::C);
}

la_status after_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return LA_OK;
}

// The tensor-core prefill for p.dk (128 or 64): the lean instance unless an
// option needs the general one, which carries the feature-map code only when
// a feature map is applied in the kernel.
la_status launch_tc(int grid, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const CUtensorMap& mo, const tc::Params& p, cudaStream_t st, const char* what) {
    const bool phi = p.phi != LA_PHI_IDENTITY;
    const bool general =
        phi || p.reverse || p.state_only || p.init_transposed || (p.mode == 0 && p.n_seg > 1) || p.seg_off;
    auto go = [&](auto kern) { kern<<<grid, tc::NUM_THREADS, tc::SMEM_BYTES, st>>>(mq, mk, mv, mo, p); };
    if (p.dk == 64) {
        if (phi) go(tc::prefill_tc_kernel<true, true, 64>);
        else if (general) go(tc::prefill_tc_kernel<true, false, 64>);
        else go(tc::prefill_tc_kernel<false, false, 64>);
    } else {
        if (phi) go(tc::prefill_tc_kernel<true, true, 128>);
        else if (general) go(tc::prefill_tc_kernel<true, false, 128>);
        else go(tc::prefill_tc_kernel<false, false, 128>);
    }
    return after_launch(what);
}

// (unit, value slice) work items per unit of the tensor-core prefill
int tc_slices(int d) { return d / tc::DVS; }

// The full-width kernel (one CTA per head over all 128 value columns) once
// the batch's heads alone fill the GPU, i.e. when the (head, 64-column value
// slice) items of the value-split kernel would need more than one wave:
// it forms Q K^T once per head and needs no more CTAs than there are heads.
// Below that the value split (and, when still under-filled, the segment
// split) keeps every SM busy.  LA_PREFILL_WIDE=1 / 0 forces it on / off at
// d = 128 (on: whole sequences, no segment split).
bool use_wide(long units, int d, const DeviceInfo* di) {
    if (d != 128) return false;
    if (const char* e = getenv("LA_PREFILL_WIDE")) {
        if (e[0] == '1') return true;
        if (e[0] == '0') return false;
    }
    return units * tc_slices(d) > di->sms;
}

// The full-width kernel: the lean instance unless the feature map, the
// reverse order or a transposed initial state asks for the general one.
la_status launch_wide(int grid, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const CUtensorMap& mo, const tc::Params& p, cudaStream_t st, const char* what) {
    const bool general = p.phi != LA_PHI_IDENTITY || p.reverse || p.init_transposed;
    if (p.phi == LA_PHI_ELU1)
        tcw::prefill_wide_kernel<true, true><<<grid, tcw::NUM_THREADS, tcw::SMEM_BYTES, st>>>(mq, mk, mv, mo, p);
    else if (general)
        tcw::prefill_wide_kernel<true><<<grid, tcw::NUM_THREADS, tcw::SMEM_BYTES, st>>>(mq, mk, mv, mo, p);
    else
        tcw::prefill_wide_kernel<false><<<grid, tcw::NUM_THREADS, tcw::SMEM_BYTES, st>>>(mq, mk, mv, mo, p);
    return after_launch(what);
}

template <typename T, int D>
void launch_simt_d(int cs, int grid, const void* q, const void* k, const void* v, void* o, const simt::Params& sp,
                   cudaStream_t st) {
    if (cs == 32)
        simt::prefill_simt_kernel<T, D, 32><<<grid, simt::NUM_THREADS, simt::smem_bytes<D, 32>(), st>>>(
            (const T*)q, (const T*)k, (const T*)v, (T*)o, sp);
    else
        simt::prefill_simt_kernel<T, D, 64><<<grid, simt::NUM_THREADS, simt::smem_bytes<D, 64>(), st>>>(
            (const T*)q, (const T*)k, (const T*)v, (T*)o, sp);
}

template <typename T>
la_status launch_simt(int d, int chunk, int grid, const void* q, const void* k, const void* v, void* o,
                      const simt::Params& sp, cudaStream_t st) {
    if (grid == 0) return LA_OK;
    const int cs = chunk ? chunk : kSimtDefaultChunk;
    if (d == 128) launch_simt_d<T, 128>(cs, grid, q, k, v, o, sp, st);
    else launch_simt_d<T, 64>(cs, grid, q, k, v, o, sp, st);
    return after_launch("prefill_simt launch");
}

}  // namespace
}  // namespace lcl

namespace lcl {
namespace {
template <typename T, typename SS>
void launch_decode(int dk, int grid, const void* q, const void* k, const void* v, void* o, void* S, int phi,
                   cudaStream_t st) {
    if (dk == 128)
        dec::decode_step_kernel<T, SS, 128><<<grid, dec::decode_threads<SS>(), 0, st>>>(
            (const T*)q, (const T*)k, (const T*)v, (T*)o, (SS*)S, phi);
    else
        dec::decode_step_kernel<T, SS, 64><<<grid, dec::decode_threads<SS>(), 0, st>>>(
            (const T*)q, (const T*)k, (const T*)v, (T*)o, (SS*)S, phi);
}
}  // namespace
}  // namespace lcl

namespace lcl {
namespace {
// verify for m drafts: the instance for the smallest draft capacity MB >= m
template <typename T, int D>
void launch_verify_d(int m, int grid, const T* q, const T* k, const T* v, T* o, const float* S, int phi,
                     cudaStream_t st) {
    // D / 2 threads per group of drafts: one group up to 12 drafts, two of 8 beyond
    if (m <= 4) dmulti::verify_kernel<T, D, 4, 4><<<grid, D / 2, 0, st>>>(q, k, v, o, S, m, phi);
    else if (m <= 8) dmulti::verify_kernel<T, D, 8, 8><<<grid, D / 2, 0, st>>>(q, k, v, o, S, m, phi);
    else if (m <= 12) dmulti::verify_kernel<T, D, 12, 12><<<grid, D / 2, 0, st>>>(q, k, v, o, S, m, phi);
    else dmulti::verify_kernel<T, D, 16, 8><<<grid, D, 0, st>>>(q, k, v, o, S, m, phi);
}
template <typename T>
void launch_verify(int dk, int m, int grid, const void* q, const void* k, const void* v, void* o, const float* S,
                   int phi, cudaStream_t st) {
    if (dk == 128) launch_verify_d<T, 128>(m, grid, (const T*)q, (const T*)k, (const T*)v, (T*)o, S, phi, st);
    else launch_verify_d<T, 64>(m, grid, (const T*)q, (const T*)k, (const T*)v, (T*)o, S, phi, st);
}

template <typename T, int D>
void launch_commit_d(int m, int grid, const T* k, const T* v, float* S, const int32_t* accepted, int H, int phi,
                     cudaStream_t st) {
    dmulti::commit_kernel<T, D><<<grid, dmulti::NUM_THREADS, 0, st>>>(k, v, S, accepted, H, m, phi);
}

template <typename T>
void launch_commit(int dk, int m, int grid, const void* k, const void* v, float* S, const int32_t* accepted, int H,
                   int phi, cudaStream_t st) {
    if (dk == 128) launch_commit_d<T, 128>(m, grid, (const T*)k, (const T*)v, S, accepted, H, phi, st);
    else launch_commit_d<T, 64>(m, grid, (const T*)k, (const T*)v, S, accepted, H, phi, st);
}

}  // namespace
}  // namespace lcl

using namespace lcl;

extern "C" {

const char* la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: unsupported configuration";
        case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA error";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: a device-side wait timed out";
    }
    return "unknown la_status";
}

const char* la_last_error(void) { return g_last_error; }

int la_version(void) { return 300; }  // 0.3.0

namespace {

// Segment split of a dense prefill: when the items (one per unit and value
// slice: d / 64 slices on the tensor cores, one on the FFMA path) fill less
// than half of the SMs, each unit's sequence is cut into segments of whole
// 128-token chunks (at least kMinSegChunks) so that about one item per SM
// remains.  LA_PREFILL_SEGMENTS=<n> overrides the count (1 = no split).
constexpr int kMinSegChunks = 8;

// On the FFMA path a chunk is compute-heavy (about 4 C d^2 FMAs on one SM), so
// there a segment of a single chunk already pays for its share of the
// state-only pass once the units leave SMs idle (fp32, B=1, H=2, N=256, d=64,
// chunk 64: 44 us a call unsplit, on 2 SMs).
constexpr int kMinSegChunksSimt = 1;
constexpr int kSimtSmallestChunk = 32;

// Segments are whole chunks of `unit` tokens (the tensor-core tile, or the
// FFMA kernel's chunk), at least min_chunks of them.
int plan_segments(long U, int N, int slices, int sms, int* seg_len, int unit = tc::C,
                  int min_chunks = kMinSegChunks) {
    const int nch = (N + unit - 1) / unit;
    *seg_len = nch * unit;
    if (N <= 0) return 1;
    int P;
    if (const char* e = getenv("LA_PREFILL_SEGMENTS")) {
        P = atoi(e);
    } else {
        const long items = U * slices;
        P = items * 2 > sms ? 1 : (int)(sms / items);
        P = std::min(P, nch / min_chunks);
    }
    P = std::max(1, std::min(P, nch));
    const int cps = (nch + P - 1) / P;  // chunks per segment
    *seg_len = cps * unit;
    return (nch + cps - 1) / cps;
}

// The most segments an FFMA-path call may plan (its chunk is not known to the
// workspace queries; the smallest chunk gives the most segments).
int plan_segments_simt_max(long U, int N, int sms) {
    int seg_len;
    return plan_segments(U, N, 1, sms, &seg_len, kSimtSmallestChunk, kMinSegChunksSimt);
}

size_t segment_workspace_bytes(long U, int P, int dk, int dv) {
    if (P <= 1) return 0;
    return (size_t)U * (size_t)(2 * P - 1) * (size_t)dk * (size_t)dv * sizeof(float);
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Scratch for phi(q) and phi(k) (bf16, `rows` rows of d) on the tensor-core
// path, for elu + 1 only: its exponentials cost the prefill kernel more than a
// separate bandwidth-bound pass over q and k, while relu (a packed max per
// pair of values) is cheaper mapped on the tiles inside the kernel.
size_t phi_workspace_bytes(long rows, int d, la_phi phi) {
    if (phi != LA_PHI_ELU1 || rows <= 0) return 0;
    return 2 * round256((size_t)rows * (size_t)d * 2);
}

// elu + 1 through the pre-pass only on the value-split kernel, whose two
// CTAs of a head would both map the tiles; the full-width kernel maps them
// once per head, a chunk ahead (B=4, H=32, N=8K: 0.31-0.33 ms mapped in the
// kernel against 0.36 ms with the pre-pass).  LA_PHI_PREPASS=1 keeps the
// pre-pass on the full-width kernel too (the two routes are tested equal).
bool phi_prepass_wanted(bool wide) { return !wide || env_flag("LA_PHI_PREPASS"); }

// phi over q and k (each `elems` bf16) into the two halves of `scratch`; on
// success q and k are redirected to the mapped copies.
la_status phi_prepass(const void** q, const void** k, void* scratch, long elems, la_phi phi, DeviceInfo* di,
                      cudaStream_t st) {
    const long n = elems / 8;  // elems is a multiple of d = 128
    uint8_t* yq = reinterpret_cast<uint8_t*>(scratch);
    uint8_t* yk = yq + round256((size_t)elems * 2);
    const long per_block = (long)phimap::NUM_THREADS * phimap::VPT;
    const int blocks = (int)std::min<long>((2 * n + per_block - 1) / per_block, 8L * di->sms);
    phimap::phi_map_kernel<<<blocks, phimap::NUM_THREADS, 0, st>>>(
        reinterpret_cast<const uint4*>(*q), reinterpret_cast<const uint4*>(*k), reinterpret_cast<uint4*>(yq),
        reinterpret_cast<uint4*>(yk), n, (int)phi);
    la_status s = after_launch("phi pre-pass launch");
    if (s != LA_OK) return s;
    *q = yq;
    *k = yk;
    return LA_OK;
}

}  // namespace

// The FFMA prefill over dense units.  When the units fill less than half of
// the SMs and the workspace holds segment_workspace_bytes(U, P, d, d), each
// unit's sequence is cut into P segments: a state-only pass sums K^T V per
// segment (all but the last one visited), seg_prefix_kernel forms each
// segment's starting state from them and `init`, and the main pass runs all
// segments at once.  Otherwise one CTA runs each unit whole.
la_status simt_dense(const void* q, const void* k, const void* v, void* o, const float* init, bool init_t,
                     float* s_out, bool reverse, la_phi phi, long U, int N, int d, la_dtype dt, int chunk,
                     DeviceInfo* di, void* ws, size_t ws_bytes, cudaStream_t st) {
    simt::Params sp{};
    sp.mode = 0;
    sp.N = N;
    sp.s0 = init;
    sp.s_out = s_out;
    sp.phi = phi;
    sp.reverse = reverse ? 1 : 0;
    sp.init_transposed = init_t ? 1 : 0;
    auto go = [&](const simt::Params& x, long grid) {
        return dt == LA_FP32 ? launch_simt<float>(d, chunk, (int)grid, q, k, v, o, x, st)
                             : launch_simt<__nv_bfloat16>(d, chunk, (int)grid, q, k, v, o, x, st);
    };
    int seg_len;
    int P = plan_segments(U, N, 1, di->sms, &seg_len, chunk ? chunk : kSimtDefaultChunk, kMinSegChunksSimt);
    if (P > 1 && (!ws || ws_bytes < segment_workspace_bytes(U, P, d, d) || !aligned16(ws) || U * P > (1L << 30)))
        P = 1;
    if (P <= 1) return go(sp, U);
    float* sums = reinterpret_cast<float*>(ws);
    float* starts = sums + (size_t)U * (P - 1) * d * d;
    simt::Params p1 = sp;
    p1.n_seg = P - 1;
    p1.seg_len = seg_len;
    p1.seg_base = reverse ? 1 : 0;  // the segments whose sums reach another segment's start
    p1.s0 = nullptr;
    p1.init_transposed = 0;
    p1.s_out = sums;
    p1.s_out_per_seg = 1;
    p1.state_only = 1;
    la_status s;
    if ((s = go(p1, U * (P - 1))) != LA_OK) return s;
    const long threads = U * (long)(d * d / 4);
    const int blocks = (int)std::min<long>((threads + segp::NUM_THREADS - 1) / segp::NUM_THREADS, 4L * di->sms);
    segp::seg_prefix_kernel<<<blocks, segp::NUM_THREADS, 0, st>>>(sums, init, starts, U, P, d * d, reverse ? 1 : 0,
                                                                 init_t ? 1 : 0, d);
    if ((s = after_launch("segment prefix launch")) != LA_OK) return s;
    sp.n_seg = P;
    sp.seg_len = seg_len;
    sp.seg_init = starts;
    return go(sp, U * P);
}

size_t la_prefill_workspace_size(int B, int H, int N, int dk, int dv, la_dtype dt) {
    return la_prefill_workspace_size_ex(B, H, N, dk, dv, dt, LA_PHI_IDENTITY);
}

size_t la_prefill_workspace_size_ex(int B, int H, int N, int dk, int dv, la_dtype dt, la_phi phi) {
    if (B <= 0 || H <= 0 || N <= 0 || dk != dv || (dk != 64 && dk != 128)) return 0;
    const bool tc = use_tensor_cores(dk, dt);
    const long U = (long)B * H;
    DeviceInfo* di;
    if (device_info(&di) != LA_OK) return tc ? phi_workspace_bytes(U * N, dk, phi) : 0;
    const size_t ph = tc && phi_prepass_wanted(use_wide(U, dk, di)) ? phi_workspace_bytes(U * N, dk, phi) : 0;
    int seg_len;
    // (a bf16 call with 32- or 64-token chunks runs on the FFMA path; sized for
    // the tensor-core plan, its workspace may leave it unsplit)
    const size_t seg = tc ? segment_workspace_bytes(U, plan_segments(U, N, tc_slices(dk), di->sms, &seg_len), dk, dv)
                          : segment_workspace_bytes(U, plan_segments_simt_max(U, N, di->sms), dk, dv);
    return ph ? round256(seg) + ph : seg;
}

la_status la_prefill(const void* q, const void* k, const void* v, void* o, const float* s0, float* s_out, int B,
                     int H, int N, int dk, int dv, la_dtype dt, int chunk, void* workspace, size_t ws_bytes,
                     la_stream_t stream) {
    return la_prefill_ex(q, k, v, o, s0, s_out, B, H, N, dk, dv, dt, chunk, LA_PHI_IDENTITY, workspace, ws_bytes,
                         stream);
}

la_status la_prefill_ex(const void* q, const void* k, const void* v, void* o, const float* s0, float* s_out, int B,
                        int H, int N, int dk, int dv, la_dtype dt, int chunk, la_phi phi, void* workspace,
                        size_t ws_bytes, la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(dk, dv, dt);
    if (s != LA_OK) return s;
    if ((s = check_phi(phi)) != LA_OK) return s;
    if (B < 0 || H < 0 || N < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d N=%d", B, H, N);
    const long U = (long)B * H;
    if (U > (1L << 30) || (long)N * U > (1L << 40)) return fail(LA_ERR_INVALID_ARG, "problem too large");
    if (U == 0) return LA_OK;
    if (N > 0 && (!q || !k || !v || !o)) return fail(LA_ERR_INVALID_ARG, "q, k, v, o must be non-null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(s0) || !aligned16(s_out))
        return fail(LA_ERR_INVALID_ARG, "all pointers must be 16-byte aligned");
    const bool tcpath = tensor_core_path(dk, dt, chunk);
    if ((s = check_chunk(chunk, tcpath)) != LA_OK) return s;
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    if (!tcpath)
        return simt_dense(q, k, v, o, s0, false, s_out, false, phi, U, N, dk, dt, chunk, di, workspace, ws_bytes, st);

    const int nvs = tc_slices(dv);
    tc::Params p{};
    p.mode = 0;
    p.dk = dk;
    p.n_items = (int)(U * nvs);
    p.H = H;
    p.N = N;
    p.dv = dv;
    p.s0 = s0;
    p.s_out = s_out;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.status = di->status;
    p.n_seg = 1;
    p.phi = phi;
    if (N == 0 && !s_out) return LA_OK;
    const bool wide = use_wide(U, dk, di);
    int seg_len;
    int P = wide ? 1 : plan_segments(U, N, tc_slices(dk), di->sms, &seg_len);
    p.seg_len = seg_len;
    const size_t ws_need = segment_workspace_bytes(U, P, dk, dv);
    if (wide || (P > 1 && (!workspace || ws_bytes < ws_need || !aligned16(workspace) ||
                           (long)U * P * nvs > (1L << 30)))) {
        P = 1;  // no room for the segment states: one pass over whole sequences
        p.seg_len = ((N + tc::C - 1) / tc::C) * tc::C;
    }
    // phi(q), phi(k) mapped up front when the workspace has room behind the
    // segment states; otherwise the kernel maps the tiles in shared memory
    const size_t off_phi = P > 1 ? round256(ws_need) : 0;
    const size_t ws_phi = phi_prepass_wanted(wide) ? phi_workspace_bytes(U * N, dk, phi) : 0;
    if (ws_phi && workspace && aligned16(workspace) && ws_bytes >= off_phi + ws_phi) {
        if ((s = phi_prepass(&q, &k, reinterpret_cast<uint8_t*>(workspace) + off_phi, U * N * dk, phi, di, st)) !=
            LA_OK)
            return s;
        p.phi = LA_PHI_IDENTITY;
    }
    // With N = 0 no tile is ever copied; the maps then only need a valid base.
    const void* bq = N > 0 ? q : s_out;
    const void* bk = N > 0 ? k : s_out;
    const void* bv = N > 0 ? v : s_out;
    const void* bo = N > 0 ? o : s_out;
    CUtensorMap mq, mk, mv, mo;
    const uint64_t row = (uint64_t)dk * 2;
    const uint64_t Nm = N > 0 ? (uint64_t)N : 1;
    const uint64_t unit = Nm * row;
    if ((s = make_map(&mq, bq, dk, Nm, U, row, unit, tc::C, 1)) != LA_OK) return s;
    if ((s = make_map(&mk, bk, dk, Nm, U, row, unit, tc::C, 1)) != LA_OK) return s;
    if ((s = make_map(&mv, bv, dv, Nm, U, row, unit, tc::C, 1)) != LA_OK) return s;
    if ((s = make_map(&mo, bo, dv, Nm, U, row, unit, 32, 1)) != LA_OK) return s;
    if (P > 1) {
        // segment split: (1) the K^T V sum of every segment but the last,
        // (2) the state before every segment, (3) all segments from those states
        float* seg_sums = reinterpret_cast<float*>(workspace);
        float* starts = seg_sums + (size_t)U * (P - 1) * dk * dv;
        tc::Params p1 = p;
        p1.n_seg = P - 1;
        p1.n_items = (int)(U * (P - 1) * nvs);
        p1.s0 = nullptr;
        p1.s_out = seg_sums;
        p1.s_out_per_seg = 1;
        p1.state_only = 1;
        if ((s = launch_tc(std::min(p1.n_items, di->sms), mq, mk, mv, mo, p1, st, "prefill_tc (segment sums) launch")) !=
            LA_OK)
            return s;
        const long threads = U * (long)(dk * dv / 4);
        const int blocks = (int)std::min<long>((threads + segp::NUM_THREADS - 1) / segp::NUM_THREADS, 4L * di->sms);
        segp::seg_prefix_kernel<<<blocks, segp::NUM_THREADS, 0, st>>>(seg_sums, s0, starts, U, P, dk * dv, 0, 0, dk);
        if ((s = after_launch("segment prefix launch")) != LA_OK) return s;
        p.n_seg = P;
        p.n_items = (int)(U * P * nvs);
        p.seg_init = starts;
    }
    if (wide) {
        p.n_items = (int)U;
        return launch_wide(std::min(p.n_items, di->sms), mq, mk, mv, mo, p, st, "prefill_wide launch");
    }
    const int grid = std::min(p.n_items, di->sms);
    return launch_tc(grid, mq, mk, mv, mo, p, st, "prefill_tc launch");
}

namespace {
size_t varlen_order_bytes(int n_seq) { return n_seq > 0 ? round256((size_t)n_seq * sizeof(int)) : 0; }

// Segment plan of a packed batch whose (sequence, head, value slice) items
// fill less than half of the SMs (`slices` per sequence and head: d / 64 on
// the tensor cores, 1 on the FFMA path): the most segments the batch may be
// cut into (about one item per SM), or 0 for no split, and the shortest
// segment (*min_seg tokens).  The host knows only the total token count T;
// the device picks the segment length from the real lengths
// (vorder::seg_plan_kernel).  With segments of at least min_seg tokens the
// batch never has more than T / min_seg + n_seq of them, which bounds the
// plan too.  LA_PREFILL_SEGMENTS = P allows P segments per sequence on
// average, of at least one chunk (1: no split).
long plan_varlen_segments(int n_seq, int T, int H, int slices, int sms, int* min_seg) {
    *min_seg = kMinSegChunks * tc::C;
    if (n_seq <= 0 || T <= 0 || H <= 0) return 0;
    long S;
    if (const char* e = getenv("LA_PREFILL_SEGMENTS")) {
        const long P = atol(e);
        if (P <= 1) return 0;
        *min_seg = tc::C;
        S = P * n_seq;
    } else {
        const long per_seq_items = (long)H * slices;
        if ((long)n_seq * per_seq_items * 2 > sms) return 0;
        S = sms / per_seq_items;  // segments that keep every item in one wave
        if ((long)T < 2L * *min_seg) return 0;
    }
    S = std::min(S, (long)T / *min_seg + n_seq);
    return S > n_seq ? S : 0;
}

// Bytes of the segment area for at most max_segs segments: the two offset
// arrays, the chosen segment length, the sums of all segments but each
// sequence's last (at most max_segs - n_seq) and the segment starts.
size_t varlen_segment_bytes(int n_seq, long max_segs, int H, int d) {
    const size_t state = (size_t)H * d * d * sizeof(float);
    return 2 * round256((size_t)(n_seq + 1) * sizeof(int)) + 256 + (size_t)(2 * max_segs - n_seq) * state;
}
}  // namespace

size_t la_prefill_varlen_workspace_size(int n_seq, int T, int H, int dk, int dv, la_dtype dt) {
    return la_prefill_varlen_workspace_size_ex(n_seq, T, H, dk, dv, dt, LA_PHI_IDENTITY);
}

size_t la_prefill_varlen_workspace_size_ex(int n_seq, int T, int H, int dk, int dv, la_dtype dt, la_phi phi) {
    const size_t base = varlen_order_bytes(n_seq);
    if (!base || T <= 0 || H <= 0 || dk != dv || (dk != 64 && dk != 128)) return base;
    const bool tc = use_tensor_cores(dk, dt);
    DeviceInfo* di;
    if (device_info(&di) != LA_OK) return base + (tc ? phi_workspace_bytes((long)T * H, dk, phi) : 0);
    size_t total = base + (tc && phi_prepass_wanted(use_wide((long)n_seq * H, dk, di))
                               ? phi_workspace_bytes((long)T * H, dk, phi)
                               : 0);
    int min_seg;
    const long max_segs = plan_varlen_segments(n_seq, T, H, tc ? tc_slices(dk) : 1, di->sms, &min_seg);
    if (max_segs) total += varlen_segment_bytes(n_seq, max_segs, H, dk);
    return total;
}

la_status la_prefill_varlen(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                            int n_seq, int T, const float* state_pool, int n_pool, const int32_t* init_idx,
                            float* s_out, int H, int dk, int dv, la_dtype dt, int chunk, void* workspace,
                            size_t ws_bytes, la_stream_t stream) {
    return la_prefill_varlen_ex(q, k, v, o, cu_seqlens, n_seq, T, state_pool, n_pool, init_idx, s_out, H, dk, dv, dt,
                                chunk, LA_PHI_IDENTITY, workspace, ws_bytes, stream);
}

la_status la_prefill_varlen_ex(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                               int n_seq, int T, const float* state_pool, int n_pool, const int32_t* init_idx,
                               float* s_out, int H, int dk, int dv, la_dtype dt, int chunk, la_phi phi,
                               void* workspace, size_t ws_bytes, la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(dk, dv, dt);
    if (s != LA_OK) return s;
    if ((s = check_phi(phi)) != LA_OK) return s;
    if (n_seq < 0 || T < 0 || H < 0 || n_pool < 0)
        return fail(LA_ERR_INVALID_ARG, "negative size n_seq=%d T=%d H=%d n_pool=%d", n_seq, T, H, n_pool);
    if (n_seq == 0 || H == 0) return LA_OK;
    if (!cu_seqlens) return fail(LA_ERR_INVALID_ARG, "cu_seqlens must be non-null");
    if (T > 0 && (!q || !k || !v || !o)) return fail(LA_ERR_INVALID_ARG, "q, k, v, o must be non-null");
    if (init_idx && (!state_pool || n_pool == 0))
        return fail(LA_ERR_INVALID_ARG, "init_idx given without a state pool");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state_pool) ||
        !aligned16(s_out) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
        (reinterpret_cast<uintptr_t>(init_idx) & 3u))
        return fail(LA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned, index arrays 4-byte aligned");
    if ((long)T * H > (1L << 40) || (long)n_seq * H > (1L << 30)) return fail(LA_ERR_INVALID_ARG, "problem too large");
    const bool tcpath = tensor_core_path(dk, dt, chunk);
    if ((s = check_chunk(chunk, tcpath)) != LA_OK) return s;
    const size_t need = varlen_order_bytes(n_seq);
    if (tcpath && (ws_bytes < need || !workspace || !aligned16(workspace)))
        return fail(LA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu", need, ws_bytes);
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    if (env_validate()) {
        std::vector<int32_t> cu(n_seq + 1), idx;
        cudaError_t e = cudaMemcpyAsync(cu.data(), cu_seqlens, sizeof(int32_t) * (n_seq + 1), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess && init_idx) {
            idx.resize(n_seq);
            e = cudaMemcpyAsync(idx.data(), init_idx, sizeof(int32_t) * n_seq, cudaMemcpyDeviceToHost, st);
        }
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "LA_VALIDATE copy of cu_seqlens");
        if (cu[0] != 0) return fail(LA_ERR_INVALID_ARG, "cu_seqlens[0] = %d, expected 0", cu[0]);
        for (int n = 0; n < n_seq; ++n)
            if (cu[n + 1] < cu[n]) return fail(LA_ERR_INVALID_ARG, "cu_seqlens decreases at %d", n);
        if (cu[n_seq] > T) return fail(LA_ERR_INVALID_ARG, "cu_seqlens[n_seq] = %d exceeds T = %d", cu[n_seq], T);
        for (size_t n = 0; n < idx.size(); ++n)
            if (idx[n] < -1 || idx[n] >= n_pool)
                return fail(LA_ERR_INVALID_ARG, "init_idx[%zu] = %d outside [-1, %d)", n, idx[n], n_pool);
    }

    if (!tcpath) {
        simt::Params sp{};
        sp.mode = 1; sp.H = H; sp.cu_seqlens = cu_seqlens; sp.pool = state_pool; sp.init_idx = init_idx;
        sp.s_out = s_out; sp.phi = phi;
        auto go = [&](const simt::Params& x, long grid) {
            return dt == LA_FP32 ? launch_simt<float>(dk, chunk, (int)grid, q, k, v, o, x, st)
                                 : launch_simt<__nv_bfloat16>(dk, chunk, (int)grid, q, k, v, o, x, st);
        };
        // the segment split as on the tensor cores (one item per sequence and
        // head), when the workspace has room for the order and the segment area
        int min_seg;
        const long max_segs = plan_varlen_segments(n_seq, T, H, 1, di->sms, &min_seg), max_nl = max_segs - n_seq;
        if (!max_segs || !workspace || !aligned16(workspace) || max_segs * H > (1L << 30) ||
            ws_bytes < need + varlen_segment_bytes(n_seq, max_segs, H, dk))
            return go(sp, (long)n_seq * H);
        int* order = reinterpret_cast<int*>(workspace);
        vorder::order_kernel<<<1, vorder::NUM_THREADS, 0, st>>>(cu_seqlens, n_seq, order);
        if ((s = after_launch("varlen order launch")) != LA_OK) return s;
        uint8_t* w = reinterpret_cast<uint8_t*>(workspace) + need;
        const size_t ints = round256((size_t)(n_seq + 1) * sizeof(int));
        int* seg_off = reinterpret_cast<int*>(w);
        int* seg_off_nl = reinterpret_cast<int*>(w + ints);
        int* seg_len = reinterpret_cast<int*>(w + 2 * ints);
        float* sums = reinterpret_cast<float*>(w + 2 * ints + 256);
        float* starts = sums + (size_t)max_nl * H * dk * dv;
        vorder::seg_plan_kernel<<<1, 32, 0, st>>>(cu_seqlens, order, n_seq, max_segs, min_seg, tc::C, seg_len, seg_off,
                                                  seg_off_nl);
        if ((s = after_launch("varlen segment plan launch")) != LA_OK) return s;
        sp.order = order;
        sp.seg_off = seg_off;
        sp.seg_off_nl = seg_off_nl;
        sp.n_seq = n_seq;
        sp.seg_len_dev = seg_len;
        if (max_nl > 0) {
            simt::Params p1 = sp;
            p1.state_only = 1;
            p1.s_out = sums;
            p1.pool = nullptr;
            p1.init_idx = nullptr;
            if ((s = go(p1, max_nl * H)) != LA_OK) return s;
        }
        const long threads = (long)n_seq * H * (dk * dv / 4);
        const int blocks = (int)std::min<long>((threads + segp::NUM_THREADS - 1) / segp::NUM_THREADS, 4L * di->sms);
        segp::seg_prefix_varlen_kernel<<<blocks, segp::NUM_THREADS, 0, st>>>(sums, state_pool, init_idx, order, seg_off,
                                                                            seg_off_nl, starts, n_seq, H, dk * dv);
        if ((s = after_launch("varlen segment prefix launch")) != LA_OK) return s;
        sp.seg_init = starts;
        return go(sp, max_segs * H);
    }

    int* order = reinterpret_cast<int*>(workspace);
    vorder::order_kernel<<<1, vorder::NUM_THREADS, 0, st>>>(cu_seqlens, n_seq, order);
    if ((s = after_launch("varlen order launch")) != LA_OK) return s;
    const size_t ws_phi =
        T > 0 && phi_prepass_wanted(use_wide((long)n_seq * H, dk, di)) ? phi_workspace_bytes((long)T * H, dk, phi) : 0;
    size_t off_seg = need;
    if (ws_phi && ws_bytes >= need + ws_phi) {
        if ((s = phi_prepass(&q, &k, reinterpret_cast<uint8_t*>(workspace) + need, (long)T * H * dk, phi, di, st)) !=
            LA_OK)
            return s;
        phi = LA_PHI_IDENTITY;
        off_seg += ws_phi;
    }
    const int nvs = tc_slices(dv);
    const bool wide = use_wide((long)n_seq * H, dk, di);
    int min_seg;
    long max_segs = wide ? 0 : plan_varlen_segments(n_seq, T, H, nvs, di->sms, &min_seg);
    if (max_segs && (ws_bytes < off_seg + varlen_segment_bytes(n_seq, max_segs, H, dk) ||
                     max_segs * H * nvs > (1L << 30)))
        max_segs = 0;  // no room for the segment states: whole sequences
    const long max_nl = max_segs - n_seq;

    tc::Params p{};
    p.mode = 1;
    p.n_seg = 1;
    p.phi = phi;
    p.dk = dk;
    p.n_items = (int)((long)n_seq * H * tc_slices(dv));
    p.H = H;
    p.dv = dv;
    p.cu_seqlens = cu_seqlens;
    p.order = order;
    p.pool = state_pool;
    p.init_idx = init_idx;
    p.s_out = s_out;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.status = di->status;
    CUtensorMap mq, mk, mv, mo;
    const uint64_t Tm = T > 0 ? (uint64_t)T : 1;
    const uint64_t head = (uint64_t)dk * 2, tok = (uint64_t)H * dk * 2;
    const void* any = q ? q : (const void*)order;
    if ((s = make_map(&mq, q ? q : any, dk, H, Tm, head, tok, 1, tc::C)) != LA_OK) return s;
    if ((s = make_map(&mk, k ? k : any, dk, H, Tm, head, tok, 1, tc::C)) != LA_OK) return s;
    if ((s = make_map(&mv, v ? v : any, dv, H, Tm, head, tok, 1, tc::C)) != LA_OK) return s;
    if ((s = make_map(&mo, o ? o : any, dv, H, Tm, head, tok, 1, 32)) != LA_OK) return s;
    if (max_segs) {
        // segments: the plan (length, offsets in work order), the sums of all
        // but each sequence's last segment, the state before every segment,
        // then every segment
        uint8_t* w = reinterpret_cast<uint8_t*>(workspace) + off_seg;
        const size_t ints = round256((size_t)(n_seq + 1) * sizeof(int));
        int* seg_off = reinterpret_cast<int*>(w);
        int* seg_off_nl = reinterpret_cast<int*>(w + ints);
        int* seg_len = reinterpret_cast<int*>(w + 2 * ints);
        float* sums = reinterpret_cast<float*>(w + 2 * ints + 256);
        float* starts = sums + (size_t)max_nl * H * dk * dv;
        vorder::seg_plan_kernel<<<1, 32, 0, st>>>(cu_seqlens, order, n_seq, max_segs, min_seg, tc::C, seg_len, seg_off,
                                                  seg_off_nl);
        if ((s = after_launch("varlen segment plan launch")) != LA_OK) return s;
        p.seg_off = seg_off;
        p.seg_off_nl = seg_off_nl;
        p.n_seq = n_seq;
        p.seg_len_dev = seg_len;
        if (max_nl > 0) {
            tc::Params p1 = p;
            p1.state_only = 1;
            p1.n_items = (int)(max_nl * H * nvs);
            p1.s_out = sums;
            p1.pool = nullptr;
            p1.init_idx = nullptr;
            if ((s = launch_tc(std::min(p1.n_items, di->sms), mq, mk, mv, mo, p1, st,
                               "prefill_tc (varlen segment sums) launch")) != LA_OK)
                return s;
        }
        const long threads = (long)n_seq * H * (dk * dv / 4);
        const int blocks = (int)std::min<long>((threads + segp::NUM_THREADS - 1) / segp::NUM_THREADS, 4L * di->sms);
        segp::seg_prefix_varlen_kernel<<<blocks, segp::NUM_THREADS, 0, st>>>(sums, state_pool, init_idx, order, seg_off,
                                                                            seg_off_nl, starts, n_seq, H, dk * dv);
        if ((s = after_launch("varlen segment prefix launch")) != LA_OK) return s;
        p.n_items = (int)(max_segs * H * nvs);
        p.seg_init = starts;
    }
    if (wide) {
        p.n_items = (int)((long)n_seq * H);
        return launch_wide(std::min(p.n_items, di->sms), mq, mk, mv, mo, p, st, "prefill_wide (varlen) launch");
    }
    const int grid = std::min(p.n_items, di->sms);
    return launch_tc(grid, mq, mk, mv, mo, p, st, "prefill_tc (varlen) launch");
}

la_status la_decode_step_ex(const void* q, const void* k, const void* v, void* o, void* S, int B, int H, int dk,
                            int dv, la_dtype dt, la_state_dtype sdt, la_phi phi, la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(dk, dv, dt);
    if (s != LA_OK) return s;
    if ((s = check_phi(phi)) != LA_OK) return s;
    if (sdt != LA_STATE_FP32 && sdt != LA_STATE_BF16 && sdt != LA_STATE_FP16 && sdt != LA_STATE_FP8_E4M3 &&
        sdt != LA_STATE_FP8_E5M2)
        return fail(LA_ERR_INVALID_ARG, "unknown state dtype %d", (int)sdt);
    if (sdt != LA_STATE_FP32 && dt != LA_BF16)
        return fail(LA_ERR_UNSUPPORTED, "a bf16 or fp16 state needs bf16 q, k, v");
    if (B < 0 || H < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d", B, H);
    const long U = (long)B * H;
    if (U == 0) return LA_OK;
    if (U > (1L << 31) - 1) return fail(LA_ERR_INVALID_ARG, "problem too large");
    if (!q || !k || !v || !o || !S) return fail(LA_ERR_INVALID_ARG, "q, k, v, o, S must be non-null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S))
        return fail(LA_ERR_INVALID_ARG, "all pointers must be 16-byte aligned");
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int grid = (int)U;
    if (dt == LA_FP32) {
        launch_decode<float, float>(dk, grid, q, k, v, o, S, phi, st);
    } else if (sdt == LA_STATE_FP32) {
        launch_decode<__nv_bfloat16, float>(dk, grid, q, k, v, o, S, phi, st);
    } else if (sdt == LA_STATE_BF16) {
        launch_decode<__nv_bfloat16, __nv_bfloat16>(dk, grid, q, k, v, o, S, phi, st);
    } else if (sdt == LA_STATE_FP16) {
        launch_decode<__nv_bfloat16, __half>(dk, grid, q, k, v, o, S, phi, st);
    } else if (sdt == LA_STATE_FP8_E4M3) {
        launch_decode<__nv_bfloat16, __nv_fp8_e4m3>(dk, grid, q, k, v, o, S, phi, st);
    } else {
        launch_decode<__nv_bfloat16, __nv_fp8_e5m2>(dk, grid, q, k, v, o, S, phi, st);
    }
    return after_launch("decode_step launch");
}

la_status la_decode_step(const void* q, const void* k, const void* v, void* o, float* S, int B, int H, int dk,
                         int dv, la_dtype dt, la_stream_t stream) {
    return la_decode_step_ex(q, k, v, o, S, B, H, dk, dv, dt, LA_STATE_FP32, LA_PHI_IDENTITY, stream);
}

// Drafts up to which the FFMA verify kernel is the faster one (measured at
// B=256, H=64, d=128, bf16, ms, FFMA / tensor cores: m = 1 0.153 / 0.206,
// m = 4 0.164 / 0.215, m = 8 0.242 / 0.225, m = 12 0.392 / 0.241, m = 16
// 0.584 / 0.261): below that the FFMA kernel streams the state at the HBM
// rate and the tensor-core kernel's per-unit chain (16 tf32 products, TMEM
// read-back) is longer than a unit's share of the bandwidth.
constexpr int kVerifyFfmaMaxM = 4;

la_status la_decode_verify(const void* q, const void* k, const void* v, void* o, const float* S, int B, int H,
                           int m, int dk, int dv, la_dtype dt, la_phi phi, la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(dk, dv, dt);
    if (s != LA_OK) return s;
    if ((s = check_phi(phi)) != LA_OK) return s;
    if (B < 0 || H < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d", B, H);
    if (m < 1 || m > dmulti::MAX_M) return fail(LA_ERR_INVALID_ARG, "m=%d outside 1..%d", m, dmulti::MAX_M);
    const long U = (long)B * H;
    if (U == 0) return LA_OK;
    if (U > (1L << 31) - 1) return fail(LA_ERR_INVALID_ARG, "problem too large");
    if (!q || !k || !v || !o || !S) return fail(LA_ERR_INVALID_ARG, "q, k, v, o, S must be non-null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S))
        return fail(LA_ERR_INVALID_ARG, "all pointers must be 16-byte aligned");
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // bf16 at d = 128: the q S_0 products on the tensor cores (tf32 reads of
    // the fp32 state) beyond kVerifyFfmaMaxM drafts (LA_VERIFY_TC=1 / 0
    // forces them on / off)
    bool tcv = dt == LA_BF16 && dk == 128 && m > kVerifyFfmaMaxM;
    if (dt == LA_BF16 && dk == 128)
        if (const char* e = getenv("LA_VERIFY_TC")) tcv = e[0] == '1';
    if (tcv) {
        CUtensorMap ms;
        if ((s = make_state_map(&ms, S, 128, (uint64_t)U)) != LA_OK) return s;
        const int grid = (int)std::min<long>(U, di->sms);
        dmulti::verify_tf32_kernel<<<grid, dmulti::vtf::THREADS, dmulti::vtf::SMEM_BYTES, st>>>(
            ms, reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(k),
            reinterpret_cast<const __nv_bfloat16*>(v), reinterpret_cast<__nv_bfloat16*>(o), U, m, phi, di->status);
    } else if (dt == LA_BF16) {
        launch_verify<__nv_bfloat16>(dk, m, (int)U, q, k, v, o, S, phi, st);
    } else {
        launch_verify<float>(dk, m, (int)U, q, k, v, o, S, phi, st);
    }
    return after_launch("decode_verify launch");
}

la_status la_decode_commit(const void* k, const void* v, float* S, const int32_t* accepted, int B, int H, int m,
                           int dk, int dv, la_dtype dt, la_phi phi, la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(dk, dv, dt);
    if (s != LA_OK) return s;
    if ((s = check_phi(phi)) != LA_OK) return s;
    if (B < 0 || H < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d", B, H);
    if (m < 1 || m > dmulti::MAX_M) return fail(LA_ERR_INVALID_ARG, "m=%d outside 1..%d", m, dmulti::MAX_M);
    const long U = (long)B * H;
    if (U == 0) return LA_OK;
    if (U > (1L << 31) - 1) return fail(LA_ERR_INVALID_ARG, "problem too large");
    if (!k || !v || !S || !accepted) return fail(LA_ERR_INVALID_ARG, "k, v, S, accepted must be non-null");
    if (!aligned16(k) || !aligned16(v) || !aligned16(S) || (reinterpret_cast<uintptr_t>(accepted) & 3u))
        return fail(LA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned, accepted 4-byte aligned");
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (env_validate()) {
        std::vector<int32_t> h(B);
        cudaError_t e = cudaMemcpyAsync(h.data(), accepted, sizeof(int32_t) * B, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "copy accepted for validation");
        for (int b = 0; b < B; ++b)
            if (h[b] < 0 || h[b] > m) return fail(LA_ERR_INVALID_ARG, "accepted[%d]=%d outside 0..%d", b, h[b], m);
    }
    const int grid = (int)U;
    if (dt == LA_BF16) launch_commit<__nv_bfloat16>(dk, m, grid, k, v, S, accepted, H, phi, st);
    else launch_commit<float>(dk, m, grid, k, v, S, accepted, H, phi, st);
    return after_launch("decode_commit launch");
}

namespace lcl {
namespace {
int* g_noalloc_ptr[kMaxDevices] = {nullptr};
unsigned long long g_noalloc_ctx[kMaxDevices] = {0};
std::mutex g_noalloc_mu;

// Per-device set-up: the device address of g_noalloc_order for the current
// device, looked up once per context (again after the context was destroyed
// and re-created, e.g. by cudaDeviceReset, whose old address is stale).
la_status noalloc_scratch(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(LA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev] || current_ctx_id() != g_noalloc_ctx[dev]) {
        void* ptr = nullptr;
        if ((e = cudaGetSymbolAddress(&ptr, g_noalloc_order)) != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
        g_noalloc_ptr[dev] = static_cast<int*>(ptr);
        g_noalloc_ctx[dev] = current_ctx_id();
    }
    *out = g_noalloc_ptr[dev];
    return LA_OK;
}
}  // namespace
}  // namespace lcl

extern "C" la_status la_prefill_varlen_noalloc(const void* q, const void* k, const void* v, void* o,
                                               const int32_t* cu_seqlens, int n_seq, int T,
                                               const float* state_pool, int n_pool, const int32_t* init_idx,
                                               float* s_out, int H, int dk, int dv, la_dtype dt, int chunk,
                                               la_stream_t stream) {
    g_last_error[0] = 0;
    if (n_seq > LA_NOALLOC_MAX_SEQS)
        return fail(LA_ERR_INVALID_ARG,
                    "n_seq = %d exceeds the %d sequences the built-in scratch holds; "
                    "use la_prefill_varlen with a workspace",
                    n_seq, LA_NOALLOC_MAX_SEQS);
    if (n_seq < 0) return fail(LA_ERR_INVALID_ARG, "negative size n_seq=%d", n_seq);
    int* scratch = nullptr;
    la_status s = noalloc_scratch(&scratch);
    if (s != LA_OK) return s;
    return la_prefill_varlen(q, k, v, o, cu_seqlens, n_seq, T, state_pool, n_pool, init_idx, s_out, H, dk, dv, dt,
                             chunk, scratch, sizeof(int) * LA_NOALLOC_MAX_SEQS, stream);
}

// One dense tensor-core pass: o = prefill(q, k, v) from `init` (transposed if
// init_t), chunks visited last to first if `reverse`.  When the (unit, value
// slice) items fill less than half of the SMs and `ws` has room, sequences are
// cut into segments as in la_prefill_ex (a state-only pass, then a prefix --
// in reverse order a suffix -- over the segment sums, then every segment).
static la_status tc_dense_pass(const void* q, const void* k, const void* v, void* o, const float* init, bool init_t,
                               float* s_out, bool reverse, long U, int N, int d, DeviceInfo* di, cudaStream_t st,
                               void* ws, size_t ws_bytes) {
    if (N == 0 && !s_out) return LA_OK;
    const int nvs = tc_slices(d);
    tc::Params p{};
    p.mode = 0;
    p.dk = d;
    p.n_items = (int)(U * nvs);
    p.N = N;
    p.dv = d;
    p.s0 = init;
    p.s_out = s_out;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.status = di->status;
    p.n_seg = 1;
    p.phi = LA_PHI_IDENTITY;
    p.reverse = reverse ? 1 : 0;
    p.init_transposed = init_t ? 1 : 0;
    const bool wide = use_wide(U, d, di);
    int seg_len;
    int P = wide ? 1 : plan_segments(U, N, tc_slices(d), di->sms, &seg_len);
    if (P > 1 && (!ws || ws_bytes < segment_workspace_bytes(U, P, d, d) || !aligned16(ws) ||
                  U * P * nvs > (1L << 30)))
        P = 1;
    p.seg_len = P > 1 ? seg_len : ((N + tc::C - 1) / tc::C) * tc::C;
    const void* any = N > 0 ? q : s_out;
    CUtensorMap mq, mk, mv, mo;
    const uint64_t row = (uint64_t)d * 2, Nm = N > 0 ? (uint64_t)N : 1, unit = Nm * row;
    la_status s;
    if ((s = make_map(&mq, N > 0 ? q : any, d, Nm, U, row, unit, tc::C, 1)) != LA_OK) return s;
    if ((s = make_map(&mk, N > 0 ? k : any, d, Nm, U, row, unit, tc::C, 1)) != LA_OK) return s;
    if ((s = make_map(&mv, N > 0 ? v : any, d, Nm, U, row, unit, tc::C, 1)) != LA_OK) return s;
    if ((s = make_map(&mo, N > 0 ? o : any, d, Nm, U, row, unit, 32, 1)) != LA_OK) return s;
    if (P > 1) {
        float* sums = reinterpret_cast<float*>(ws);
        float* starts = sums + (size_t)U * (P - 1) * d * d;
        tc::Params p1 = p;
        p1.n_seg = P - 1;
        p1.seg_base = reverse ? 1 : 0;  // the segments whose sums reach another segment's start
        p1.n_items = (int)(U * (P - 1) * nvs);
        p1.s0 = nullptr;
        p1.init_transposed = 0;
        p1.s_out = sums;
        p1.s_out_per_seg = 1;
        p1.state_only = 1;
        if ((s = launch_tc(std::min(p1.n_items, di->sms), mq, mk, mv, mo, p1, st, "prefill_tc (segment sums) launch")) !=
            LA_OK)
            return s;
        const long threads = U * (long)(d * d / 4);
        const int blocks = (int)std::min<long>((threads + segp::NUM_THREADS - 1) / segp::NUM_THREADS, 4L * di->sms);
        segp::seg_prefix_kernel<<<blocks, segp::NUM_THREADS, 0, st>>>(sums, init, starts, U, P, d * d, reverse ? 1 : 0,
                                                                     init_t ? 1 : 0, d);
        if ((s = after_launch("segment prefix launch")) != LA_OK) return s;
        p.n_seg = P;
        p.n_items = (int)(U * P * nvs);
        p.seg_init = starts;
        p.init_transposed = 0;  // the segment starts are in the usual layout
    }
    if (wide) {
        p.n_items = (int)U;
        return launch_wide(std::min(p.n_items, di->sms), mq, mk, mv, mo, p, st, "prefill_wide (backward pass) launch");
    }
    return launch_tc(std::min(p.n_items, di->sms), mq, mk, mv, mo, p, st, "prefill_tc (backward pass) launch");
}

size_t la_prefill_backward_workspace_size(int B, int H, int N, int d_k, int d_v, la_dtype dt) {
    if (B <= 0 || H <= 0 || N <= 0 || d_k != d_v || (d_k != 64 && d_k != 128)) return 0;
    DeviceInfo* di;
    if (device_info(&di) != LA_OK) return 0;
    int seg_len;
    const long U = (long)B * H;
    if (!use_tensor_cores(d_k, dt)) return segment_workspace_bytes(U, plan_segments_simt_max(U, N, di->sms), d_k, d_v);
    return segment_workspace_bytes(U, plan_segments(U, N, tc_slices(d_k), di->sms, &seg_len), d_k, d_v);
}

la_status la_prefill_backward(const void* q, const void* k, const void* v, const void* dout, const float* s0,
                              const float* ds_n, void* dq, void* dk, void* dv, float* ds0, int B, int H, int N,
                              int d_k, int d_v, la_dtype dt, la_stream_t stream) {
    return la_prefill_backward_ex(q, k, v, dout, s0, ds_n, dq, dk, dv, ds0, B, H, N, d_k, d_v, dt, nullptr, 0,
                                  stream);
}

la_status la_prefill_backward_ex(const void* q, const void* k, const void* v, const void* dout, const float* s0,
                                 const float* ds_n, void* dq, void* dk, void* dv, float* ds0, int B, int H, int N,
                                 int d_k, int d_v, la_dtype dt, void* workspace, size_t ws_bytes,
                                 la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(d_k, d_v, dt);
    if (s != LA_OK) return s;
    if (B < 0 || H < 0 || N < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d N=%d", B, H, N);
    const long U = (long)B * H;
    if (U > (1L << 29) || (long)N * U > (1L << 40)) return fail(LA_ERR_INVALID_ARG, "problem too large");
    if (U == 0) return LA_OK;
    if (N > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv))
        return fail(LA_ERR_INVALID_ARG, "q, k, v, dout, dq, dk, dv must be non-null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(s0) || !aligned16(ds_n) || !aligned16(ds0))
        return fail(LA_ERR_INVALID_ARG, "all pointers must be 16-byte aligned");
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Each gradient is a forward pass over permuted inputs (G_t is the suffix
    // sum dS_N + sum_{t' >= t} q_t'^T do_t'):
    //   dq_t = do_t S_t^T : prefill(dO, V, K) from s0^T
    //   dk_t = v_t G_t^T  : prefill(V, dO, Q) from dS_N^T, chunks last to first
    //   dv_t = k_t G_t    : prefill(K, Q, dO) from dS_N, chunks last to first;
    //                       its final state is G_1 = dS_0
    // on the tensor cores for bf16 with d = 128 (unless LA_BACKWARD_SIMT=1),
    // else on the FFMA path
    if (use_tensor_cores(d_k, dt) && !env_flag("LA_BACKWARD_SIMT")) {
        if (N > 0) {
            if ((s = tc_dense_pass(dout, v, k, dq, s0, true, nullptr, false, U, N, d_k, di, st, workspace, ws_bytes)) !=
                LA_OK)
                return s;
            if ((s = tc_dense_pass(v, dout, q, dk, ds_n, true, nullptr, true, U, N, d_k, di, st, workspace, ws_bytes)) !=
                LA_OK)
                return s;
        }
        // (the passes run in stream order, so they share the workspace)
        return tc_dense_pass(k, q, dout, dv, ds_n, false, ds0, true, U, N, d_k, di, st, workspace, ws_bytes);
    }
    if (N == 0 && !ds0) return LA_OK;
    if (N > 0) {
        if ((s = simt_dense(dout, v, k, dq, s0, true, nullptr, false, LA_PHI_IDENTITY, U, N, d_k, dt, 0, di,
                            workspace, ws_bytes, st)) != LA_OK)
            return s;
        if ((s = simt_dense(v, dout, q, dk, ds_n, true, nullptr, true, LA_PHI_IDENTITY, U, N, d_k, dt, 0, di,
                            workspace, ws_bytes, st)) != LA_OK)
            return s;
    }
    return simt_dense(k, q, dout, dv, ds_n, false, ds0, true, LA_PHI_IDENTITY, U, N, d_k, dt, 0, di, workspace,
                      ws_bytes, st);
}

size_t la_prefill_host_workspace_size(int B, int H, int N, int dk, int dv, la_dtype dt, int group) {
    if (B <= 0 || H <= 0 || N < 0 || group <= 0 || dk <= 0 || dv <= 0) return 0;
    const size_t esz = dt == LA_FP32 ? 4 : 2;
    const long g = std::min<long>(group, (long)B * H);
    const size_t tok = round256((size_t)g * N * dk * esz) * 2 + round256((size_t)g * N * dv * esz) * 2;
    const size_t st = round256((size_t)g * dk * dv * 4) * 2;
    return 2 * (tok + st);  // two staging buffers
}

la_status la_prefill_host(const void* q, const void* k, const void* v, void* o, const float* s0, float* s_out, int B,
                          int H, int N, int dk, int dv, la_dtype dt, int group, void* workspace, size_t ws_bytes,
                          la_stream_t stream) {
    g_last_error[0] = 0;
    la_status s = check_dims(dk, dv, dt);
    if (s != LA_OK) return s;
    if (B < 0 || H < 0 || N < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d N=%d", B, H, N);
    if (group <= 0) return fail(LA_ERR_INVALID_ARG, "group = %d must be positive", group);
    const long U = (long)B * H;
    if (U == 0) return LA_OK;
    if (U > (1L << 30) || (long)N * U > (1L << 40)) return fail(LA_ERR_INVALID_ARG, "problem too large");
    if (N > 0 && (!q || !k || !v || !o)) return fail(LA_ERR_INVALID_ARG, "q, k, v, o must be non-null");
    const size_t need = la_prefill_host_workspace_size(B, H, N, dk, dv, dt, group);
    if (!workspace || ws_bytes < need || !aligned16(workspace))
        return fail(LA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu", need, ws_bytes);
    DeviceInfo* di;
    if ((s = device_info(&di)) != LA_OK) return s;
    cudaError_t e = cudaSuccess;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        if (!di->h2d && (e = cudaStreamCreateWithFlags(&di->h2d, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreateWithFlags");
        if (!di->d2h && (e = cudaStreamCreateWithFlags(&di->d2h, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreateWithFlags");
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const long g = std::min<long>(group, U);
    const size_t esz = dt == LA_FP32 ? 4 : 2;
    const size_t qk_b = round256((size_t)g * N * dk * esz), vo_b = round256((size_t)g * N * dv * esz);
    const size_t s_b = round256((size_t)g * dk * dv * 4);
    const size_t buf_b = 2 * qk_b + 2 * vo_b + 2 * s_b;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    // events: start, then per staging buffer "copied in", "computed", "copied out"
    cudaEvent_t ev[7] = {};
    for (int i = 0; i < 7 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    cudaEvent_t ev_start = ev[0], *ev_in = ev + 1, *ev_comp = ev + 3, *ev_out = ev + 5;
    auto cleanup = [&]() {
        for (int i = 0; i < 7; ++i)
            if (ev[i]) cudaEventDestroy(ev[i]);
    };
    auto cu = [&](cudaError_t x, const char* what) -> la_status {
        if (x == cudaSuccess) return LA_OK;
        cleanup();
        return cuda_fail(x, what);
    };
    if (e != cudaSuccess) return cu(e, "cudaEventCreate");
    // the copy streams start after the work already queued on the caller's stream
    if ((s = cu(cudaEventRecord(ev_start, st), "cudaEventRecord")) != LA_OK) return s;
    if ((s = cu(cudaStreamWaitEvent(di->h2d, ev_start, 0), "cudaStreamWaitEvent")) != LA_OK) return s;
    if ((s = cu(cudaStreamWaitEvent(di->d2h, ev_start, 0), "cudaStreamWaitEvent")) != LA_OK) return s;
    const auto H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;
    for (long u0 = 0, i = 0; u0 < U; u0 += g, ++i) {
        const int b = (int)(i & 1);
        const long n = std::min(g, U - u0);
        uint8_t* base = ws + b * buf_b;
        uint8_t *dq = base, *dk_ = dq + qk_b, *dv_ = dk_ + qk_b, *do_ = dv_ + vo_b, *ds0 = do_ + vo_b, *dso = ds0 + s_b;
        const size_t qk_n = (size_t)n * N * dk * esz, vo_n = (size_t)n * N * dv * esz, s_n = (size_t)n * dk * dv * 4;
        const size_t qk_off = (size_t)u0 * N * dk * esz, vo_off = (size_t)u0 * N * dv * esz;
        const size_t s_off = (size_t)u0 * dk * dv;
        // buffer b is free once group i - 2 has been copied out
        if (i >= 2 && (s = cu(cudaStreamWaitEvent(di->h2d, ev_out[b], 0), "cudaStreamWaitEvent")) != LA_OK) return s;
        if (qk_n) {
            if ((s = cu(cudaMemcpyAsync(dq, (const uint8_t*)q + qk_off, qk_n, H2D, di->h2d), "copy q")) != LA_OK ||
                (s = cu(cudaMemcpyAsync(dk_, (const uint8_t*)k + qk_off, qk_n, H2D, di->h2d), "copy k")) != LA_OK ||
                (s = cu(cudaMemcpyAsync(dv_, (const uint8_t*)v + vo_off, vo_n, H2D, di->h2d), "copy v")) != LA_OK)
                return s;
        }
        if (s0 && (s = cu(cudaMemcpyAsync(ds0, s0 + s_off, s_n, H2D, di->h2d), "copy s0")) != LA_OK) return s;
        if ((s = cu(cudaEventRecord(ev_in[b], di->h2d), "cudaEventRecord")) != LA_OK) return s;
        if ((s = cu(cudaStreamWaitEvent(st, ev_in[b], 0), "cudaStreamWaitEvent")) != LA_OK) return s;
        s = la_prefill_ex(dq, dk_, dv_, do_, s0 ? (const float*)ds0 : nullptr, s_out ? (float*)dso : nullptr, 1,
                          (int)n, N, dk, dv, dt, 0, LA_PHI_IDENTITY, nullptr, 0, stream);
        if (s != LA_OK) {
            cleanup();
            return s;
        }
        if ((s = cu(cudaEventRecord(ev_comp[b], st), "cudaEventRecord")) != LA_OK) return s;
        if ((s = cu(cudaStreamWaitEvent(di->d2h, ev_comp[b], 0), "cudaStreamWaitEvent")) != LA_OK) return s;
        if (vo_n && (s = cu(cudaMemcpyAsync((uint8_t*)o + vo_off, do_, vo_n, D2H, di->d2h), "copy o")) != LA_OK)
            return s;
        if (s_out && (s = cu(cudaMemcpyAsync(s_out + s_off, dso, s_n, D2H, di->d2h), "copy s_out")) != LA_OK)
            return s;
        if ((s = cu(cudaEventRecord(ev_out[b], di->d2h), "cudaEventRecord")) != LA_OK) return s;
    }
    // the caller's stream continues once the last copy out (and so every one) is done
    const long last = (U + g - 1) / g - 1;
    if ((s = cu(cudaStreamWaitEvent(st, ev_out[last & 1], 0), "cudaStreamWaitEvent")) != LA_OK) return s;
    cleanup();
    return LA_OK;
}

la_status la_selftest_wait_timeout(int timeout_us, la_stream_t stream) {
    g_last_error[0] = 0;
    if (timeout_us < 1 || timeout_us > 1000000)
        return fail(LA_ERR_INVALID_ARG, "timeout_us = %d outside [1, 1000000]", timeout_us);
    DeviceInfo* di;
    la_status s = device_info(&di);
    if (s != LA_OK) return s;
    selftest::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<unsigned long long>(timeout_us) * 1000ull, di->status);
    return after_launch("selftest launch");
}

la_status la_device_status(int* out, int clear) {
    g_last_error[0] = 0;
    if (!out) return fail(LA_ERR_INVALID_ARG, "out must be non-null");
    DeviceInfo* di;
    la_status s = device_info(&di);
    if (s != LA_OK) return s;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    int v = 0;
    if ((e = cudaMemcpy(&v, di->status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "status read");
    if (clear && (e = cudaMemset(di->status, 0, sizeof(int))) != cudaSuccess) return cuda_fail(e, "status clear");
    *out = v;
    return LA_OK;
}

}  // extern "C"

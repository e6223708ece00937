"""Causal linear attention (Lightning Attention, phi = identity) for B200.

Python binding of the C ABI in ``include/la.h``: every function below only
checks and marshals arguments (torch tensors -> device pointers, the current
CUDA stream) and calls the CUDA library; all computation runs in its kernels.

    S_t = S_{t-1} + k_t (x) v_t,   o_t = q_t S_t

(page "MiniMax-M1で理解する…" (zenn.dev), section "線形アテンションの数学的基礎";
tiled as on page "MiniMax: «Почему M2 в итоге стала моделью с полным
вниманием?»", section 1, glossary entry "Lightning Attention").
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _abi
from ._abi import LAError, lib

__all__ = ["prefill", "prefill_host", "prefill_varlen", "prefill_varlen_noalloc", "prefill_backward", "decode_step",
           "decode_verify",
           "decode_commit",
           "device_status", "LAError",
           "lib", "prefill_workspace_size", "prefill_varlen_workspace_size"]

_DT = {torch.bfloat16: _abi.LA_BF16, torch.float32: _abi.LA_FP32}
PHI = {"identity": _abi.LA_PHI_IDENTITY, "elu1": _abi.LA_PHI_ELU1, "relu": _abi.LA_PHI_RELU}


def _phi_code(phi: str) -> int:
    if phi not in PHI:
        raise ValueError(f"unknown feature map {phi!r}; one of {sorted(PHI)}")
    return PHI[phi]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")
    return _DT[t.dtype]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device: torch.device):
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _need_host(t: torch.Tensor, name: str, dtype=None):
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def prefill_workspace_size(B: int, H: int, N: int, d: int, dtype: torch.dtype, phi: str = "identity") -> int:
    return int(lib.la_prefill_workspace_size_ex(B, H, N, d, d, _DT[dtype], _phi_code(phi)))


def prefill_varlen_workspace_size(n_seq: int, T: int, H: int, d: int, dtype: torch.dtype,
                                  phi: str = "identity") -> int:
    return int(lib.la_prefill_varlen_workspace_size_ex(n_seq, T, H, d, d, _DT[dtype], _phi_code(phi)))


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, s0: Optional[torch.Tensor] = None, *,
            chunk: int = 0, out: Optional[torch.Tensor] = None, s_out: Optional[torch.Tensor] = None,
            return_state: bool = True, workspace: Optional[torch.Tensor] = None, phi: str = "identity"
            ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Dense prefill over q, k, v of shape [B, H, N, d]; returns (O, S_N).

    s0 (fp32 [B, H, d, d]) is the state before the first token (zero if None);
    phi ("identity", "elu1", "relu") is the feature map on q and k.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, q.device)
    if q.dim() != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B, H, N, dk] and v [B, H, N, dv]")
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, q.device)
    if s0 is not None:
        _need(s0, "s0", torch.float32, q.device)
        if tuple(s0.shape) != (B, H, dk, dv):
            raise ValueError("s0 must be [B, H, dk, dv]")
    if s_out is None and return_state:
        s_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if s_out is not None:
        _need(s_out, "s_out", torch.float32, q.device)
    need = int(lib.la_prefill_workspace_size_ex(B, H, N, dk, dv, dt, _phi_code(phi)))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _abi.check(lib.la_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(s0), _ptr(s_out),
                                     B, H, N, dk, dv, dt, chunk, _phi_code(phi), _ptr(workspace), ws_bytes,
                                     _stream(q.device)),
                   "la_prefill_ex")
    return out, s_out


def prefill_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, s0: Optional[torch.Tensor] = None, *,
                 group: int = 8, out: Optional[torch.Tensor] = None, s_out: Optional[torch.Tensor] = None,
                 return_state: bool = True, workspace: Optional[torch.Tensor] = None,
                 device: Optional[torch.device] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``prefill`` on host tensors (page-locked for overlap): q, k, v [B, H, N, d]
    and s0 [B, H, d, d] fp32 on the CPU; returns host (O, S_N).

    Groups of ``group`` (batch, head) units are copied in, computed and copied
    out on overlapping streams of ``device`` (default: the current CUDA
    device).  Asynchronous: synchronise that device's current stream before
    reading the results.
    """
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need_host(t, n, q.dtype)
    if q.dim() != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B, H, N, dk] and v [B, H, N, dv]")
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    pin = torch.cuda.is_available()
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, pin_memory=pin)
    _need_host(out, "out", q.dtype)
    if s0 is not None:
        _need_host(s0, "s0", torch.float32)
        if tuple(s0.shape) != (B, H, dk, dv):
            raise ValueError("s0 must be [B, H, dk, dv]")
    if s_out is None and return_state:
        s_out = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=pin)
    if s_out is not None:
        _need_host(s_out, "s_out", torch.float32)
    need = int(lib.la_prefill_host_workspace_size(B, H, N, dk, dv, dt, group))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _abi.check(lib.la_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(s0), _ptr(s_out), B, H, N, dk, dv,
                                       dt, group, _ptr(workspace), ws_bytes, _stream(dev)), "la_prefill_host")
    return out, s_out


def prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dout: torch.Tensor,
                     s0: Optional[torch.Tensor] = None, ds_n: Optional[torch.Tensor] = None, *,
                     need_ds0: bool = True, workspace: Optional[torch.Tensor] = None):
    """Gradients of ``prefill`` for dL/dO = dout and dL/dS_N = ds_n (zero if None).

    q, k, v, dout: [B, H, N, d]; s0, ds_n: fp32 [B, H, d, d] or None.
    Returns (dq, dk, dv, ds0) with dq, dk, dv in the input dtype and ds0 fp32
    (None unless need_ds0).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, n, q.dtype, q.device)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or dout.shape != v.shape:
        raise ValueError("q, k, v, dout must all be [B, H, N, d]")
    B, H, N, d = q.shape
    for t, n in ((s0, "s0"), (ds_n, "ds_n")):
        if t is not None:
            _need(t, n, torch.float32, q.device)
            if tuple(t.shape) != (B, H, d, d):
                raise ValueError(f"{n} must be [B, H, d, d]")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds0 = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device) if need_ds0 else None
    need = int(lib.la_prefill_backward_workspace_size(B, H, N, d, d, _dtype_code(q)))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _abi.check(lib.la_prefill_backward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(s0), _ptr(ds_n), _ptr(dq),
                                              _ptr(dk), _ptr(dv), _ptr(ds0), B, H, N, d, d, _dtype_code(q),
                                              _ptr(workspace), ws_bytes, _stream(q.device)), "la_prefill_backward_ex")
    return dq, dk, dv, ds0


def _check_packed(q, k, v, cu_seqlens, state_pool, init_idx, out, s_out):
    """Device, dtype, contiguity and shape checks of a packed ragged batch;
    returns (T, H, dk, dv, n_seq, n_pool).  Run before any launch, so that a
    wrongly sized buffer never reaches a kernel."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, q.device)
    _need(cu_seqlens, "cu_seqlens", torch.int32, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError("q, k must be [T, H, dk] and v [T, H, dv]")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be [n_seq + 1]")
    T, H, dk = q.shape
    dv = v.shape[-1]
    n_seq = cu_seqlens.numel() - 1
    if out is not None:
        _need(out, "out", q.dtype, q.device)
        if tuple(out.shape) != (T, H, dv):
            raise ValueError(f"out must be [T, H, dv] = {(T, H, dv)}, got {tuple(out.shape)}")
    n_pool = 0
    if state_pool is not None:
        _need(state_pool, "state_pool", torch.float32, q.device)
        if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (H, dk, dv):
            raise ValueError("state_pool must be [n_pool, H, dk, dv]")
        n_pool = state_pool.shape[0]
    if init_idx is not None:
        _need(init_idx, "init_idx", torch.int32, q.device)
        if init_idx.numel() != n_seq:
            raise ValueError("init_idx must have n_seq entries")
    if s_out is not None:
        _need(s_out, "s_out", torch.float32, q.device)
        if tuple(s_out.shape) != (n_seq, H, dk, dv):
            raise ValueError(f"s_out must be [n_seq, H, dk, dv] = {(n_seq, H, dk, dv)}, got {tuple(s_out.shape)}")
    return T, H, dk, dv, n_seq, n_pool


def prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                   state_pool: Optional[torch.Tensor] = None, init_idx: Optional[torch.Tensor] = None, *,
                   chunk: int = 0, out: Optional[torch.Tensor] = None, s_out: Optional[torch.Tensor] = None,
                   return_state: bool = True, workspace: Optional[torch.Tensor] = None, phi: str = "identity"
                   ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Packed ragged prefill: q, k [T, H, d], v [T, H, d], cu_seqlens int32 [n_seq + 1].

    Sequence n starts from state_pool[init_idx[n]] when init_idx[n] >= 0;
    phi is the feature map on q and k.  Returns (O [T, H, d], S [n_seq, H, d, d]).
    """
    T, H, dk, dv, n_seq, n_pool = _check_packed(q, k, v, cu_seqlens, state_pool, init_idx, out, s_out)
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    if s_out is None and return_state:
        s_out = torch.empty((max(n_seq, 0), H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(lib.la_prefill_varlen_workspace_size_ex(n_seq, T, H, dk, dv, dt, _phi_code(phi)))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _abi.check(lib.la_prefill_varlen_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), n_seq, T,
                                            _ptr(state_pool), n_pool, _ptr(init_idx), _ptr(s_out), H, dk, dv, dt,
                                            chunk, _phi_code(phi), _ptr(workspace), ws_bytes, _stream(q.device)),
                   "la_prefill_varlen_ex")
    return out, s_out


def prefill_varlen_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                           state_pool: Optional[torch.Tensor] = None, init_idx: Optional[torch.Tensor] = None, *,
                           out: torch.Tensor, s_out: Optional[torch.Tensor] = None, chunk: int = 0) -> None:
    """prefill_varlen for callers that cannot allocate device memory.

    The caller passes every output buffer; the library uses its built-in
    scratch (at most ``_abi.NOALLOC_MAX_SEQS`` sequences per call) instead of a
    workspace.  Calls share that scratch: order them on one stream.  With no
    workspace the call never cuts sequences into segments, so batches of a few
    long sequences run one CTA per (sequence, head, value slice); the feature
    map is the identity.
    """
    if out is None:
        raise ValueError("out is required: this call allocates nothing")
    T, H, dk, dv, n_seq, n_pool = _check_packed(q, k, v, cu_seqlens, state_pool, init_idx, out, s_out)
    with torch.cuda.device(q.device):
        _abi.check(lib.la_prefill_varlen_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), n_seq, T,
                                                 _ptr(state_pool), n_pool, _ptr(init_idx), _ptr(s_out), H, dk, dv,
                                                 _dtype_code(q), chunk, _stream(q.device)),
                   "la_prefill_varlen_noalloc")


_STATE_DT = {torch.float32: _abi.LA_STATE_FP32, torch.bfloat16: _abi.LA_STATE_BF16,
             torch.float16: _abi.LA_STATE_FP16, torch.float8_e4m3fn: _abi.LA_STATE_FP8_E4M3,
             torch.float8_e5m2: _abi.LA_STATE_FP8_E5M2}


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, S: torch.Tensor, *,
                out: Optional[torch.Tensor] = None, phi: str = "identity") -> torch.Tensor:
    """One token per (batch, head): S <- S + k (x) v in place, returns o = q S.

    q, k, v: [B, H, d]; S: [B, H, d, d] in fp32, or in bf16 / fp16 /
    float8_e4m3fn / float8_e5m2 (state stored in low precision, updated in fp32
    and rounded to nearest even, the 8-bit formats saturating at their largest
    finite value; needs bf16 q, k, v).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, q.device)
    if S.dtype not in _STATE_DT:
        raise TypeError(f"S must be float32, bfloat16, float16, float8_e4m3fn or float8_e5m2, got {S.dtype}")
    _need(S, "S", S.dtype, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.shape[:2] != q.shape[:2]:
        raise ValueError("q, k must be [B, H, dk] and v [B, H, dv]")
    B, H, dk = q.shape
    dv = v.shape[-1]
    if tuple(S.shape) != (B, H, dk, dv):
        raise ValueError("S must be [B, H, dk, dv]")
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, q.device)
    with torch.cuda.device(q.device):
        _abi.check(lib.la_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(S), B, H, dk, dv,
                                         _dtype_code(q), _STATE_DT[S.dtype], _phi_code(phi), _stream(q.device)),
                   "la_decode_step_ex")
    return out


def decode_verify(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, S: torch.Tensor, *,
                  out: Optional[torch.Tensor] = None, phi: str = "identity") -> torch.Tensor:
    """Outputs for m draft tokens per (batch, head) without changing S.

    q, k, v: [B, H, m, d] (1 <= m <= 16); S: fp32 [B, H, d, d] (read only).
    Returns o [B, H, m, d] with o_t = q_t (S + sum_{s<=t} k_s (x) v_s).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, q.device)
    _need(S, "S", torch.float32, q.device)
    if q.dim() != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B, H, m, dk] and v [B, H, m, dv]")
    B, H, m, dk = q.shape
    dv = v.shape[-1]
    if tuple(S.shape) != (B, H, dk, dv):
        raise ValueError("S must be [B, H, dk, dv]")
    if out is None:
        out = torch.empty((B, H, m, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, q.device)
    with torch.cuda.device(q.device):
        _abi.check(lib.la_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(S), B, H, m, dk, dv,
                                        _dtype_code(q), _phi_code(phi), _stream(q.device)), "la_decode_verify")
    return out


def decode_commit(k: torch.Tensor, v: torch.Tensor, S: torch.Tensor, accepted: torch.Tensor, *,
                  phi: str = "identity") -> None:
    """S <- S + sum_{t < accepted[b]} k_t (x) v_t in place (the accepted drafts).

    k, v: [B, H, m, d]; S: fp32 [B, H, d, d]; accepted: int32 [B] on the device.
    """
    _need(k, "k", k.dtype, k.device)
    _need(v, "v", k.dtype, k.device)
    _need(S, "S", torch.float32, k.device)
    _need(accepted, "accepted", torch.int32, k.device)
    B, H, m, dk = k.shape
    dv = v.shape[-1]
    if tuple(S.shape) != (B, H, dk, dv) or accepted.numel() != B:
        raise ValueError("S must be [B, H, dk, dv] and accepted [B]")
    with torch.cuda.device(k.device):
        _abi.check(lib.la_decode_commit(_ptr(k), _ptr(v), _ptr(S), _ptr(accepted), B, H, m, dk, dv,
                                        _dtype_code(k), _phi_code(phi), _stream(k.device)), "la_decode_commit")


def device_status(clear: bool = True) -> int:
    """Device status word (0 = ok, 4 = a bounded device wait timed out). Synchronizes."""
    import ctypes
    v = ctypes.c_int(0)
    _abi.check(lib.la_device_status(ctypes.byref(v), 1 if clear else 0), "la_device_status")
    return int(v.value)

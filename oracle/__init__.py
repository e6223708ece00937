"""fp64 CPU oracle for causal linear attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library in ``long_context_linear_b200`` and never imports it.

What it computes (page "MiniMax-M1で理解する：大規模言語モデルのコンテキスト長
限界を突破する革新的アーキテクチャ" (zenn.dev), section "線形アテンションの数学的
基礎"): with phi = identity,

* recurrent form   S_t = S_{t-1} + k_t v_t^T,  o_t = q_t S_t      (``recurrent``)
* factorised form  O = (Q K^T ⊙ M) V + Q S0,   S_N = S0 + K^T V    (``quadratic``)
  where M is the causal mask that keeps the diagonal (the tiled reading of
  page "MiniMax: «Почему M2 в итоге стала моделью с полным вниманием?»",
  section 1, glossary entry "Lightning Attention");
* one decode step  S <- S + k v^T, o = q S                          (``decode``)
* packed ragged batches with an optional resumed state per sequence (``varlen``);
* gradients of the recurrent form for given dO and dS_N (``backward``): the
  chain rule through the recurrence, dq_t = do_t S_t^T, and with
  G_t = sum_{t'>=t} q_t'^T do_t' + dS_N, dk_t = G_t v_t, dv_t = G_t^T k_t,
  dS_0 = G_1.

Every function takes ``phi`` (None / "identity", "elu1", "relu"): the
element-wise feature map of the same page's phi(Q)(phi(K)^T V), applied in
float64 to q and k before the recurrence (``feature_map``).

Inputs are the exact stored values (bf16 or fp32) widened to float64; all
arithmetic is float64.  Pins: ``tests/test_oracle.py``.  No function here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc -O2 -fopenmp) into ``oracle/_build``."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        for name in ("oracle_recurrent", "oracle_quadratic"):
            fn = getattr(lib, name)
            fn.argtypes = [ctypes.c_int] * 4 + [dp] * 6
            fn.restype = None
        lib.oracle_decode.argtypes = [ctypes.c_int] * 3 + [dp] * 5
        lib.oracle_decode.restype = None
        lib.oracle_varlen.argtypes = [ctypes.c_int, ip] + [ctypes.c_int] * 3 + [dp] * 4 + [ip, dp, dp]
        lib.oracle_varlen.restype = None
        lib.oracle_backward.argtypes = [ctypes.c_int] * 4 + [dp] * 10
        lib.oracle_backward.restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _f64(a) -> np.ndarray:
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (CPU): widen exactly
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def feature_map(x, phi: Optional[str]) -> np.ndarray:
    """phi applied element-wise in float64: identity, elu(x) + 1 or relu(x)."""
    x = _f64(x)
    if phi in (None, "identity"):
        return x
    if phi == "elu1":
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    if phi == "relu":
        return np.maximum(x, 0.0)
    raise ValueError(f"unknown feature map {phi!r}")


def _dense(fn, q, k, v, s0, phi=None):
    q, k, v, s0 = feature_map(q, phi), feature_map(k, phi), _f64(v), _f64(s0)
    *lead, N, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and tuple(v.shape[:-1]) == tuple(q.shape[:-1])
    U = int(np.prod(lead)) if lead else 1
    o = np.zeros(tuple(lead) + (N, dv), np.float64)
    s_out = np.zeros(tuple(lead) + (dk, dv), np.float64)
    if s0 is not None:
        assert s0.shape == s_out.shape
    fn(U, N, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(s0), _ptr(o), _ptr(s_out))
    return o, s_out


def recurrent(q, k, v, s0=None, phi=None) -> Tuple[np.ndarray, np.ndarray]:
    """Token-by-token recurrence on dense [..., N, d] inputs -> (O, S_N)."""
    return _dense(_load().oracle_recurrent, q, k, v, s0, phi)


def quadratic(q, k, v, s0=None, phi=None) -> Tuple[np.ndarray, np.ndarray]:
    """Masked quadratic form (Q K^T ⊙ M) V + Q S0 and S0 + K^T V (small N)."""
    return _dense(_load().oracle_quadratic, q, k, v, s0, phi)


def decode(q, k, v, S, phi=None) -> Tuple[np.ndarray, np.ndarray]:
    """One decode step: returns (o, S_new); the input S is not modified."""
    q, k, v = feature_map(q, phi), feature_map(k, phi), _f64(v)
    S = _f64(S).copy()
    dk, dv = q.shape[-1], v.shape[-1]
    U = int(np.prod(q.shape[:-1]))
    o = np.zeros(tuple(q.shape[:-1]) + (dv,), np.float64)
    _load().oracle_decode(U, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(o))
    return o, S


def varlen(q, k, v, cu_seqlens, state_pool=None, init_idx=None, phi=None):
    """Packed ragged batch: q,k [T,H,dk], v [T,H,dv] -> (O [T,H,dv], S [n_seq,H,dk,dv])."""
    q, k, v = feature_map(q, phi), feature_map(k, phi), _f64(v)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    T, H, dk = q.shape
    dv = v.shape[-1]
    n_seq = int(cu.shape[0]) - 1
    pool = _f64(state_pool)
    idx = None if init_idx is None else np.ascontiguousarray(np.asarray(init_idx, dtype=np.int32))
    o = np.zeros((T, H, dv), np.float64)
    s_out = np.zeros((n_seq, H, dk, dv), np.float64)
    ip = ctypes.POINTER(ctypes.c_int)
    _load().oracle_varlen(n_seq, cu.ctypes.data_as(ip), H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                          _ptr(pool), idx.ctypes.data_as(ip) if idx is not None else ip(),
                          _ptr(o), _ptr(s_out))
    return o, s_out


def backward(q, k, v, do, s0=None, ds_n=None):
    """Gradients (dq, dk, dv, ds0) of the dense recurrent form for dL/dO = do
    and dL/dS_N = ds_n (zero if None); shapes as ``recurrent``."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    s0, ds_n = _f64(s0), _f64(ds_n)
    *lead, N, d_k = q.shape
    d_v = v.shape[-1]
    assert k.shape == q.shape and v.shape == do.shape and tuple(v.shape[:-1]) == tuple(q.shape[:-1])
    U = int(np.prod(lead)) if lead else 1
    dq, dk = np.zeros_like(q), np.zeros_like(k)
    dv = np.zeros_like(v)
    ds0 = np.zeros(tuple(lead) + (d_k, d_v), np.float64)
    _load().oracle_backward(U, N, d_k, d_v, _ptr(q), _ptr(k), _ptr(v), _ptr(s0), _ptr(do), _ptr(ds_n),
                            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds0))
    return dq, dk, dv, ds0

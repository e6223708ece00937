"""Decode step with the state stored in low precision — TEST INFRASTRUCTURE ONLY.

Same import rule as the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may use it.

The pages warn that the recurrent state of linear attention is far more
sensitive to numerical precision than a KV cache: it is rewritten at every
token, so rounding errors from low-precision state storage accumulate (page
"MiniMax: «Почему M2 в итоге стала моделью с полным вниманием?» (конспект)",
section 4; page "ノーフリーランチ：MiniMax M2が高効率アテンション機構を解体",
infrastructure section).  This module states what "fp32 compute, low-precision
storage" means for one decode step of S_t = S_{t-1} + k_t v_t^T, o_t = q_t S_t
(page "MiniMax-M1で理解する…", section "線形アテンションの数学的基礎"):

* every state element is updated in fp32: s = RN_fp32(S_stored + k_i v_j)
  (for bf16 inputs the product k_i v_j has at most 16 significant bits and is
  exact in fp32, so this is one fp32 addition of the exact product);
* the result is rounded to the storage format (bf16, fp16, or the 8-bit
  formats e4m3 / e5m2) to nearest even; the 8-bit formats saturate to their
  largest finite value (448 / 57344) instead of overflowing;
* o = q S uses the stored, rounded state (computed here in float64).

Because the stored state is a rounding decision taken in fp32 on both sides, a
GPU implementation of the same rule must reproduce the stored state bit for
bit; ``o`` is compared within tolerance.  Pins: ``tests/test_oracle.py``.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

FORMATS = ("fp32", "bf16", "fp16", "fp8_e4m3", "fp8_e5m2")

# 8-bit floating-point formats: (mantissa bits, exponent of the smallest
# normal value, largest finite value).  e4m3: bias 7, no infinities, the
# all-ones code is NaN, so the largest finite value is 1.75 * 2^8; e5m2: bias
# 15, IEEE-like, largest finite 1.75 * 2^15.
FP8 = {"fp8_e4m3": (3, -6, 448.0), "fp8_e5m2": (2, -14, 57344.0)}


def round_bf16(x) -> np.ndarray:
    """float32 values rounded to bfloat16 (8 significant bits) to nearest even,
    returned as float32.  Finite inputs only."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32)


def round_fp16(x) -> np.ndarray:
    """float32 values rounded to IEEE binary16 to nearest even, as float32."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def round_fp8(x, fmt: str) -> np.ndarray:
    """float32 values rounded to an 8-bit format (``FP8``) to nearest even,
    saturating at the largest finite value, returned as float32.  Finite
    inputs only.  Below the smallest normal value the spacing stays that of
    the smallest binade (subnormals)."""
    mant, emin, vmax = FP8[fmt]
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                          # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, emin)                 # binade of a (or the subnormal range)
    quantum = np.ldexp(1.0, e - mant)            # spacing of representable values there
    r = np.round(a / quantum) * quantum          # a / quantum is exact; np.round is half-to-even
    r = np.minimum(r, vmax)
    return (np.sign(x) * r).astype(np.float32)


def round_to(x, fmt: str) -> np.ndarray:
    if fmt in FP8:
        return round_fp8(x, fmt)
    if fmt == "fp32":
        return np.asarray(x, dtype=np.float32)
    if fmt == "bf16":
        return round_bf16(x)
    if fmt == "fp16":
        return round_fp16(x)
    raise ValueError(f"unknown storage format {fmt!r}")


def _f32(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (any dtype) -> exact float32 values
        a = a.detach().cpu().float().numpy()
    return np.asarray(a, dtype=np.float32)


def decode_lowp(q, k, v, S, fmt: str) -> Tuple[np.ndarray, np.ndarray]:
    """One decode step with the state stored in ``fmt``.

    q, k, v: [..., d_k] / [..., d_v] (values exactly representable in fp32);
    S: [..., d_k, d_v] holding values of the storage format.  Returns
    (o float64 [..., d_v], S_new float32 holding values of ``fmt``).
    """
    q32, k32, v32, S32 = _f32(q), _f32(k), _f32(v), _f32(S)
    prod = k32[..., :, None] * v32[..., None, :]     # float32 products
    S_new = round_to(S32 + prod, fmt)                # one fp32 addition, then storage rounding
    o = np.einsum("...i,...ij->...j", q32.astype(np.float64), S_new.astype(np.float64))
    return o, S_new

"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic, so the oracle and the CUDA library can both consume
its output without sharing any computation.

Distributions follow the workloads of the method's statement: Q, K ~ N(0,1)/sqrt(d),
V ~ N(0,1), drawn in fp32 and rounded (round-to-nearest-even, by torch's cast)
to the input dtype.  Integer length mixes are uniform over the stated ranges.

``outer_product_state`` draws a random fp32 state with the statistics of a
state that has absorbed L random tokens: the sum of L outer products k v^T of
freshly drawn k, v.  It uses a library matmul (torch, tf32 off) and only
serves as an input recipe (decode starting states and resumed prefix states);
the values it returns are handed to both the oracle and the GPU as inputs.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import torch

_DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32, "f32": torch.float32}


def torch_dtype(dt) -> torch.dtype:
    if isinstance(dt, torch.dtype):
        return dt
    return _DTYPES[dt]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def qkv(shape_qk: Sequence[int], dv: int, dtype="bf16", seed: int = 0,
        device="cpu") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K with shape ``shape_qk`` (last dim d_k) ~ N(0,1)/sqrt(d_k); V ~ N(0,1)
    with the last dim replaced by ``dv``.  Drawn in fp32, cast to ``dtype``."""
    dt = torch_dtype(dtype)
    g = _gen(seed, device)
    dk = int(shape_qk[-1])
    shape_v = tuple(shape_qk[:-1]) + (int(dv),)
    scale = 1.0 / math.sqrt(dk)
    q = (torch.randn(tuple(shape_qk), generator=g, device=device, dtype=torch.float32) * scale).to(dt)
    k = (torch.randn(tuple(shape_qk), generator=g, device=device, dtype=torch.float32) * scale).to(dt)
    v = torch.randn(shape_v, generator=g, device=device, dtype=torch.float32).to(dt)
    return q, k, v


def dense(B: int, H: int, N: int, d: int, dtype="bf16", seed: int = 0, device="cpu", dv: int = None):
    """Dense prefill inputs in layout [B, H, N, d]."""
    return qkv((B, H, N, d), d if dv is None else dv, dtype, seed, device)


def integer_valued(shape: Sequence[int], seed: int = 0, lo: int = -1, hi: int = 1,
                   dtype=torch.float32, device="cpu") -> torch.Tensor:
    """Integers drawn uniformly from [lo, hi], stored exactly in ``dtype``."""
    g = _gen(seed, device)
    return torch.randint(lo, hi + 1, tuple(shape), generator=g, device=device).to(dtype)


def lengths(n: int, lo: int, hi: int, seed: int = 0) -> List[int]:
    """``n`` integers uniform on [lo, hi] (inclusive)."""
    g = _gen(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def cu_seqlens(lens: Sequence[int]) -> torch.Tensor:
    """int32 prefix offsets [0, l0, l0+l1, ...] of a packed ragged batch."""
    out = [0]
    for x in lens:
        out.append(out[-1] + int(x))
    return torch.tensor(out, dtype=torch.int32)


def choose(n: int, m: int, seed: int = 0) -> List[int]:
    """A seeded random subset of ``m`` of the indices 0..n-1, sorted."""
    g = _gen(seed, "cpu")
    return sorted(int(x) for x in torch.randperm(n, generator=g)[:m])


def outer_product_state(units: int, dk: int, dv: int, L: Sequence[int], seed: int = 0,
                        device="cpu", block: int = 4096) -> torch.Tensor:
    """fp32 states [units, dk, dv]: unit u is the sum of L[u] outer products k v^T
    with k ~ N(0,1)/sqrt(dk) and v ~ N(0,1) drawn fresh (bf16-rounded, as
    inputs are).  Accumulated in fp32 blocks of ``block`` tokens on ``device``."""
    assert len(L) == units
    g = _gen(seed, device)
    prev_tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        S = torch.zeros(units, dk, dv, dtype=torch.float32, device=device)
        Lt = torch.tensor([int(x) for x in L], device=device)
        Lmax = int(max(L)) if units else 0
        scale = 1.0 / math.sqrt(dk)
        for t0 in range(0, Lmax, block):
            nb = min(block, Lmax - t0)
            k = (torch.randn(units, nb, dk, generator=g, device=device) * scale).to(torch.bfloat16).float()
            v = torch.randn(units, nb, dv, generator=g, device=device).to(torch.bfloat16).float()
            live = (torch.arange(t0, t0 + nb, device=device)[None, :] < Lt[:, None]).float()
            k = k * live[:, :, None]
            S += torch.bmm(k.transpose(1, 2), v)
        return S
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev_tf32

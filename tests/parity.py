"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (relative Frobenius error per (batch, head) unit, max over units):
  bf16 inputs: O <= 5e-3 and max|O - O_ref| <= 2e-2 * max|O_ref|;
               final state S <= 1e-4 (fp32 accumulation of exact bf16 products)
  fp32 inputs: O and S <= 1e-4
"""
import numpy as np
import torch

BF16_O_REL = 5e-3
BF16_O_MAXABS = 2e-2
STATE_REL = 1e-4
FP32_O_REL = 1e-4


def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def rel_per_unit(got, ref, lead: int) -> np.ndarray:
    """Relative Frobenius error of each unit; ``lead`` leading dims index units."""
    g, r = to64(got), to64(ref)
    U = int(np.prod(g.shape[:lead])) if lead else 1
    g = g.reshape(U, -1)
    r = r.reshape(U, -1)
    num = np.linalg.norm(g - r, axis=1)
    den = np.maximum(np.linalg.norm(r, axis=1), 1e-30)
    return num / den


def assert_out(got, ref, dtype, lead: int, what="O"):
    g, r = to64(got), to64(ref)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    rel = rel_per_unit(g, r, lead)
    if dtype == torch.bfloat16:
        assert rel.max() <= BF16_O_REL, f"{what}: max per-unit rel err {rel.max():.3e} > {BF16_O_REL}"
        scale = np.abs(r).max() if r.size else 0.0
        err = np.abs(g - r).max() if r.size else 0.0
        assert err <= BF16_O_MAXABS * scale + 1e-30, f"{what}: max abs err {err:.3e} > 2e-2 * {scale:.3e}"
    else:
        assert rel.max() <= FP32_O_REL, f"{what}: max per-unit rel err {rel.max():.3e} > {FP32_O_REL}"
    return float(rel.max()) if rel.size else 0.0


def assert_state(got, ref, lead: int, tol=STATE_REL):
    g = to64(got)
    assert np.isfinite(g).all(), "S: non-finite values"
    rel = rel_per_unit(g, ref, lead)
    assert rel.max() <= tol, f"S: max per-unit rel err {rel.max():.3e} > {tol}"
    return float(rel.max()) if rel.size else 0.0


def guarded(shape, dtype, device="cuda", guard=4096):
    """A NaN-filled buffer with a NaN guard region behind it: returns (view, full)."""
    n = int(np.prod(shape)) if len(shape) else 1
    full = torch.full((n + guard,), float("nan"), dtype=dtype, device=device)
    return full[:n].view(shape), full


def assert_guard_intact(full, n):
    tail = full[n:]
    assert torch.isnan(tail.float()).all(), "write past the end of an output buffer"

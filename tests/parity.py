"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances, per (batch, head) unit -- or (sequence, head) unit of a packed
batch -- with the maximum over units required to pass:
  bf16 inputs: O relative Frobenius error <= 5e-3 and
               max|O - O_ref| <= 2e-2 * max|O_ref| (both within the unit);
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


def _check_units(rel, err, scale, dtype, what):
    """rel, err, scale: per-unit relative error, max abs error and max |ref|."""
    if rel.size == 0:
        return 0.0
    worst = int(np.argmax(rel))
    if dtype == torch.bfloat16:
        assert rel.max() <= BF16_O_REL, f"{what}: unit {worst} rel err {rel.max():.3e} > {BF16_O_REL}"
        bad = np.nonzero(err > BF16_O_MAXABS * scale + 1e-30)[0]
        assert bad.size == 0, (f"{what}: unit {int(bad[0])} max abs err {err[bad[0]]:.3e} > "
                               f"2e-2 * {scale[bad[0]]:.3e}")
    else:
        assert rel.max() <= FP32_O_REL, f"{what}: unit {worst} rel err {rel.max():.3e} > {FP32_O_REL}"
    return float(rel.max())


def assert_out(got, ref, dtype, lead: int, what="O"):
    """Outputs of dense units: ``lead`` leading dims index units."""
    g, r = to64(got), to64(ref)
    assert g.shape == r.shape, f"{what}: shape {g.shape} != {r.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    U = int(np.prod(g.shape[:lead])) if lead else 1
    g2, r2 = g.reshape(U, -1), r.reshape(U, -1)
    if g2.shape[1] == 0:
        return 0.0
    rel = np.linalg.norm(g2 - r2, axis=1) / np.maximum(np.linalg.norm(r2, axis=1), 1e-30)
    err = np.abs(g2 - r2).max(axis=1)
    scale = np.abs(r2).max(axis=1)
    return _check_units(rel, err, scale, dtype, what)


def assert_varlen_out(got, ref, cu_seqlens, dtype, what="O"):
    """Outputs of a packed batch [T, H, d]: one unit per (sequence, head);
    empty sequences have no rows and are skipped."""
    g, r = to64(got), to64(ref)
    assert g.shape == r.shape, f"{what}: shape {g.shape} != {r.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    cu = np.asarray(cu_seqlens.cpu() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens, dtype=np.int64)
    starts = cu[:-1][cu[1:] > cu[:-1]]
    if starts.size == 0:
        return 0.0
    d2 = ((g - r) ** 2).sum(axis=2)          # [T, H]
    r2 = (r ** 2).sum(axis=2)
    ea = np.abs(g - r).max(axis=2)
    ra = np.abs(r).max(axis=2)
    rel = np.sqrt(np.add.reduceat(d2, starts, axis=0)) / np.maximum(np.sqrt(np.add.reduceat(r2, starts, axis=0)),
                                                                     1e-30)
    err = np.maximum.reduceat(ea, starts, axis=0)
    scale = np.maximum.reduceat(ra, starts, axis=0)
    return _check_units(rel.ravel(), err.ravel(), scale.ravel(), dtype, what)


def assert_state(got, ref, lead: int, tol=STATE_REL):
    g = to64(got)
    assert np.isfinite(g).all(), "S: non-finite values"
    rel = rel_per_unit(g, ref, lead)
    assert rel.max() <= tol, f"S: unit {int(np.argmax(rel))} rel err {rel.max():.3e} > {tol}"
    return float(rel.max()) if rel.size else 0.0


def guarded(shape, dtype, device="cuda", guard=4096):
    """A NaN-filled buffer with a NaN guard region behind it: returns (view, full)."""
    n = int(np.prod(shape)) if len(shape) else 1
    full = torch.full((n + guard,), float("nan"), dtype=dtype, device=device)
    return full[:n].view(shape), full


def assert_guard_intact(full, n):
    tail = full[n:]
    assert torch.isnan(tail.float()).all(), "write past the end of an output buffer"

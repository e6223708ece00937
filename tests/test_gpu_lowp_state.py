"""Decode with the state stored in bf16 / fp16 / fp8 (updated in fp32), through the C ABI.

Parity: the stored state is a rounding decision taken in fp32 on both sides,
so the GPU state must equal oracle/lowp.py's bit for bit after every step; o
is compared within the bf16 tolerance.  Study: how fast low-precision storage
drifts from the exact recurrence (pages "MiniMax: «Почему M2 …»", section 4,
and "ノーフリーランチ：MiniMax M2…", infrastructure section: the state is
rewritten at every token, so its rounding errors accumulate).
"""
import numpy as np
import pytest
import torch

import synth
from tests.parity import assert_out

pytestmark = pytest.mark.gpu

TORCH_FMT = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16,
             "fp8_e4m3": torch.float8_e4m3fn, "fp8_e5m2": torch.float8_e5m2}


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


@pytest.mark.parametrize("fmt", ["bf16", "fp16", "fp32", "fp8_e4m3", "fp8_e5m2"])
@pytest.mark.parametrize("d", [64, 128])
def test_lowp_state_matches_oracle_bit_for_bit(la, fmt, d):
    from oracle import lowp
    B, H, T = 2, 3, 24
    U = B * H
    L = [2000 + 500 * u for u in range(U)]
    S32 = synth.outer_product_state(U, d, d, L, seed=17).view(B, H, d, d)
    # the stored starting state, rounded by the oracle's rule
    S = torch.from_numpy(lowp.round_to(S32.numpy(), fmt)).to(TORCH_FMT[fmt]).cuda()
    S_ref = S.float().cpu().numpy()
    qs, ks, vs = synth.qkv((T, B, H, d), d, "bf16", seed=19)
    for t in range(T):
        o = la.decode_step(qs[t].cuda(), ks[t].cuda(), vs[t].cuda(), S)
        o_ref, S_ref = lowp.decode_lowp(qs[t], ks[t], vs[t], S_ref, fmt)
        got = S.float().cpu().numpy()
        assert np.array_equal(got, S_ref), f"step {t}: {np.count_nonzero(got != S_ref)} state elements differ"
        assert_out(o.cpu().view(U, d), o_ref.reshape(U, d), torch.bfloat16, 1)
    assert la.device_status() == 0


def test_lowp_state_drift_over_steps(la, oracle_mod):
    """Relative Frobenius error of the stored state against the exact fp64
    recurrence after T steps, from states built from 16K-token prefixes.  fp32
    storage stays at rounding level; fp16, bf16 and the 8-bit formats drift,
    the more the fewer mantissa bits they keep."""
    B, H, d = 4, 8, 128
    U = B * H
    steps = (64, 512, 2048)
    S32 = synth.outer_product_state(U, d, d, [16384] * U, seed=23).view(B, H, d, d)
    exact = S32.double().numpy().reshape(U, d, d)
    states = {f: S32.to(TORCH_FMT[f]).cuda() for f in TORCH_FMT}
    start_err = {f: np.linalg.norm(states[f].double().cpu().numpy().reshape(U, d, d) - exact) /
                 np.linalg.norm(exact) for f in TORCH_FMT}
    qs, ks, vs = synth.qkv((steps[-1], B, H, d), d, "bf16", seed=29)
    err = {f: {} for f in TORCH_FMT}
    for t in range(steps[-1]):
        for f in TORCH_FMT:
            la.decode_step(qs[t].cuda(), ks[t].cuda(), vs[t].cuda(), states[f])
        _, exact = oracle_mod.decode(qs[t].view(U, d), ks[t].view(U, d), vs[t].view(U, d), exact)
        if t + 1 in steps:
            for f in TORCH_FMT:
                got = states[f].double().cpu().numpy().reshape(U, d, d)
                err[f][t + 1] = float(np.linalg.norm(got - exact) / np.linalg.norm(exact))
    assert la.device_status() == 0
    print("\nstate error vs exact after T steps (start: rounding of the initial state)")
    for f in TORCH_FMT:
        print(f"  {f}: start {start_err[f]:.2e}  " + "  ".join(f"T={t}: {err[f][t]:.2e}" for t in steps))
    assert err["fp32"][steps[-1]] < 1e-6
    final = {f: err[f][steps[-1]] for f in TORCH_FMT}
    # fewer mantissa bits, more drift: 23 > 10 > 7 > 3 > 2
    assert final["fp32"] < final["fp16"] < final["bf16"] < final["fp8_e4m3"] < final["fp8_e5m2"]
    # storage rounding accumulates: the drift grows with the number of rewrites
    for f in ("fp16", "bf16"):
        assert err[f][steps[-1]] > err[f][steps[0]] > start_err[f]
    for f in ("fp8_e4m3", "fp8_e5m2"):
        assert err[f][steps[-1]] > err[f][steps[0]]

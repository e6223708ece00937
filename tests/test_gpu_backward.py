"""Gradients of the prefill (la_prefill_backward) against the fp64 oracle's
chain rule through the recurrence (itself pinned to finite differences and to
autograd of the quadratic form in tests/test_oracle.py).  bf16 (d = 128 or
64) runs three tensor-core passes (two of them in reverse token order); fp32
and LA_BACKWARD_SIMT=1 run the same passes on the FFMA kernel."""
import numpy as np
import pytest
import torch

import synth
from tests.parity import assert_out, assert_state, rel_per_unit, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _grad_case(B, H, N, d, dtype, seed, with_states):
    q, k, v = synth.dense(B, H, N, d, dtype, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    dout = (torch.randn(B, H, N, d, generator=g)).to(q.dtype)
    s0 = synth.outer_product_state(B * H, d, d, [200] * (B * H), seed=seed + 2).view(B, H, d, d) if with_states else None
    ds_n = torch.randn(B, H, d, d, generator=g) if with_states else None
    return q, k, v, dout, s0, ds_n


def _check(x_gpu, x_ref, dtype, lead=2):
    # gradients in the input dtype: the output bar for bf16, 1e-4 for fp32
    if dtype == torch.bfloat16:
        assert_out(x_gpu, x_ref, dtype, lead)
    else:
        rel = rel_per_unit(to64(x_gpu), x_ref, lead)
        assert rel.max() <= 1e-4, rel.max()


@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (1, 2, 33), (2, 2, 200), (1, 3, 1000)])
@pytest.mark.parametrize("dtype,d,simt", [("fp32", 64, 0), ("fp32", 128, 0), ("bf16", 128, 0), ("bf16", 128, 1),
                                          ("bf16", 64, 0)])
@pytest.mark.parametrize("with_states", [False, True])
def test_backward_matches_oracle(la, oracle_mod, monkeypatch, B, H, N, dtype, d, simt, with_states):
    if simt:
        monkeypatch.setenv("LA_BACKWARD_SIMT", "1")
    q, k, v, dout, s0, ds_n = _grad_case(B, H, N, d, dtype, seed=N + d + B, with_states=with_states)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(),
                                          None if s0 is None else s0.cuda(), None if ds_n is None else ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        _check(g.cpu(), r, q.dtype)
    assert_state(ds0.cpu(), rs0, 2, tol=1e-4)


def test_backward_empty_sequence(la):
    q = torch.zeros(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")
    ds_n = torch.randn(1, 2, 128, 128, device="cuda")
    dq, dk, dv, ds0 = la.prefill_backward(q, q, q, q, None, ds_n)
    assert dq.shape == (1, 2, 0, 128)
    assert torch.equal(ds0, ds_n)


@pytest.mark.parametrize("B,H,N", [(1, 2, 4096 + 77), (3, 1, 129), (2, 3, 640)])
def test_backward_tc_many_chunks(la, oracle_mod, B, H, N):
    q, k, v, dout, s0, ds_n = _grad_case(B, H, N, 128, "bf16", seed=B + N, with_states=True)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert_out(g.cpu(), r, torch.bfloat16, 2)
    assert_state(ds0.cpu(), rs0, 2, tol=1e-4)


def test_backward_tc_integer_inputs_bit_exact(la, oracle_mod):
    """Inputs in {-1,0,1} (states in [-20, 20]): every product and partial sum
    of the three passes is an integer well inside the range where fp32 and
    bf16(S) are exact, so each gradient equals the bf16 rounding of the exact
    one and dS0 equals it bit for bit."""
    B, H, N, d = 1, 2, 1000, 128
    q, k, v, dout = (synth.integer_valued((B, H, N, d), seed=s, dtype=torch.bfloat16) for s in (11, 12, 13, 14))
    s0 = synth.integer_valued((B, H, d, d), seed=15, lo=-20, hi=20, dtype=torch.float32)
    ds_n = synth.integer_valued((B, H, d, d), seed=16, lo=-20, hi=20, dtype=torch.float32)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert torch.equal(g.cpu(), torch.from_numpy(r).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(ds0.cpu()), rs0)


def test_backward_tc_no_ds0(la, oracle_mod):
    q, k, v, dout, _, _ = _grad_case(1, 2, 300, 128, "bf16", seed=5, with_states=False)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), need_ds0=False)
    torch.cuda.synchronize()
    assert ds0 is None
    rq, rk, rv, _ = oracle_mod.backward(q, k, v, dout)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert_out(g.cpu(), r, torch.bfloat16, 2)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_ffma_integer_inputs_bit_exact(la, oracle_mod, d):
    """fp32 inputs in {-1,0,1} with integer states: the FFMA passes keep every
    product and partial sum exact, so all four gradients equal the oracle's bit
    for bit."""
    B, H, N = 1, 2, 300
    q, k, v, dout = (synth.integer_valued((B, H, N, d), seed=s) for s in (21, 22, 23, 24))
    s0 = synth.integer_valued((B, H, d, d), seed=25, lo=-20, hi=20)
    ds_n = synth.integer_valued((B, H, d, d), seed=26, lo=-20, hi=20)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv), (ds0, rs0)):
        np.testing.assert_array_equal(to64(g.cpu()), r)


@pytest.mark.parametrize("segments,d", [("2", 128), ("3", 128), ("5", 128), ("3", 64)])
def test_backward_tc_segments_match_oracle(la, oracle_mod, monkeypatch, segments, d):
    """Each tensor-core pass cut into segments (state-only pass, prefix or, in
    reverse order, suffix over the segment sums, then all segments)."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    q, k, v, dout, s0, ds_n = _grad_case(1, 2, 3000, d, "bf16", seed=31, with_states=True)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert_out(g.cpu(), r, torch.bfloat16, 2)
    assert_state(ds0.cpu(), rs0, 2, tol=1e-4)


@pytest.mark.parametrize("segments", ["1", "4"])
def test_backward_tc_segments_integer_inputs_bit_exact(la, oracle_mod, monkeypatch, segments):
    """With inputs in {-1,0,1} every sum is exact whatever its order, so the
    segmented passes equal the oracle bit for bit, like the unsplit ones."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    B, H, N, d = 1, 2, 1500, 128
    q, k, v, dout = (synth.integer_valued((B, H, N, d), seed=s, dtype=torch.bfloat16) for s in (41, 42, 43, 44))
    s0 = synth.integer_valued((B, H, d, d), seed=45, lo=-20, hi=20, dtype=torch.float32)
    ds_n = synth.integer_valued((B, H, d, d), seed=46, lo=-20, hi=20, dtype=torch.float32)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert torch.equal(g.cpu(), torch.from_numpy(r).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(ds0.cpu()), rs0)


@pytest.mark.parametrize("segments,d", [("2", 128), ("3", 128), ("3", 64)])
def test_backward_ffma_segments_match_oracle(la, oracle_mod, monkeypatch, segments, d):
    """fp32: each FFMA pass cut into segments (state-only pass, prefix or, in
    reverse order, suffix over the segment sums, then all segments)."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    q, k, v, dout, s0, ds_n = _grad_case(1, 2, 3000, d, "fp32", seed=33, with_states=True)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        _check(g.cpu(), r, q.dtype)
    assert_state(ds0.cpu(), rs0, 2, tol=1e-4)


@pytest.mark.parametrize("segments", ["2", "5"])
def test_backward_ffma_segments_integer_bit_exact(la, oracle_mod, monkeypatch, segments):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    B, H, N, d = 1, 2, 1300, 128
    q, k, v, dout = (synth.integer_valued((B, H, N, d), seed=s) for s in (71, 72, 73, 74))
    s0 = synth.integer_valued((B, H, d, d), seed=75, lo=-20, hi=20)
    ds_n = synth.integer_valued((B, H, d, d), seed=76, lo=-20, hi=20)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for g, r in ((dq, rq), (dk, rk), (dv, rv), (ds0, rs0)):
        np.testing.assert_array_equal(to64(g.cpu()), r)

"""Dense prefill on the GPU against the fp64 oracle (tensor-core bf16 path at
d = 128 and 64, FFMA fp32 path), through the C ABI via the Python binding."""
import numpy as np
import pytest
import torch

import synth
from tests.parity import assert_guard_intact, assert_out, assert_state, guarded, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _state(B, H, d, seed, L=300):
    return synth.outer_product_state(B * H, d, d, [L] * (B * H), seed=seed).view(B, H, d, d)


def _run(la, q, k, v, s0=None, chunk=0):
    B, H, N, d = q.shape
    out, full_o = guarded((B, H, N, d), q.dtype)
    s_out, full_s = guarded((B, H, d, d), torch.float32)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), None if s0 is None else s0.cuda(), chunk=chunk, out=out,
                      s_out=s_out)
    torch.cuda.synchronize()
    assert_guard_intact(full_o, out.numel())
    assert_guard_intact(full_s, s_out.numel())
    assert la.device_status() == 0
    return o.cpu(), s.cpu()


TC_SHAPES = [(1, 1, 1), (1, 2, 5), (1, 2, 127), (1, 2, 128), (1, 1, 129), (2, 3, 300), (1, 2, 1000),
             (2, 2, 4096), (3, 1, 385)]


@pytest.mark.parametrize("B,H,N", TC_SHAPES)
@pytest.mark.parametrize("with_s0", [False, True])
def test_tc_bf16_matches_oracle(la, oracle_mod, B, H, N, with_s0):
    q, k, v = synth.dense(B, H, N, 128, "bf16", seed=B * 1000 + H * 100 + N)
    s0 = _state(B, H, 128, seed=N) if with_s0 else None
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


@pytest.mark.parametrize("chunk", [0, 128])
def test_tc_chunk_argument(la, oracle_mod, chunk):
    q, k, v = synth.dense(1, 2, 700, 128, "bf16", seed=5)
    o, s = _run(la, q, k, v, chunk=chunk)
    ro, rs = oracle_mod.recurrent(q, k, v)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_tc_integer_inputs_bit_exact(la, oracle_mod):
    """Inputs in {-1,0,1}: every product and partial sum on the tensor-core
    path is an exactly representable integer (the running state stays well
    inside |S| <= 256, where bf16(S) is exact; fp32 sums stay below 2^24), so
    O must equal the bf16 rounding of the exact result and S must equal it bit
    for bit."""
    B, H, N, d = 1, 2, 1000, 128
    q = synth.integer_valued((B, H, N, d), seed=1, dtype=torch.bfloat16)
    k = synth.integer_valued((B, H, N, d), seed=2, dtype=torch.bfloat16)
    v = synth.integer_valued((B, H, N, d), seed=3, dtype=torch.bfloat16)
    s0 = synth.integer_valued((B, H, d, d), seed=4, lo=-20, hi=20, dtype=torch.float32)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    want_o = torch.from_numpy(ro).to(torch.bfloat16)
    assert torch.equal(o, want_o)
    np.testing.assert_array_equal(to64(s), rs)


def test_tc_empty_sequence_copies_state(la):
    q = torch.zeros(2, 3, 0, 128, dtype=torch.bfloat16)
    s0 = _state(2, 3, 128, seed=9)
    o, s = _run(la, q, q, q, s0)
    assert o.shape == (2, 3, 0, 128)
    assert torch.equal(s, s0)
    o, s = _run(la, q, q, q, None)
    assert torch.count_nonzero(s) == 0


def test_tc_first_output_invariant(la):
    """o_1 = (q_1 . k_1) v_1 with a zero initial state."""
    q, k, v = synth.dense(2, 4, 64, 128, "bf16", seed=77)
    o, _ = _run(la, q, k, v)
    qd, kd, vd = to64(q[:, :, 0]), to64(k[:, :, 0]), to64(v[:, :, 0])
    want = np.einsum("bhi,bhi->bh", qd, kd)[..., None] * vd
    got = to64(o[:, :, 0])
    assert np.abs(got - want).max() <= 2e-2 * np.abs(want).max()


def test_tc_split_invariance(la, oracle_mod):
    """prefill(0..n) then resume(n..N) from its exported state == prefill(0..N)."""
    q, k, v = synth.dense(1, 2, 900, 128, "bf16", seed=3)
    o, s = _run(la, q, k, v)
    for n in (128, 333):
        oa, sa = _run(la, q[:, :, :n], k[:, :, :n], v[:, :, :n])
        ob, sb = _run(la, q[:, :, n:], k[:, :, n:], v[:, :, n:], sa)
        assert_out(torch.cat([oa, ob], 2), to64(o), torch.bfloat16, 2)
        assert_state(sb, to64(s), 2, tol=1e-5)


@pytest.mark.parametrize("d,chunk", [(64, 64), (64, 32), (128, 64), (128, 32)])
@pytest.mark.parametrize("N", [1, 63, 256, 300])
def test_fp32_matches_oracle(la, oracle_mod, d, chunk, N):
    q, k, v = synth.dense(1, 2, N, d, "fp32", seed=N + d)
    s0 = _state(1, 2, d, seed=1) if N == 300 else None
    o, s = _run(la, q, k, v, s0, chunk=chunk)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.float32, 2)
    assert_state(s, rs, 2)


def test_fp32_small_config_exact_shape(la, oracle_mod):
    """B=1, H=2, N=256, d=64, fp32, chunk 64, zero initial state: final state
    relative error <= 1e-4 (both against the recurrence and the quadratic form)."""
    q, k, v = synth.dense(1, 2, 256, 64, "fp32", seed=1)
    o, s = _run(la, q, k, v, None, chunk=64)
    ro, rs = oracle_mod.recurrent(q, k, v)
    qo, qs = oracle_mod.quadratic(q, k, v)
    for ref_o, ref_s in ((ro, rs), (qo, qs)):
        assert_out(o, ref_o, torch.float32, 2)
        assert_state(s, ref_s, 2)


def test_fp32_integer_inputs_bit_exact(la, oracle_mod):
    q = synth.integer_valued((1, 2, 64, 64), seed=5)
    k = synth.integer_valued((1, 2, 64, 64), seed=6)
    v = synth.integer_valued((1, 2, 64, 64), seed=7)
    o, s = _run(la, q, k, v, chunk=64)
    ro, rs = oracle_mod.recurrent(q, k, v)
    np.testing.assert_array_equal(to64(o), ro)
    np.testing.assert_array_equal(to64(s), rs)


@pytest.mark.parametrize("N", [1, 100, 257])
def test_bf16_d64_matches_oracle(la, oracle_mod, N):
    q, k, v = synth.dense(2, 2, N, 64, "bf16", seed=N)
    s0 = _state(2, 2, 64, seed=2)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_unsupported_chunk_raises(la):
    q, k, v = synth.dense(1, 1, 10, 128, "bf16", seed=0)
    with pytest.raises(la.LAError):
        la.prefill(q.cuda(), k.cuda(), v.cuda(), chunk=48)


def test_tc_many_units_per_cta(la, oracle_mod):
    """512 (batch, head) units = 1024 items on the persistent grid (about 7
    items per CTA, boustrophedon order), each with a ragged last chunk and its
    own initial state; a sample of units against the oracle."""
    B, H, N = 32, 16, 200
    q, k, v = synth.dense(B, H, N, 128, "bf16", seed=71)
    s0 = _state(B, H, 128, seed=72, L=100)
    o, s = _run(la, q, k, v, s0)
    units = synth.choose(B * H, 24, seed=73)
    qf, kf, vf, of, sf, s0f = (x.reshape(B * H, *x.shape[2:]) for x in (q, k, v, o, s, s0))
    idx = torch.tensor(units)
    ro, rs = oracle_mod.recurrent(qf[idx], kf[idx], vf[idx], s0f[idx])
    assert_out(of[idx], ro, torch.bfloat16, 1)
    assert_state(sf[idx], rs, 1)


@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (2, 3, 300), (1, 2, 1000), (3, 1, 4096 + 5)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_tc_d64_matches_oracle(la, oracle_mod, B, H, N, with_s0):
    """d = 64 on the tensor cores: one 64-column panel, one value slice per
    head, the K^T V product's second half a copy of the first."""
    q, k, v = synth.dense(B, H, N, 64, "bf16", seed=B * 7 + H + N)
    s0 = _state(B, H, 64, seed=N) if with_s0 else None
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_tc_d64_integer_inputs_bit_exact(la, oracle_mod):
    B, H, N, d = 2, 2, 1000, 64
    q = synth.integer_valued((B, H, N, d), seed=51, dtype=torch.bfloat16)
    k = synth.integer_valued((B, H, N, d), seed=52, dtype=torch.bfloat16)
    v = synth.integer_valued((B, H, N, d), seed=53, dtype=torch.bfloat16)
    s0 = synth.integer_valued((B, H, d, d), seed=54, lo=-20, hi=20, dtype=torch.float32)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert torch.equal(o, torch.from_numpy(ro).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(s), rs)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("chunk", [32, 64])
def test_bf16_small_chunks_match_oracle(la, oracle_mod, d, chunk):
    """bf16 with 32- or 64-token chunks runs on the FFMA kernel (the tensor-core
    tiles are 128 tokens long); the chunk length does not change the result
    beyond rounding, so the bars are the same."""
    q, k, v = synth.dense(2, 2, 300, d, "bf16", seed=d + chunk)
    s0 = _state(2, 2, d, seed=chunk)
    o, s = _run(la, q, k, v, s0, chunk=chunk)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_bf16_chunk64_varlen_matches_oracle(la, oracle_mod):
    lens = [300, 0, 1, 129, 64]
    cu = synth.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 2, 128
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=7)
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), chunk=64)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.varlen(q, k, v, cu)
    from tests.parity import assert_varlen_out
    assert_varlen_out(o.cpu(), ro, cu, torch.bfloat16)
    assert_state(s.cpu(), rs, 2)

"""Packed ragged prefill with prefix resume on the GPU against the fp64 oracle."""

import numpy as np
import pytest
import torch

import synth
from tests.parity import assert_guard_intact, assert_out, assert_state, assert_varlen_out, guarded, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _case(lens, H, d, dtype, seed, n_pool=3, resume=None):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, d), d, dtype, seed=seed)
    pool = synth.outer_product_state(n_pool * H, d, d, [400] * (n_pool * H), seed=seed + 1).view(n_pool, H, d, d)
    if resume is None:
        resume = [(i % (n_pool + 1)) - 1 for i in range(len(lens))]
    idx = torch.tensor(resume, dtype=torch.int32)
    return cu, q, k, v, pool, idx


def _run(la, cu, q, k, v, pool, idx, chunk=0):
    T, H, d = q.shape
    n = cu.numel() - 1
    out, full_o = guarded((T, H, d), q.dtype)
    s_out, full_s = guarded((n, H, d, d), torch.float32)
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), idx.cuda(), chunk=chunk,
                             out=out, s_out=s_out)
    torch.cuda.synchronize()
    assert_guard_intact(full_o, out.numel())
    assert_guard_intact(full_s, s_out.numel())
    assert la.device_status() == 0
    return o.cpu(), s.cpu()


LENS = [
    [300, 0, 1, 128, 129, 1000, 5, 256],
    [127, 2, 640],
    [4096, 1, 77],
]


@pytest.mark.parametrize("lens", LENS)
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 128)])
def test_varlen_matches_oracle(la, oracle_mod, lens, dtype, d):
    cu, q, k, v, pool, idx = _case(lens, 3, d, dtype, seed=sum(lens) + d)
    o, s = _run(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    dt = synth.torch_dtype(dtype)
    assert_varlen_out(o, ro, cu, dt)
    assert_state(s, rs, 2)


def test_varlen_zero_length_copies_initial_state(la, oracle_mod):
    cu, q, k, v, pool, idx = _case([0, 10, 0], 2, 128, "bf16", seed=4, resume=[1, -1, -1])
    o, s = _run(la, cu, q, k, v, pool, idx)
    assert torch.equal(s[0], pool[1])
    assert torch.count_nonzero(s[2]) == 0


def test_varlen_equals_dense_loop(la):
    """A packed batch equals one dense prefill call per sequence."""
    lens = [513, 200, 1]
    H, d = 2, 128
    cu, q, k, v, pool, idx = _case(lens, H, d, "bf16", seed=12)
    o, s = _run(la, cu, q, k, v, pool, idx)
    for n, L in enumerate(lens):
        a, b = int(cu[n]), int(cu[n + 1])
        s0 = pool[idx[n]].unsqueeze(0).cuda() if idx[n] >= 0 else None
        qd = q[a:b].transpose(0, 1).unsqueeze(0).contiguous().cuda()
        kd = k[a:b].transpose(0, 1).unsqueeze(0).contiguous().cuda()
        vd = v[a:b].transpose(0, 1).unsqueeze(0).contiguous().cuda()
        od, sd = la.prefill(qd, kd, vd, s0)
        assert_out(o[a:b].transpose(0, 1), to64(od[0]), torch.bfloat16, 1)
        assert_state(s[n], to64(sd[0]), 1, tol=1e-5)


def test_varlen_validation_rejects_bad_offsets(la, monkeypatch):
    monkeypatch.setenv("LA_VALIDATE", "1")
    cu, q, k, v, pool, idx = _case([10, 20], 1, 128, "bf16", seed=1)
    bad = torch.tensor([0, 25, 20], dtype=torch.int32)
    with pytest.raises(la.LAError):
        la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), bad.cuda(), pool.cuda(), idx.cuda())
    bad_idx = torch.tensor([0, 7], dtype=torch.int32)
    with pytest.raises(la.LAError):
        la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), bad_idx.cuda())
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), idx.cuda())
    torch.cuda.synchronize()


@pytest.mark.parametrize("n_seq", [4096, 5000])
def test_varlen_many_short_sequences(la, oracle_mod, n_seq):
    """The largest batch the device sort orders longest-first (4096), and one
    beyond it (kept in its own order); lengths 0 .. 24, a third resumed."""
    rng = np.random.default_rng(n_seq)
    lens = [int(x) for x in rng.integers(0, 25, n_seq)]
    resume = [int(x) for x in rng.integers(-1, 3, n_seq)]
    cu, q, k, v, pool, idx = _case(lens, 2, 128, "bf16", seed=9, n_pool=3, resume=resume)
    o, s = _run(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert_varlen_out(o, ro, cu, torch.bfloat16)
    assert_state(s, rs, 2)


@pytest.mark.parametrize("segments", ["2", "3", "7"])
@pytest.mark.parametrize("d", [128, 64])
def test_varlen_segments_match_oracle(la, oracle_mod, monkeypatch, segments, d):
    """A packed batch cut into segments (LA_PREFILL_SEGMENTS forces about that
    many per sequence of average length): the sums of all but each sequence's
    last segment, per-sequence prefix states from the pool, then all segments.
    Lengths include an empty sequence, a one-token one and ragged tails."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    lens = [1500, 0, 1, 700, 3000, 129]
    cu, q, k, v, pool, idx = _case(lens, 3, d, "bf16", seed=61, n_pool=2, resume=[0, 1, -1, 1, -1, 0])
    o, s = _run(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert_varlen_out(o, ro, cu, torch.bfloat16)
    assert_state(s, rs, 2)


def test_varlen_segments_automatic(la, oracle_mod):
    """Two long sequences with two heads fill 8 of the SMs unsplit: the library
    cuts them into segments by itself."""
    lens = [9000, 5000]
    cu, q, k, v, pool, idx = _case(lens, 2, 128, "bf16", seed=63, n_pool=1, resume=[0, -1])
    assert la.prefill_varlen_workspace_size(2, sum(lens), 2, 128, torch.bfloat16) > 4 * 256
    o, s = _run(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert_varlen_out(o, ro, cu, torch.bfloat16)
    assert_state(s, rs, 2)


@pytest.mark.parametrize("segments", ["1", "4"])
def test_varlen_segments_integer_inputs_bit_exact(la, oracle_mod, monkeypatch, segments):
    """Inputs in {-1,0,1} with integer pool states: every partial sum is exact,
    so the split and unsplit runs both equal the oracle bit for bit."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    lens = [1000, 3, 600, 0, 257]
    cu = synth.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 2, 128
    q, k, v = (synth.integer_valued((T, H, d), seed=s, dtype=torch.bfloat16) for s in (71, 72, 73))
    pool = synth.integer_valued((2, H, d, d), seed=74, lo=-20, hi=20, dtype=torch.float32)
    idx = torch.tensor([1, -1, 0, 0, -1], dtype=torch.int32)
    o, s = _run(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert torch.equal(o, torch.from_numpy(ro).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(s), rs)

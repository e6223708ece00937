"""The full-width tensor-core prefill (one CTA per head over all 128 value
columns) against the fp64 oracle.

The library takes this kernel by itself once a batch's heads fill the GPU
(more than half as many heads as SMs at d = 128); LA_PREFILL_WIDE=1 forces it
for the small cases below, LA_PREFILL_WIDE=0 forces the value-split kernel,
and the two must agree.  Dense and packed batches, ragged tails, resumed
states, feature maps, the backward's reverse passes and more heads than SMs
(several heads per CTA on the persistent grid) are covered, and integer
inputs must come out bit-exact as on the value-split kernel.
"""
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


@pytest.fixture
def wide(monkeypatch):
    monkeypatch.setenv("LA_PREFILL_WIDE", "1")


def _state(B, H, d, seed, L=300):
    return synth.outer_product_state(B * H, d, d, [L] * (B * H), seed=seed).view(B, H, d, d)


def _run(la, q, k, v, s0=None, phi="identity"):
    B, H, N, d = q.shape
    out, full_o = guarded((B, H, N, d), q.dtype)
    s_out, full_s = guarded((B, H, d, d), torch.float32)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), None if s0 is None else s0.cuda(), out=out, s_out=s_out, phi=phi)
    torch.cuda.synchronize()
    assert_guard_intact(full_o, out.numel())
    assert_guard_intact(full_s, s_out.numel())
    assert la.device_status() == 0
    return o.cpu(), s.cpu()


SHAPES = [(1, 1, 1), (1, 2, 5), (1, 2, 127), (1, 2, 128), (1, 1, 129), (2, 3, 300), (1, 2, 1000), (2, 2, 4096),
          (3, 1, 385)]


@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("with_s0", [False, True])
def test_wide_matches_oracle(la, oracle_mod, wide, B, H, N, with_s0):
    q, k, v = synth.dense(B, H, N, 128, "bf16", seed=B * 1000 + H * 100 + N + 7)
    s0 = _state(B, H, 128, seed=N + 3) if with_s0 else None
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_wide_integer_inputs_bit_exact(la, oracle_mod, wide):
    """Inputs in {-1,0,1} and an integer initial state: every product and
    partial sum is an exact integer and bf16(S) is exact (|S| <= 256), so O is
    the bf16 rounding of the exact result and S equals it bit for bit."""
    B, H, N, d = 1, 2, 1000, 128
    q, k, v = (synth.integer_valued((B, H, N, d), seed=s, dtype=torch.bfloat16) for s in (11, 12, 13))
    s0 = synth.integer_valued((B, H, d, d), seed=14, lo=-20, hi=20, dtype=torch.float32)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert torch.equal(o, torch.from_numpy(ro).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(s), rs)


def test_wide_and_value_split_agree(la, monkeypatch):
    """Both kernels on the same batch: equal within the output's rounding, and
    the final states within fp32 summation order."""
    q, k, v = synth.dense(2, 3, 1500, 128, "bf16", seed=21, device="cuda")
    s0 = _state(2, 3, 128, seed=22).cuda()
    monkeypatch.setenv("LA_PREFILL_WIDE", "1")
    o1, s1 = la.prefill(q, k, v, s0)
    monkeypatch.setenv("LA_PREFILL_WIDE", "0")
    o2, s2 = la.prefill(q, k, v, s0)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert_out(o1.cpu(), to64(o2), torch.bfloat16, 2)
    assert_state(s1.cpu(), to64(s2), 2, tol=1e-6)


def test_wide_chosen_for_many_heads(la, oracle_mod):
    """B=1, H=80: 160 value-slice items would need two waves on 148 SMs, so
    the library takes the full-width kernel by itself (80 CTAs)."""
    q, k, v = synth.dense(1, 80, 700, 128, "bf16", seed=31)
    o, s = _run(la, q, k, v)
    ro, rs = oracle_mod.recurrent(q, k, v)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_wide_more_heads_than_sms(la, oracle_mod):
    """400 heads on the persistent grid (two or three per CTA, boustrophedon
    order), each with a ragged last chunk and its own initial state: every
    unit against the oracle."""
    B, H, N = 4, 100, 200
    q, k, v = synth.dense(B, H, N, 128, "bf16", seed=41)
    s0 = _state(B, H, 128, seed=42, L=100)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_wide_empty_sequence_copies_state(la, wide):
    q = torch.zeros(2, 3, 0, 128, dtype=torch.bfloat16)
    s0 = _state(2, 3, 128, seed=9)
    o, s = la.prefill(q.cuda(), q.cuda(), q.cuda(), s0.cuda())
    torch.cuda.synchronize()
    assert o.numel() == 0
    assert torch.equal(s.cpu(), s0)


# ---------------------------------------------------------------- packed batches
def _packed(lens, H, seed, n_pool=2, resume=None):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, 128), 128, "bf16", seed=seed)
    pool = synth.outer_product_state(n_pool * H, 128, 128, [400] * (n_pool * H), seed=seed + 1).view(n_pool, H, 128, 128)
    if resume is None:
        resume = [(i % (n_pool + 1)) - 1 for i in range(len(lens))]
    return cu, q, k, v, pool, torch.tensor(resume, dtype=torch.int32)


def _run_packed(la, cu, q, k, v, pool, idx, phi="identity"):
    T, H, d = q.shape
    n = cu.numel() - 1
    out, full_o = guarded((T, H, d), q.dtype)
    s_out, full_s = guarded((n, H, d, d), torch.float32)
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), idx.cuda(), out=out, s_out=s_out,
                             phi=phi)
    torch.cuda.synchronize()
    assert_guard_intact(full_o, out.numel())
    assert_guard_intact(full_s, s_out.numel())
    assert la.device_status() == 0
    return o.cpu(), s.cpu()


@pytest.mark.parametrize("lens", [[300, 0, 1, 128, 129, 1000, 5, 256], [127, 2, 640], [4096, 1, 77]])
def test_wide_varlen_matches_oracle(la, oracle_mod, wide, lens):
    cu, q, k, v, pool, idx = _packed(lens, 3, seed=sum(lens) + 5)
    o, s = _run_packed(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert_varlen_out(o, ro, cu, torch.bfloat16)
    assert_state(s, rs, 2)


def test_wide_varlen_many_short_sequences(la, oracle_mod):
    """4096 sequences of 0 .. 24 tokens, 2 heads (8192 heads: the library's own
    choice is the full-width kernel), a third of them resumed."""
    rng = np.random.default_rng(77)
    n_seq = 4096
    lens = [int(x) for x in rng.integers(0, 25, n_seq)]
    resume = [int(x) for x in rng.integers(-1, 3, n_seq)]
    cu, q, k, v, pool, idx = _packed(lens, 2, seed=78, n_pool=3, resume=resume)
    o, s = _run_packed(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert_varlen_out(o, ro, cu, torch.bfloat16)
    assert_state(s, rs, 2)


def test_wide_varlen_integer_inputs_bit_exact(la, oracle_mod, wide):
    lens = [1000, 3, 600, 0, 257]
    cu = synth.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 2, 128
    q, k, v = (synth.integer_valued((T, H, d), seed=s, dtype=torch.bfloat16) for s in (81, 82, 83))
    pool = synth.integer_valued((2, H, d, d), seed=84, lo=-20, hi=20, dtype=torch.float32)
    idx = torch.tensor([1, -1, 0, 0, -1], dtype=torch.int32)
    o, s = _run_packed(la, cu, q, k, v, pool, idx)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert torch.equal(o, torch.from_numpy(ro).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(s), rs)


# ---------------------------------------------------------------- feature maps
TC_STATE_TOL = {"identity": 1e-4, "relu": 1e-4, "elu1": 5e-3}


@pytest.mark.parametrize("phi", ["relu", "elu1"])
def test_wide_prefill_with_phi(la, oracle_mod, wide, phi):
    q, k, v = synth.dense(2, 2, 700, 128, "bf16", seed=51)
    o, s = _run(la, q, k, v, phi=phi)
    ro, rs = oracle_mod.recurrent(q, k, v, phi=phi)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2, tol=TC_STATE_TOL[phi])


def test_wide_relu_in_kernel_equals_identity_on_mapped_inputs(la, wide):
    """relu of a bf16 value is exact: mapping the tiles in the kernel must give
    exactly the identity prefill of relu(q), relu(k)."""
    q, k, v = synth.dense(2, 3, 1500, 128, "bf16", seed=93, device="cuda")
    o1, s1 = la.prefill(q, k, v, phi="relu")
    o2, s2 = la.prefill(torch.relu(q), torch.relu(k), v)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


def test_wide_elu1_in_kernel_equals_prepass(la, wide, monkeypatch):
    """elu + 1 mapped by the kernel (no workspace) and by the pre-pass
    (workspace given, the pre-pass forced on the full-width kernel) round phi
    to bf16 the same way: bit-identical."""
    monkeypatch.setenv("LA_PHI_PREPASS", "1")
    B, H, N, d = 1, 2, 3000, 128
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=95, device="cuda")
    ws = torch.empty(la.prefill_workspace_size(B, H, N, d, torch.bfloat16, "elu1"), dtype=torch.uint8,
                     device="cuda")
    outs = []
    for w in (ws, None):
        o = torch.empty_like(v)
        s = torch.empty(B, H, d, d, dtype=torch.float32, device="cuda")
        st = la.lib.la_prefill_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None, s.data_ptr(), B, H,
                                  N, d, d, 0, 0, la.PHI["elu1"], None if w is None else w.data_ptr(),
                                  0 if w is None else w.numel(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, la.lib.la_last_error()
        outs.append((o, s))
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])


def test_wide_elu1_needs_no_prepass_workspace(la):
    """Shapes that run on the full-width kernel map elu + 1 in the kernel and
    ask for no room for mapped copies of q and k."""
    args = (4, 32, 8192, 128, torch.bfloat16)
    assert la.prefill_workspace_size(*args, "elu1") == la.prefill_workspace_size(*args)
    assert la.prefill_varlen_workspace_size(64, 64 * 1000, 32, 128, torch.bfloat16, "elu1") == \
        la.prefill_varlen_workspace_size(64, 64 * 1000, 32, 128, torch.bfloat16)
    # two heads run on the value split, where the pre-pass pays
    assert la.prefill_workspace_size(1, 2, 3000, 128, torch.bfloat16, "elu1") > \
        la.prefill_workspace_size(1, 2, 3000, 128, torch.bfloat16)


@pytest.mark.parametrize("phi", ["relu", "elu1"])
def test_wide_varlen_with_phi(la, oracle_mod, wide, phi):
    lens = [0, 1, 130, 257, 1000]
    cu, q, k, v, pool, idx = _packed(lens, 2, seed=55)
    o, s = _run_packed(la, cu, q, k, v, pool, idx, phi=phi)
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx, phi=phi)
    assert_varlen_out(o, ro, cu, torch.bfloat16)
    assert_state(s, rs, 2, tol=TC_STATE_TOL[phi])


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (1, 2, 33), (2, 2, 200), (1, 3, 1000)])
@pytest.mark.parametrize("with_states", [False, True])
def test_wide_backward_matches_oracle(la, oracle_mod, wide, B, H, N, with_states):
    d = 128
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=B * 100 + N)
    g = torch.Generator().manual_seed(N + 1)
    dout = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    s0 = _state(B, H, d, seed=N + 2, L=200) if with_states else None
    ds_n = torch.randn(B, H, d, d, generator=g) if with_states else None
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(),
                                          None if s0 is None else s0.cuda(), None if ds_n is None else ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, dout, s0, ds_n)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert_out(got.cpu(), ref, torch.bfloat16, 2)
    assert_state(ds0.cpu(), rs0, 2)


def test_wide_backward_integer_inputs_bit_exact(la, oracle_mod, wide):
    B, H, N, d = 1, 2, 700, 128
    q, k, v, do = (synth.integer_valued((B, H, N, d), seed=s, dtype=torch.bfloat16) for s in (61, 62, 63, 64))
    s0 = synth.integer_valued((B, H, d, d), seed=65, lo=-8, hi=8, dtype=torch.float32)
    ds_n = synth.integer_valued((B, H, d, d), seed=66, lo=-8, hi=8, dtype=torch.float32)
    dq, dk, dv, ds0 = la.prefill_backward(q.cuda(), k.cuda(), v.cuda(), do.cuda(), s0.cuda(), ds_n.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    rq, rk, rv, rs0 = oracle_mod.backward(q, k, v, do, s0, ds_n)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert torch.equal(got.cpu(), torch.from_numpy(ref).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(ds0.cpu()), rs0)

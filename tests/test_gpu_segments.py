"""Segment split of the dense tensor-core prefill (few units, long sequences).

The sequence of each unit is cut into segments of whole chunks; a state-only
pass sums K^T V per segment, a prefix kernel forms the state before every
segment, and the main pass runs all segments from those states.  The result is
the same recurrence (page "MiniMax-M1で理解する…", section
"線形アテンションの数学的基礎"), so every case is checked against the fp64
oracle, and inputs whose every partial sum is an exact integer must agree bit
for bit whatever the segment count.
"""
import ctypes

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


def _run(la, q, k, v, s0=None):
    B, H, N, d = q.shape
    out, full_o = guarded((B, H, N, d), q.dtype)
    s_out, full_s = guarded((B, H, d, d), torch.float32)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), None if s0 is None else s0.cuda(), out=out, s_out=s_out)
    torch.cuda.synchronize()
    assert_guard_intact(full_o, out.numel())
    assert_guard_intact(full_s, s_out.numel())
    assert la.device_status() == 0
    return o.cpu(), s.cpu()


def _state(B, H, d, seed, L=300):
    return synth.outer_product_state(B * H, d, d, [L] * (B * H), seed=seed).view(B, H, d, d)


@pytest.mark.parametrize("B,H,N", [(1, 1, 20000), (1, 2, 9000), (2, 1, 4096 + 77)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_auto_segments_match_oracle(la, oracle_mod, B, H, N, with_s0):
    assert la.prefill_workspace_size(B, H, N, 128, torch.bfloat16) > 0, "shape should be split"
    q, k, v = synth.dense(B, H, N, 128, "bf16", seed=7 * N + B + H)
    s0 = _state(B, H, 128, seed=N) if with_s0 else None
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


@pytest.mark.parametrize("segments", ["1", "2", "3", "7", "40"])
def test_forced_segment_counts(la, oracle_mod, monkeypatch, segments):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    q, k, v = synth.dense(1, 2, 5000, 128, "bf16", seed=11)
    s0 = _state(1, 2, 128, seed=12)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


@pytest.mark.parametrize("segments", ["1", "4", "9"])
def test_segments_integer_inputs_bit_exact(la, oracle_mod, monkeypatch, segments):
    """Inputs in {-1,0,1} and an integer S0: every product and partial sum is an
    exact integer (|S| stays well inside the range where bf16(S) is exact), so
    the split must not change a single bit."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    B, H, N, d = 1, 2, 1500, 128
    q = synth.integer_valued((B, H, N, d), seed=21, dtype=torch.bfloat16)
    k = synth.integer_valued((B, H, N, d), seed=22, dtype=torch.bfloat16)
    v = synth.integer_valued((B, H, N, d), seed=23, dtype=torch.bfloat16)
    s0 = synth.integer_valued((B, H, d, d), seed=24, lo=-20, hi=20, dtype=torch.float32)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert torch.equal(o, torch.from_numpy(ro).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(s), rs)


def test_without_workspace_runs_unsplit(la, oracle_mod):
    """A caller that passes no workspace gets the one-pass sweep (same result)."""
    B, H, N, d = 1, 1, 6000, 128
    assert la.prefill_workspace_size(B, H, N, d, torch.bfloat16) > 0
    q, k, v = (x.cuda() for x in synth.dense(B, H, N, d, "bf16", seed=31))
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device="cuda")
    st = la.lib.la_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None, s.data_ptr(), B, H, N, d,
                           d, 0, 0, None, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q.cpu(), k.cpu(), v.cpu())
    assert_out(o.cpu(), ro, torch.bfloat16, 2)
    assert_state(s.cpu(), rs, 2)


def test_workspace_size_follows_the_plan(la):
    # 64 heads fill the GPU: no split, no workspace
    assert la.prefill_workspace_size(1, 64, 131072, 128, torch.bfloat16) == 0
    # short sequences are never split
    assert la.prefill_workspace_size(1, 1, 512, 128, torch.bfloat16) == 0
    # one head over 64K tokens: (2P - 1) fp32 states of 128 x 128
    n = la.prefill_workspace_size(1, 1, 65536, 128, torch.bfloat16)
    assert n > 0 and n % (128 * 128 * 4) == 0 and (n // (128 * 128 * 4)) % 2 == 1


@pytest.mark.parametrize("segments", ["1", "3"])
def test_segments_d64(la, oracle_mod, monkeypatch, segments):
    """The segment split at d = 64 (one value slice per unit)."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    q, k, v = synth.dense(1, 2, 5000, 64, "bf16", seed=91)
    s0 = _state(1, 2, 64, seed=92)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


# ---------------------------------------------------------------- FFMA path
# fp32 inputs run on the FFMA prefill, one CTA per (unit, segment); the same
# split applies when the units fill less than half of the SMs.

@pytest.mark.parametrize("B,H,N", [(1, 1, 9000), (1, 2, 5000 + 77)])
@pytest.mark.parametrize("d", [128, 64])
def test_ffma_auto_segments_match_oracle(la, oracle_mod, B, H, N, d):
    assert la.prefill_workspace_size(B, H, N, d, torch.float32) > 0, "shape should be split"
    q, k, v = synth.dense(B, H, N, d, "fp32", seed=3 * N + d)
    s0 = _state(B, H, d, seed=N + 1)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o, ro, torch.float32, 2)
    assert_state(s, rs, 2)


@pytest.mark.parametrize("segments", ["2", "3", "7"])
@pytest.mark.parametrize("chunk", [0, 32])
def test_ffma_forced_segments(la, oracle_mod, monkeypatch, segments, chunk):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    q, k, v = synth.dense(1, 2, 3000, 128, "fp32", seed=41)
    s0 = _state(1, 2, 128, seed=42)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), s0.cuda(), chunk=chunk)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o.cpu(), ro, torch.float32, 2)
    assert_state(s.cpu(), rs, 2)


@pytest.mark.parametrize("segments", ["1", "4", "9"])
@pytest.mark.parametrize("d", [128, 64])
def test_ffma_segments_integer_inputs_bit_exact(la, oracle_mod, monkeypatch, segments, d):
    """Inputs in {-1,0,1} and an integer S0 keep every fp32 product and partial
    sum exact, so the split must not change a single bit."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    B, H, N = 1, 2, 1500
    q, k, v = (synth.integer_valued((B, H, N, d), seed=s) for s in (51, 52, 53))
    s0 = synth.integer_valued((B, H, d, d), seed=54, lo=-20, hi=20)
    o, s = _run(la, q, k, v, s0)
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    np.testing.assert_array_equal(to64(o), ro)
    np.testing.assert_array_equal(to64(s), rs)


@pytest.mark.parametrize("phi", ["elu1", "relu"])
def test_ffma_segments_with_phi(la, oracle_mod, monkeypatch, phi):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", "3")
    q, k, v = synth.dense(1, 2, 2500, 128, "fp32", seed=61)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, phi=phi)
    assert_out(o.cpu(), ro, torch.float32, 2)
    assert_state(s.cpu(), rs, 2)


@pytest.mark.parametrize("N,chunk", [(256, 64), (256, 32), (100, 32), (64 + 5, 64), (64, 64), (1, 32)])
@pytest.mark.parametrize("d", [64, 128])
def test_ffma_short_sequences_split_by_chunk(la, oracle_mod, N, chunk, d):
    """Short sequences on few units are cut into segments of whole FFMA chunks
    (one chunk each at the least), from the given start state; ragged tails
    included."""
    B, H = 1, 2
    q, k, v = synth.dense(B, H, N, d, "fp32", seed=N + chunk + d)
    s0 = _state(B, H, d, seed=N + 3)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), s0.cuda(), chunk=chunk)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    assert_out(o.cpu(), ro, torch.float32, 2)
    assert_state(s.cpu(), rs, 2)


@pytest.mark.parametrize("chunk", [32, 64])
@pytest.mark.parametrize("segments", [None, "1"])
def test_ffma_short_sequences_integer_inputs_bit_exact(la, oracle_mod, monkeypatch, chunk, segments):
    """The chunk-sized segments of a short sequence, and the unsplit run, give
    the oracle's result bit for bit on integer-valued inputs."""
    if segments:
        monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    B, H, N, d = 1, 2, 256 + 17, 64
    q, k, v = (synth.integer_valued((B, H, N, d), seed=s) for s in (71, 72, 73))
    s0 = synth.integer_valued((B, H, d, d), seed=74, lo=-20, hi=20)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), s0.cuda(), chunk=chunk)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, s0)
    np.testing.assert_array_equal(to64(o.cpu()), ro)
    np.testing.assert_array_equal(to64(s.cpu()), rs)


def test_ffma_workspace_size_follows_the_plan(la):
    # one item per unit on the FFMA path: 128 units fill the GPU, 8 do not
    assert la.prefill_workspace_size(1, 128, 65536, 128, torch.float32) == 0
    n = la.prefill_workspace_size(1, 8, 65536, 128, torch.float32)
    assert n > 0 and n % (8 * 128 * 128 * 4) == 0
    # a short sequence on few units is split too (segments of whole FFMA chunks)
    assert la.prefill_workspace_size(1, 2, 256, 64, torch.float32) > 0


def _varlen_case(lens, H, d, seed, dtype="fp32", n_pool=2):
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, d), d, dtype, seed=seed)
    pool = synth.outer_product_state(n_pool * H, d, d, [300] * (n_pool * H), seed=seed + 1).view(n_pool, H, d, d)
    init = torch.tensor([(i % (n_pool + 1)) - 1 for i in range(len(lens))], dtype=torch.int32)
    return cu, q, k, v, pool, init


@pytest.mark.parametrize("lens,H,d", [([9000, 1, 0, 3000], 2, 128), ([20000], 1, 64), ([5000, 7000], 3, 128)])
def test_ffma_varlen_auto_segments_match_oracle(la, oracle_mod, lens, H, d):
    """A packed fp32 batch of few long sequences: one CTA per (segment, head)."""
    cu, q, k, v, pool, init = _varlen_case(lens, H, d, seed=sum(lens) % 97 + d)
    T = int(cu[-1])
    base = la.prefill_varlen_workspace_size(len(lens), T, H, d, torch.float32)
    assert base >= H * d * d * 4, "shape should be split (the workspace holds segment states)"
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), init.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, init)
    assert_out(o.cpu(), ro, torch.float32, 2)
    assert_state(s.cpu(), rs, 1)


@pytest.mark.parametrize("segments", ["2", "5"])
def test_ffma_varlen_forced_segments_integer_bit_exact(la, oracle_mod, monkeypatch, segments):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    lens, H, d = [1500, 0, 700, 1], 2, 128
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    T = int(cu[-1])
    q, k, v = (synth.integer_valued((T, H, d), seed=s) for s in (81, 82, 83))
    pool = synth.integer_valued((2, H, d, d), seed=84, lo=-20, hi=20)
    init = torch.tensor([1, 0, -1, 1], dtype=torch.int32)
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), init.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, init)
    np.testing.assert_array_equal(to64(o.cpu()), ro)
    np.testing.assert_array_equal(to64(s.cpu()), rs)

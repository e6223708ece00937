"""la_prefill_host: the prefill on host-resident (page-locked) tensors, copied
in, computed and copied out in overlapping groups of (batch, head) units.  It
runs the same single-pass kernels on the same data as la_prefill without the
segment split, so its results must equal those bit for bit; one case also goes
to the fp64 oracle."""
import pytest
import torch

import synth
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("B,H,N,d,dtype,group,with_s0", [
    (1, 3, 1000, 128, "bf16", 2, False),     # groups 2 + 1
    (2, 5, 300, 128, "bf16", 3, True),       # 10 units in groups of 3 (3, 3, 3, 1)
    (1, 16, 4096, 128, "bf16", 4, True),
    (1, 4, 777, 128, "bf16", 64, False),     # one group larger than the batch
    (2, 2, 200, 64, "fp32", 1, True),        # FFMA path, one unit per group
    (2, 3, 500, 64, "bf16", 4, True),        # tensor cores at d = 64
])
def test_host_prefill_equals_device_prefill(la, monkeypatch, B, H, N, d, dtype, group, with_s0):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", "1")  # the reference in one pass, as every host group runs
    q, k, v = synth.dense(B, H, N, d, dtype, seed=B * 100 + H + N)
    s0 = synth.outer_product_state(B * H, d, d, [300] * (B * H), seed=N).view(B, H, d, d) if with_s0 else None
    o_ref, s_ref = la.prefill(q.cuda(), k.cuda(), v.cuda(), None if s0 is None else s0.cuda())
    o, s = la.prefill_host(_pinned(q), _pinned(k), _pinned(v), None if s0 is None else _pinned(s0), group=group)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert o.device.type == "cpu" and s.device.type == "cpu"
    assert torch.equal(o, o_ref.cpu())
    assert torch.equal(s, s_ref.cpu())


def test_host_prefill_matches_oracle(la, oracle_mod):
    q, k, v = synth.dense(1, 6, 1500, 128, "bf16", seed=12)
    o, s = la.prefill_host(_pinned(q), _pinned(k), _pinned(v), group=4)
    torch.cuda.synchronize()
    ro, rs = oracle_mod.recurrent(q, k, v)
    assert_out(o, ro, torch.bfloat16, 2)
    assert_state(s, rs, 2)


def test_host_prefill_empty_sequence_copies_state(la):
    q = torch.zeros(1, 3, 0, 128, dtype=torch.bfloat16)
    s0 = synth.outer_product_state(3, 128, 128, [100] * 3, seed=2).view(1, 3, 128, 128)
    o, s = la.prefill_host(q, q, q, _pinned(s0), group=2)
    torch.cuda.synchronize()
    assert o.shape == (1, 3, 0, 128)
    assert torch.equal(s, s0)


def test_host_prefill_pageable_memory(la, monkeypatch):
    """Pageable host memory still gives the right answer (without overlap)."""
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", "1")
    q, k, v = synth.dense(1, 2, 333, 128, "bf16", seed=4)
    o_ref, s_ref = la.prefill(q.cuda(), k.cuda(), v.cuda())
    o = torch.empty_like(v)
    s = torch.empty(1, 2, 128, 128)
    la.prefill_host(q, k, v, group=1, out=o, s_out=s)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref.cpu()) and torch.equal(s, s_ref.cpu())

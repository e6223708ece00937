"""Batched decode step on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import synth
from tests.parity import assert_out, assert_state, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_steps_match_oracle(la, oracle_mod, dtype, d):
    B, H, steps = 5, 3, 6
    S0 = synth.outer_product_state(B * H, d, d, synth.lengths(B * H, 100, 2000, seed=d), seed=d).view(B, H, d, d)
    q, k, v = synth.qkv((steps, B, H, d), d, dtype, seed=11 + d)
    S_gpu = S0.cuda()
    S_ref = S0.double().numpy()
    for t in range(steps):
        o = la.decode_step(q[t].cuda(), k[t].cuda(), v[t].cuda(), S_gpu)
        ro, S_ref = oracle_mod.decode(q[t], k[t], v[t], S_ref)
        assert_out(o.cpu(), ro, synth.torch_dtype(dtype), 2)
    assert_state(S_gpu.cpu(), S_ref, 2, tol=1e-5)
    assert la.device_status() == 0


def test_decode_equals_prefill(la):
    """m decode steps from S match a GPU prefill of the same m tokens from S."""
    B, H, m, d = 2, 4, 40, 128
    S0 = synth.outer_product_state(B * H, d, d, [500] * (B * H), seed=3).view(B, H, d, d)
    q, k, v = synth.dense(B, H, m, d, "bf16", seed=8)
    o_p, s_p = la.prefill(q.cuda(), k.cuda(), v.cuda(), S0.cuda())
    S = S0.cuda()
    outs = [la.decode_step(q[:, :, t].contiguous().cuda(), k[:, :, t].contiguous().cuda(),
                           v[:, :, t].contiguous().cuda(), S) for t in range(m)]
    o_d = torch.stack(outs, 2)
    assert_out(o_d.cpu(), to64(o_p), torch.bfloat16, 2)
    assert_state(S.cpu(), to64(s_p), 2, tol=1e-5)


def test_decode_integer_exact(la, oracle_mod):
    B, H, d = 3, 2, 128
    S0 = synth.integer_valued((B, H, d, d), seed=1, lo=-50, hi=50)
    q = synth.integer_valued((B, H, d), seed=2, dtype=torch.bfloat16)
    k = synth.integer_valued((B, H, d), seed=3, dtype=torch.bfloat16)
    v = synth.integer_valued((B, H, d), seed=4, dtype=torch.bfloat16)
    S = S0.cuda()
    o = la.decode_step(q.cuda(), k.cuda(), v.cuda(), S)
    ro, rs = oracle_mod.decode(q, k, v, S0)
    assert torch.equal(o.cpu(), torch.from_numpy(ro).to(torch.bfloat16))
    np.testing.assert_array_equal(to64(S), rs)

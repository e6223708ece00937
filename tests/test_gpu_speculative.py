"""Speculative decoding: verify m draft tokens, then commit the accepted prefix.

The state of a recurrent layer cannot be truncated after the fact (page
"MiniMax: «Почему M2 …»", section 4), so the library keeps S untouched while
verifying and advances it by exactly the accepted drafts afterwards.  Checks:
verify's outputs against the fp64 recurrence run over the m drafts from S;
commit's state against the recurrence over the accepted prefix, and bit for
bit against the same number of la_decode_step calls.
"""
import pytest
import torch

import synth
from tests.parity import assert_out, assert_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _case(B, H, m, d, dtype, seed):
    U = B * H
    S = synth.outer_product_state(U, d, d, [3000 + 100 * (u % 12) for u in range(U)], seed=seed).view(B, H, d, d)
    q, k, v = synth.qkv((B, H, m, d), d, dtype, seed=seed + 1)
    return S, q, k, v


@pytest.mark.parametrize("m", [1, 2, 4, 7, 8, 10, 12, 13, 16])  # every draft-capacity instance (4, 8, 12, 16)
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "bf16"), (128, "fp32"), (64, "fp32")])
def test_verify_matches_recurrence_over_drafts(la, oracle_mod, m, d, dtype):
    B, H = 3, 4
    S, q, k, v = _case(B, H, m, d, dtype, seed=m * 10 + d)
    Sd = S.cuda()
    o = la.decode_verify(q.cuda(), k.cuda(), v.cuda(), Sd)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(Sd.cpu(), S), "verify must not change the state"
    ro, _ = oracle_mod.recurrent(q, k, v, S)
    assert_out(o.cpu(), ro, q.dtype, 2)


@pytest.mark.parametrize("m", [1, 3, 4, 5, 8, 13, 16])
@pytest.mark.parametrize("phi", ["identity", "relu", "elu1"])
@pytest.mark.parametrize("B,H", [(3, 4), (2, 200)])  # 12 units; 400 units, several per CTA of the persistent grid
def test_verify_tensor_cores_match_recurrence(la, oracle_mod, monkeypatch, m, phi, B, H):
    """bf16 at d = 128 with the q S_0 products on the tensor cores (the fp32
    S_0 read as tf32, fp32 accumulation), forced for every m: the fp64
    recurrence over the drafts at the bf16 output bars, per unit, and the
    FFMA kernel (fp32 S_0) within the same bars."""
    d = 128
    S, q, k, v = _case(B, H, m, d, "bf16", seed=m * 7 + 1)
    Sd = S.cuda()
    monkeypatch.setenv("LA_VERIFY_TC", "1")
    o_tc = la.decode_verify(q.cuda(), k.cuda(), v.cuda(), Sd, phi=phi)
    monkeypatch.setenv("LA_VERIFY_TC", "0")
    o_ff = la.decode_verify(q.cuda(), k.cuda(), v.cuda(), Sd, phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(Sd.cpu(), S), "verify must not change the state"
    ro, _ = oracle_mod.recurrent(q, k, v, S, phi=phi)
    assert_out(o_tc.cpu(), ro, torch.bfloat16, 2)
    assert_out(o_tc.cpu(), o_ff.cpu().double().numpy(), torch.bfloat16, 2)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_commit_matches_recurrence_over_accepted_prefix(la, oracle_mod, m):
    B, H, d = 5, 3, 128
    S, q, k, v = _case(B, H, m, d, "bf16", seed=100 + m)
    accepted = torch.tensor([(b * 3) % (m + 1) for b in range(B)], dtype=torch.int32)
    accepted[0], accepted[-1] = 0, m
    Sd = S.cuda()
    la.decode_commit(k.cuda(), v.cuda(), Sd, accepted.cuda())
    torch.cuda.synchronize()
    assert la.device_status() == 0
    got = Sd.cpu()
    for b in range(B):
        a = int(accepted[b])
        if a == 0:
            assert torch.equal(got[b], S[b])
            continue
        _, rs = oracle_mod.recurrent(q[b:b + 1, :, :a], k[b:b + 1, :, :a], v[b:b + 1, :, :a], S[b:b + 1])
        assert_state(got[b:b + 1], rs, 2, tol=1e-6)


@pytest.mark.parametrize("m,acc", [(6, [0, 2, 5, 6]), (12, [1, 9, 12, 0])])  # both commit instances (m <= 8, m > 8)
def test_commit_equals_decode_steps_bit_for_bit(la, m, acc):
    """Commit adds the accepted tokens with one fused multiply-add each, in
    token order, exactly as consecutive decode steps do."""
    B, H, d = 4, 2, 128
    S, q, k, v = _case(B, H, m, d, "bf16", seed=7 + m)
    accepted = torch.tensor(acc, dtype=torch.int32)
    S_commit = S.cuda()
    la.decode_commit(k.cuda(), v.cuda(), S_commit, accepted.cuda())
    for b in range(B):
        S_steps = S[b:b + 1].cuda()
        for t in range(int(accepted[b])):
            la.decode_step(q[b:b + 1, :, t].cuda(), k[b:b + 1, :, t].cuda(), v[b:b + 1, :, t].cuda(), S_steps)
        assert torch.equal(S_commit[b:b + 1].cpu(), S_steps.cpu()), f"sequence {b}"
    assert la.device_status() == 0


def test_verify_then_commit_equals_decoding_the_accepted_tokens(la):
    """The usual flow: verify 4 drafts, accept 3, commit, then decode on; the
    outputs of the accepted drafts equal those of plain decode steps."""
    B, H, m, d = 2, 4, 4, 128
    S, q, k, v = _case(B, H, m, d, "bf16", seed=9)
    Sd = S.cuda()
    o_ver = la.decode_verify(q.cuda(), k.cuda(), v.cuda(), Sd)
    la.decode_commit(k.cuda(), v.cuda(), Sd, torch.full((B,), 3, dtype=torch.int32, device="cuda"))
    S_steps = S.cuda()
    for t in range(3):
        o_t = la.decode_step(q[:, :, t].cuda(), k[:, :, t].cuda(), v[:, :, t].cuda(), S_steps)
        assert_out(o_ver[:, :, t].cpu(), o_t.cpu().double().numpy(), torch.bfloat16, 2)
    assert torch.equal(Sd.cpu(), S_steps.cpu())
    assert la.device_status() == 0


def test_commit_validation_rejects_out_of_range_counts(la, monkeypatch):
    monkeypatch.setenv("LA_VALIDATE", "1")
    B, H, m, d = 2, 1, 4, 128
    S, q, k, v = _case(B, H, m, d, "bf16", seed=11)
    with pytest.raises(la.LAError):
        la.decode_commit(k.cuda(), v.cuda(), S.cuda(), torch.tensor([1, 5], dtype=torch.int32, device="cuda"))

"""Parity at the full benchmark sizes, in the launch configuration bench.py times.

Each test runs the whole batch through the C ABI exactly as the benchmark does
(same shapes, same calls) and compares every (batch, head) or (sequence, head)
unit of it with the fp64 oracle, in groups of units so that host memory stays
bounded.  Decode keeps a seeded sample of 256 units over its 1024 steps (the
oracle then follows those units step by step), and the speculative case a
sample of 256 units.
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


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _group(oracle_mod):
    # units per oracle call: one per host thread, at least 8 (bounded host memory)
    return max(8, min(16, oracle_mod.num_threads()))


def test_prefill_b4_h32_n8192(la, oracle_mod):
    B, H, N, d = 4, 32, 8192, 128
    dev = torch.device("cuda")
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=61, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    la.prefill(q, k, v, None, out=o, s_out=s)
    assert la.device_status() == 0
    qf, kf, vf, of, sf = (x.view(B * H, *x.shape[2:]) for x in (q, k, v, o, s))
    G = 4 * _group(oracle_mod)
    for u0 in range(0, B * H, G):
        u1 = min(B * H, u0 + G)
        ro, rs = oracle_mod.recurrent(qf[u0:u1].cpu(), kf[u0:u1].cpu(), vf[u0:u1].cpu())
        assert_out(of[u0:u1].cpu(), ro, torch.bfloat16, 1, what=f"O units {u0}..{u1 - 1}")
        assert_state(sf[u0:u1].cpu(), rs, 1)
    del q, k, v, o, s
    _free()


def test_long_prefill_h64_n131072(la, oracle_mod):
    B, H, N, d = 1, 64, 131072, 128
    dev = torch.device("cuda")
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=3, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    la.prefill(q, k, v, None, out=o, s_out=s)
    assert la.device_status() == 0
    G = _group(oracle_mod)
    for h0 in range(0, H, G):
        h1 = min(H, h0 + G)
        ro, rs = oracle_mod.recurrent(q[0, h0:h1].cpu(), k[0, h0:h1].cpu(), v[0, h0:h1].cpu())
        assert_out(o[0, h0:h1].cpu(), ro, torch.bfloat16, 1, what=f"O heads {h0}..{h1 - 1}")
        assert_state(s[0, h0:h1].cpu(), rs, 1)
        del ro, rs
    del q, k, v, o, s
    _free()


def test_decode_b256_h64_1024_steps(la, oracle_mod):
    B, H, d, steps = 256, 64, 128, 1024
    dev = torch.device("cuda")
    U = B * H
    L_seq = synth.lengths(B, 1024, 65536, seed=41)
    L = [L_seq[u // H] for u in range(U)]
    S = torch.empty(U, d, d, dtype=torch.float32, device=dev)
    for u0 in range(0, U, 2048):
        S[u0:u0 + 2048] = synth.outer_product_state(min(2048, U - u0), d, d, L[u0:u0 + 2048], seed=7 + u0,
                                                    device=dev)
    S = S.view(B, H, d, d)
    units = synth.choose(U, 256, seed=3)
    idx = torch.tensor(units, device=dev)
    S_ref = S.view(U, d, d)[idx].double().cpu().numpy()
    qs, ks, vs = synth.qkv((steps, B, H, d), d, "bf16", seed=43, device=dev)
    o = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    check = {0, 1, 511, 1023}
    for t in range(steps):
        la.decode_step(qs[t], ks[t], vs[t], S, out=o)
        qt, kt, vt = (x[t].view(U, d)[idx].cpu() for x in (qs, ks, vs))
        ro, S_ref = oracle_mod.decode(qt, kt, vt, S_ref)
        if t in check:
            assert_out(o.view(U, d)[idx].cpu(), ro, torch.bfloat16, 1, what=f"o at step {t + 1}")
    assert la.device_status() == 0
    assert_state(S.view(U, d, d)[idx].cpu(), S_ref, 1, tol=1e-5)
    del qs, ks, vs, S, o
    _free()


def test_varlen_64_sequences_with_resume(la, oracle_mod):
    n_seq, H, d = 64, 32, 128
    dev = torch.device("cuda")
    lens = synth.lengths(n_seq, 1024, 32768, seed=51)
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=53, device=dev)
    resumed = synth.choose(n_seq, 32, seed=55)
    pool = synth.outer_product_state(32 * H, d, d, [4096] * (32 * H), seed=57, device=dev).view(32, H, d, d)
    init = torch.full((n_seq,), -1, dtype=torch.int32)
    for j, n in enumerate(resumed):
        init[n] = j
    o, s = la.prefill_varlen(q, k, v, cu.to(dev), pool, init.to(dev))
    assert la.device_status() == 0
    # every (sequence, head) unit: one oracle call per sequence over its 32 heads
    for n in range(n_seq):
        a, b = int(cu[n]), int(cu[n + 1])
        qn, kn, vn = (x[a:b].transpose(0, 1).cpu() for x in (q, k, v))
        s0 = pool[int(init[n])].cpu() if init[n] >= 0 else None
        ro, rs = oracle_mod.recurrent(qn, kn, vn, s0)
        assert_out(o[a:b].transpose(0, 1).cpu(), ro, torch.bfloat16, 1, what=f"O of sequence {n}")
        assert_state(s[n].cpu(), rs, 1)
        del qn, kn, vn, ro, rs
    del q, k, v, o, s, pool
    _free()


def test_backward_b4_h32_n8192(la, oracle_mod):
    """The gradients at the 8K prefill shape (three tensor-core passes), every
    unit against the oracle's chain rule."""
    B, H, N, d = 4, 32, 8192, 128
    dev = torch.device("cuda")
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=81, device=dev)
    _, _, do = synth.dense(B, H, N, d, "bf16", seed=91, device=dev)
    ds_n = torch.randn(B, H, d, d, device=dev, generator=torch.Generator(device=dev).manual_seed(93))
    dq, dk, dv, ds0 = la.prefill_backward(q, k, v, do, None, ds_n)
    assert la.device_status() == 0
    G = 2 * _group(oracle_mod)
    for u0 in range(0, B * H, G):
        sl = slice(u0, min(B * H, u0 + G))
        flat = lambda x: x.view(B * H, *x.shape[2:])[sl].cpu()  # noqa: E731
        rq, rk, rv, rs0 = oracle_mod.backward(flat(q), flat(k), flat(v), flat(do), None, flat(ds_n))
        for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
            assert_out(flat(g), r, torch.bfloat16, 1, what=f"{n} units from {u0}")
        assert_state(flat(ds0), rs0, 1)
    del q, k, v, do, dq, dk, dv, ds0
    _free()


def test_speculative_b256_h64_m4(la, oracle_mod):
    """Verify and commit of 4 drafts at the decode shape, 256 sampled units
    against the fp64 recurrence over the drafts."""
    B, H, d, m = 256, 64, 128, 4
    dev = torch.device("cuda")
    U = B * H
    g = torch.Generator(device=dev).manual_seed(97)
    S = torch.randn(B, H, d, d, device=dev, generator=g) * 8.0   # the magnitude of a 8K-token state
    q, k, v = synth.qkv((B, H, m, d), d, "bf16", seed=99, device=dev)
    accepted = torch.randint(0, m + 1, (B,), generator=g, device=dev, dtype=torch.int32)
    units = synth.choose(U, 256, seed=8)
    idx = torch.tensor(units, device=dev)
    S_before = S.view(U, d, d)[idx].cpu()
    o = la.decode_verify(q, k, v, S)
    la.decode_commit(k, v, S, accepted)
    assert la.device_status() == 0
    qf, kf, vf, of = (x.view(U, m, d)[idx].cpu() for x in (q, k, v, o))
    ro, _ = oracle_mod.recurrent(qf, kf, vf, S_before)
    assert_out(of, ro, torch.bfloat16, 1)
    S_after = S.view(U, d, d)[idx].cpu()
    for j, u in enumerate(units):
        a = int(accepted[u // H])
        if a == 0:
            assert torch.equal(S_after[j], S_before[j])
            continue
        _, rs = oracle_mod.recurrent(qf[j:j + 1, :a], kf[j:j + 1, :a], vf[j:j + 1, :a], S_before[j:j + 1])
        assert_state(S_after[j:j + 1], rs, 1, tol=1e-6)
    del S, q, k, v, o
    _free()

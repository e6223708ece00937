"""Feature maps phi (identity, elu + 1, relu) on every path, against the fp64
oracle with the same phi applied in float64 (page "MiniMax-M1で理解する…",
section "線形アテンションの数学的基礎": phi(Q) (phi(K)^T V))."""
import numpy as np
import pytest
import torch

import synth
from tests.parity import assert_out, assert_state, assert_varlen_out

pytestmark = pytest.mark.gpu

PHIS = ["elu1", "relu"]
# On the bf16 tensor-core prefill phi(q), phi(k) are tensor-core operands, so
# they are rounded to bf16: relu(x) of a bf16 x is exact, elu(x) + 1 is not,
# and the state then inherits that operand rounding (up to 2^-9 relative per
# element of phi(k)); its bar there is the output's 5e-3.  The fp32 paths keep
# phi in fp32 and meet the 1e-4 state bar.
TC_STATE_TOL = {"elu1": 5e-3, "relu": 1e-4}


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _state(U, d, seed):
    return synth.outer_product_state(U, d, d, [400] * U, seed=seed)


@pytest.mark.parametrize("phi", PHIS)
@pytest.mark.parametrize("B,H,N", [(1, 2, 1), (1, 2, 200), (2, 3, 1000), (1, 1, 4096 + 33)])
def test_tc_prefill_with_phi(la, oracle_mod, phi, B, H, N):
    q, k, v = synth.dense(B, H, N, 128, "bf16", seed=N + 3)
    s0 = _state(B * H, 128, seed=N).view(B, H, 128, 128)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), s0.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, s0, phi=phi)
    assert_out(o.cpu(), ro, torch.bfloat16, 2)
    assert_state(s.cpu(), rs, 2, tol=TC_STATE_TOL[phi])


@pytest.mark.parametrize("phi", PHIS)
def test_tc_prefill_with_phi_and_segments(la, oracle_mod, monkeypatch, phi):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", "3")
    q, k, v = synth.dense(1, 2, 3000, 128, "bf16", seed=77)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, phi=phi)
    assert_out(o.cpu(), ro, torch.bfloat16, 2)
    assert_state(s.cpu(), rs, 2, tol=TC_STATE_TOL[phi])


@pytest.mark.parametrize("phi", PHIS)
@pytest.mark.parametrize("dtype,d", [("fp32", 64), ("fp32", 128)])
def test_ffma_prefill_with_phi(la, oracle_mod, phi, dtype, d):
    q, k, v = synth.dense(2, 2, 300, d, dtype, seed=d + 1)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, phi=phi)
    assert_out(o.cpu(), ro, q.dtype, 2)
    assert_state(s.cpu(), rs, 2)


@pytest.mark.parametrize("phi", PHIS)
def test_tc_d64_prefill_with_phi(la, oracle_mod, phi):
    """bf16 with d = 64 runs on the tensor cores too (phi(q), phi(k) in bf16)."""
    q, k, v = synth.dense(2, 2, 300, 64, "bf16", seed=65)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.recurrent(q, k, v, phi=phi)
    assert_out(o.cpu(), ro, q.dtype, 2)
    assert_state(s.cpu(), rs, 2, tol=TC_STATE_TOL[phi])


@pytest.mark.parametrize("phi", PHIS)
def test_varlen_with_phi(la, oracle_mod, phi):
    lens = [0, 1, 130, 257, 1000]
    cu = synth.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 2, 128
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=5)
    pool = _state(2 * H, d, seed=6).view(2, H, d, d)
    init = torch.tensor([-1, 0, 1, -1, 0], dtype=torch.int32)
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), pool.cuda(), init.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, init, phi=phi)
    assert_varlen_out(o.cpu(), ro, cu, torch.bfloat16)
    assert_state(s.cpu(), rs, 2, tol=TC_STATE_TOL[phi])


@pytest.mark.parametrize("phi", PHIS)
def test_decode_with_phi(la, oracle_mod, phi):
    B, H, d, T = 2, 3, 128, 8
    S = _state(B * H, d, seed=8).view(B, H, d, d)
    Sd = S.cuda()
    S_ref = S.double().numpy()
    qs, ks, vs = synth.qkv((T, B, H, d), d, "bf16", seed=9)
    for t in range(T):
        o = la.decode_step(qs[t].cuda(), ks[t].cuda(), vs[t].cuda(), Sd, phi=phi)
        ro, S_ref = oracle_mod.decode(qs[t], ks[t], vs[t], S_ref, phi=phi)
        assert_out(o.cpu(), ro, torch.bfloat16, 2)
    assert_state(Sd.cpu(), S_ref, 2, tol=1e-6)
    assert la.device_status() == 0


@pytest.mark.parametrize("phi", PHIS)
def test_verify_and_commit_with_phi(la, oracle_mod, phi):
    B, H, m, d = 2, 2, 5, 128
    S = _state(B * H, d, seed=10).view(B, H, d, d)
    q, k, v = synth.qkv((B, H, m, d), d, "bf16", seed=11)
    Sd = S.cuda()
    o = la.decode_verify(q.cuda(), k.cuda(), v.cuda(), Sd, phi=phi)
    ro, rs = oracle_mod.recurrent(q, k, v, S, phi=phi)
    assert_out(o.cpu(), ro, torch.bfloat16, 2)
    la.decode_commit(k.cuda(), v.cuda(), Sd, torch.full((B,), m, dtype=torch.int32, device="cuda"), phi=phi)
    assert_state(Sd.cpu(), rs, 2, tol=1e-6)
    assert la.device_status() == 0


def test_identity_phi_is_the_default(la):
    q, k, v = (x.cuda() for x in synth.dense(1, 2, 700, 128, "bf16", seed=12))
    o1, s1 = la.prefill(q, k, v)
    o2, s2 = la.prefill(q, k, v, phi="identity")
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_unknown_phi_is_rejected(la):
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        la.prefill(q, q, q, phi="tanh")


def _raw_prefill(la, q, k, v, phi, ws):
    """la_prefill_ex through the C ABI with the given (possibly too small) workspace."""
    B, H, N, d = q.shape
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=q.device)
    wsb = 0 if ws is None else ws.numel()
    st = la.lib.la_prefill_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None, s.data_ptr(), B, H, N,
                              d, d, 0, 0, la.PHI[phi], None if ws is None else ws.data_ptr(), wsb,
                              torch.cuda.current_stream().cuda_stream)
    assert st == 0, la.lib.la_last_error()
    return o, s


@pytest.mark.parametrize("segments", [None, "3"])
@pytest.mark.parametrize("d", [128, 64])
def test_tc_phi_prepass_equals_in_kernel_mapping(la, monkeypatch, segments, d):
    """With room in the workspace q and k are mapped by a pre-pass (elu + 1);
    without it the kernel maps the tiles in shared memory.  Both round phi to
    bf16 the same way, so the results are bit-identical."""
    if segments:
        monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    phi = "elu1"
    B, H, N = 1, 2, 3000
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=91, device="cuda")
    full = la.prefill_workspace_size(B, H, N, d, torch.bfloat16, phi)
    seg = la.prefill_workspace_size(B, H, N, d, torch.bfloat16)
    assert full >= seg + 2 * B * H * N * d * 2
    ws_full = torch.empty(full, dtype=torch.uint8, device="cuda")
    ws_seg = torch.empty(seg, dtype=torch.uint8, device="cuda") if seg else None
    o1, s1 = _raw_prefill(la, q, k, v, phi, ws_full)
    o2, s2 = _raw_prefill(la, q, k, v, phi, ws_seg)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


@pytest.mark.parametrize("segments", [None, "3"])
@pytest.mark.parametrize("d", [128, 64])
def test_tc_relu_in_kernel_equals_identity_on_mapped_inputs(la, monkeypatch, segments, d):
    """relu of a bf16 value is exact, so mapping the tiles inside the kernel
    must give exactly the identity prefill of relu(q), relu(k) (mapped by
    torch here)."""
    if segments:
        monkeypatch.setenv("LA_PREFILL_SEGMENTS", segments)
    q, k, v = synth.dense(2, 3, 1500, d, "bf16", seed=93, device="cuda")
    o1, s1 = la.prefill(q, k, v, phi="relu")
    o2, s2 = la.prefill(torch.relu(q), torch.relu(k), v)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


def test_relu_needs_no_phi_workspace(la):
    """relu is mapped inside the prefill kernel whatever the workspace."""
    assert la.prefill_workspace_size(2, 4, 3000, 128, torch.bfloat16, "relu") == \
        la.prefill_workspace_size(2, 4, 3000, 128, torch.bfloat16)
    assert la.prefill_varlen_workspace_size(3, 5000, 4, 128, torch.bfloat16, "relu") == \
        la.prefill_varlen_workspace_size(3, 5000, 4, 128, torch.bfloat16)


@pytest.mark.parametrize("phi", ["elu1"])
def test_varlen_phi_prepass_equals_in_kernel_mapping(la, phi):
    lens = [700, 1, 129, 2000]
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device="cuda")
    T, H, d = int(cu[-1]), 3, 128
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=5, device="cuda")
    outs = []
    for with_phi_room in (True, False):
        n = la.prefill_varlen_workspace_size(len(lens), T, H, d, torch.bfloat16, phi if with_phi_room else "identity")
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        o = torch.empty_like(v)
        s = torch.empty(len(lens), H, d, d, dtype=torch.float32, device="cuda")
        st = la.lib.la_prefill_varlen_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), cu.data_ptr(),
                                         len(lens), T, None, 0, None, s.data_ptr(), H, d, d, 0, 0, la.PHI[phi],
                                         ws.data_ptr(), n, torch.cuda.current_stream().cuda_stream)
        assert st == 0, la.lib.la_last_error()
        outs.append((o, s))
    torch.cuda.synchronize()
    assert la.device_status() == 0
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("phi", PHIS)
def test_varlen_with_phi_and_segments(la, oracle_mod, monkeypatch, phi):
    monkeypatch.setenv("LA_PREFILL_SEGMENTS", "3")
    lens = [2000, 1, 900]
    cu = synth.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 2, 128
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=8)
    o, s = la.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), phi=phi)
    torch.cuda.synchronize()
    assert la.device_status() == 0
    ro, rs = oracle_mod.varlen(q, k, v, cu, phi=phi)
    assert_varlen_out(o.cpu(), ro, cu, torch.bfloat16)
    assert_state(s.cpu(), rs, 2, tol=TC_STATE_TOL[phi])

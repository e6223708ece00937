"""The library's calls are stream-ordered and never synchronise the host, so
a launch-bound loop of them can be captured in a CUDA graph and replayed.
Replays must give exactly the eager results."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def test_decode_steps_in_a_cuda_graph(la):
    B, H, d, T = 4, 8, 128, 16
    S0 = synth.outer_product_state(B * H, d, d, [500] * (B * H), seed=3).view(B, H, d, d).cuda()
    q, k, v = synth.qkv((T, B, H, d), d, "bf16", seed=4, device="cuda")
    # eager
    S_e = S0.clone()
    o_e = torch.empty(T, B, H, d, dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        la.decode_step(q[t], k[t], v[t], S_e, out=o_e[t])
    # captured: T steps in one graph, replayed from the same starting state
    S_g = S0.clone()
    o_g = torch.empty_like(o_e)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        la.decode_step(q[0], k[0], v[0], S0.clone(), out=o_g[0])
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t in range(T):
            la.decode_step(q[t], k[t], v[t], S_g, out=o_g[t])
    for _ in range(2):  # replay twice from the same start
        S_g.copy_(S0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(S_g, S_e)
        assert torch.equal(o_g, o_e)
    assert la.device_status() == 0


def test_prefill_and_backward_in_a_cuda_graph(la):
    q, k, v = synth.dense(1, 4, 700, 128, "bf16", seed=5, device="cuda")
    _, _, do = synth.dense(1, 4, 700, 128, "bf16", seed=6, device="cuda")
    o_e, s_e = la.prefill(q, k, v)
    g_e = la.prefill_backward(q, k, v, do)
    o_g, s_g = torch.empty_like(o_e), torch.empty_like(s_e)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds0 = torch.empty_like(s_e)
    ws = torch.empty(max(la.prefill_workspace_size(1, 4, 700, 128, torch.bfloat16), 1), dtype=torch.uint8,
                     device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        la.prefill(q, k, v, out=o_g, s_out=s_g, workspace=ws)
        st = la.lib.la_prefill_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), None, None,
                                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ds0.data_ptr(), 1, 4, 700, 128,
                                        128, 0, torch.cuda.current_stream().cuda_stream)
        assert st == 0
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o_g, o_e) and torch.equal(s_g, s_e)
    for a, b in zip((dq, dk, dv, ds0), g_e):
        assert torch.equal(a, b)
    assert la.device_status() == 0

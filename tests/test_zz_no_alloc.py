"""The allocation-free ragged prefill entry point (la_prefill_varlen_noalloc).

Some callers cannot allocate device memory when they call the library (a host
framework that owns all device memory, or a serving loop where cudaMalloc is
not allowed).  For them the library offers a variant of la_prefill_varlen
that uses a scratch array built into the library instead of a caller-provided
workspace.  This file checks, through the C ABI, that two calls in a row give
the same results as the workspace-based entry point and as the fp64 oracle,
for both input types and both head sizes, that batches larger than the
built-in scratch are refused, and that the Python wrapper checks its buffers'
shapes before it launches anything.  It is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synth
from tests.parity import assert_state, assert_varlen_out, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _batch(lens, H, d, dtype, seed):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, d), d, dtype, seed=seed)
    pool = synth.outer_product_state(2 * H, d, d, [300] * (2 * H), seed=seed + 1).view(2, H, d, d)
    idx = torch.tensor([(i % 3) - 1 for i in range(len(lens))], dtype=torch.int32)
    return cu, q, k, v, pool, idx


def _noalloc(la, cu, q, k, v, pool, idx):
    T, H, d = q.shape
    n = cu.numel() - 1
    o = torch.full_like(v, float("nan"))
    s = torch.full((n, H, d, d), float("nan"), dtype=torch.float32, device=q.device)
    dt = 0 if q.dtype == torch.bfloat16 else 1
    st = la.lib.la_prefill_varlen_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), cu.data_ptr(), n, T, pool.data_ptr(),
        pool.shape[0], idx.data_ptr(), s.data_ptr(), H, d, d, dt, 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, la.lib.la_last_error()
    return o, s


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 128), ("fp32", 64)])
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(la, oracle_mod, dtype, d):
    # two different batches in a row: the second call must not depend on what
    # the first one left in the shared scratch
    dt = synth.torch_dtype(dtype)
    for lens, seed in (([700, 1, 0, 129, 2048, 77], 11), ([5, 300, 128, 1000], 12)):
        cu, q, k, v, pool, idx = _batch(lens, 3, d, dtype, seed + d)
        cu_d, q_d, k_d, v_d, pool_d, idx_d = (x.cuda() for x in (cu, q, k, v, pool, idx))
        o_ref, s_ref = la.prefill_varlen(q_d, k_d, v_d, cu_d, pool_d, idx_d)
        o, s = _noalloc(la, cu_d, q_d, k_d, v_d, pool_d, idx_d)
        torch.cuda.synchronize()
        assert_varlen_out(o.cpu(), to64(o_ref), cu, dt)
        assert_state(s.cpu(), to64(s_ref), 2, tol=1e-5)
        ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
        assert_varlen_out(o.cpu(), ro, cu, dt)
        assert_state(s.cpu(), rs, 2)
    assert la.device_status() == 0


def test_noalloc_python_wrapper(la, oracle_mod):
    cu, q, k, v, pool, idx = _batch([40, 0, 300], 2, 128, "bf16", seed=21)
    dev = [x.cuda() for x in (cu, q, k, v, pool, idx)]
    out = torch.empty_like(dev[3])
    s_out = torch.empty(3, 2, 128, 128, dtype=torch.float32, device="cuda")
    la.prefill_varlen_noalloc(dev[1], dev[2], dev[3], dev[0], dev[4], dev[5], out=out, s_out=s_out)
    torch.cuda.synchronize()
    ro, rs = oracle_mod.varlen(q, k, v, cu, pool, idx)
    assert_varlen_out(out.cpu(), ro, cu, torch.bfloat16)
    assert_state(s_out.cpu(), rs, 2)


def test_noalloc_python_wrapper_rejects_wrong_shapes(la):
    cu, q, k, v, pool, idx = (x.cuda() for x in _batch([40, 9], 2, 128, "bf16", seed=22))
    T, H, d = q.shape
    good_out = torch.empty_like(v)
    cases = [
        dict(out=torch.empty(T - 1, H, d, dtype=q.dtype, device="cuda")),           # out too short
        dict(out=good_out, s_out=torch.empty(1, H, d, d, device="cuda")),           # s_out for 1 of 2 sequences
        dict(out=good_out, state_pool=pool[:, :1].contiguous()),                    # pool with 1 of 2 heads
        dict(out=good_out, init_idx=idx[:1].contiguous()),                          # init_idx too short
    ]
    for extra in cases:
        args = dict(state_pool=pool, init_idx=idx)
        args.update(extra)
        sp, ii = args.pop("state_pool"), args.pop("init_idx")
        with pytest.raises(ValueError):
            la.prefill_varlen_noalloc(q, k, v, cu, sp, ii, **args)
    with pytest.raises(ValueError):
        la.prefill_varlen_noalloc(q, k, v[:, :, :64].contiguous(), cu, out=good_out)
    torch.cuda.synchronize()
    assert la.device_status() == 0


def test_noalloc_rejects_batches_beyond_its_scratch(la):
    from long_context_linear_b200 import _abi
    n = _abi.NOALLOC_MAX_SEQS + 1
    st = la.lib.la_prefill_varlen_noalloc(None, None, None, None, 1 << 20, n, 0, None, 0, None, None, 1, 128, 128,
                                          0, 0, None)
    assert st == _abi.LA_ERR_INVALID_ARG
    assert b"scratch" in la.lib.la_last_error()

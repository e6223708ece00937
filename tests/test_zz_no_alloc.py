"""The allocation-free ragged prefill entry point (la_prefill_varlen_noalloc).

Some callers cannot allocate device memory when they call the library (a host
framework that owns all device memory, or a serving loop where cudaMalloc is
not allowed).  For them the library offers a variant of la_prefill_varlen
that uses a scratch array built into the library instead of a caller-provided
workspace.  This file checks, through the C ABI, that two calls in a row give
the same results as the workspace-based entry point, and that batches larger
than the built-in scratch are refused.  It is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synth
from tests.parity import assert_out, assert_state, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import long_context_linear_b200 as la
    return la


def _batch(lens, H, d, seed):
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=seed)
    pool = synth.outer_product_state(2 * H, d, d, [300] * (2 * H), seed=seed + 1).view(2, H, d, d)
    idx = torch.tensor([(i % 3) - 1 for i in range(len(lens))], dtype=torch.int32)
    return [x.cuda() for x in (cu, q, k, v, pool, idx)]


def _noalloc(la, cu, q, k, v, pool, idx):
    T, H, d = q.shape
    n = cu.numel() - 1
    o = torch.full_like(v, float("nan"))
    s = torch.full((n, H, d, d), float("nan"), dtype=torch.float32, device=q.device)
    st = la.lib.la_prefill_varlen_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), cu.data_ptr(), n, T, pool.data_ptr(),
        pool.shape[0], idx.data_ptr(), s.data_ptr(), H, d, d, 0, 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, la.lib.la_last_error()
    return o, s


def test_noalloc_matches_workspace_entry_point_twice(la):
    # two different batches in a row: the second call must not depend on what
    # the first one left in the shared scratch
    for lens, seed in (([700, 1, 0, 129, 2048, 77], 11), ([5, 300, 128, 1000], 12)):
        cu, q, k, v, pool, idx = _batch(lens, 3, 128, seed)
        o_ref, s_ref = la.prefill_varlen(q, k, v, cu, pool, idx)
        o, s = _noalloc(la, cu, q, k, v, pool, idx)
        torch.cuda.synchronize()
        for n in range(len(lens)):
            a, b = int(cu[n]), int(cu[n + 1])
            if b > a:
                assert_out(o[a:b].transpose(0, 1).cpu(), to64(o_ref[a:b].transpose(0, 1)), torch.bfloat16, 1)
        assert_state(s.cpu(), to64(s_ref), 2)
    assert la.device_status() == 0


def test_noalloc_rejects_batches_beyond_its_scratch(la):
    from long_context_linear_b200 import _abi
    n = _abi.NOALLOC_MAX_SEQS + 1
    st = la.lib.la_prefill_varlen_noalloc(None, None, None, None, 1 << 20, n, 0, None, 0, None, None, 1, 128, 128,
                                          0, 0, None)
    assert st == _abi.LA_ERR_INVALID_ARG
    assert b"scratch" in la.lib.la_last_error()

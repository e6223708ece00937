"""The C-ABI library loads without a GPU, exports every symbol include/la.h
declares, and rejects bad arguments on the host before touching the device."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from long_context_linear_b200 import _abi  # built by conftest at session start
    return _abi.lib


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", src)
    return names


def test_header_declares_entry_points():
    names = _declared_functions()
    for want in ("la_prefill", "la_prefill_varlen", "la_decode_step", "la_status_string",
                 "la_prefill_workspace_size", "la_prefill_varlen_workspace_size", "la_device_status"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    from long_context_linear_b200 import _abi
    for name in _declared_functions():
        assert hasattr(lib, name), f"{name} missing from {_abi.LIB_PATH}"
        assert name in _abi.SIGNATURES, f"{name} has no binding signature"


def test_status_strings(lib):
    for s in range(5):
        assert lib.la_status_string(s)
    assert b"unknown" in lib.la_status_string(99)
    assert lib.la_version() >= 100


def test_workspace_sizes(lib):
    assert lib.la_prefill_workspace_size(4, 32, 8192, 128, 128, 0) == 0
    assert lib.la_prefill_varlen_workspace_size(0, 0, 32, 128, 128, 0) == 0
    ws = lib.la_prefill_varlen_workspace_size(64, 10 ** 6, 32, 128, 128, 0)
    assert ws >= 64 * 4 and ws % 256 == 0


def test_workspace_sizes_with_feature_map(lib):
    # identity and relu (mapped inside the kernel) add nothing; elu+1 adds
    # phi(q) and phi(k) in bf16 for the pre-pass on the tensor-core path
    base = lib.la_prefill_varlen_workspace_size(64, 1000, 32, 128, 128, 0)
    for phi in (0, 2):
        assert lib.la_prefill_workspace_size_ex(4, 32, 8192, 128, 128, 0, phi) == 0
        assert lib.la_prefill_varlen_workspace_size_ex(64, 1000, 32, 128, 128, 0, phi) == base
    assert lib.la_prefill_workspace_size_ex(4, 32, 8192, 128, 128, 0, 1) == 2 * 4 * 32 * 8192 * 128 * 2
    assert lib.la_prefill_workspace_size_ex(4, 32, 8192, 128, 128, 1, 1) == 0  # fp32: mapped at load
    assert lib.la_prefill_varlen_workspace_size_ex(64, 1000, 32, 128, 128, 0, 1) == base + 2 * 1000 * 32 * 256
    assert lib.la_prefill_varlen_workspace_size_ex(64, 1001, 3, 128, 128, 0, 1) == (
        lib.la_prefill_varlen_workspace_size(64, 1001, 3, 128, 128, 0) + 2 * ((1001 * 3 * 256 + 255) // 256 * 256))


FAKE = 1 << 20  # a 16-byte aligned non-null "device pointer"; never dereferenced on these paths


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, s0=None, s_out=None, B=1, H=1, N=16, dk=128, dv=128, dt=0,
             chunk=0, ws=None, wsb=0, stream=None)
    a.update(kw)
    return lib.la_prefill(a["q"], a["k"], a["v"], a["o"], a["s0"], a["s_out"], a["B"], a["H"], a["N"], a["dk"],
                          a["dv"], a["dt"], a["chunk"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96, dv=96), 2),          # unsupported head dim
    (dict(dk=128, dv=64), 2),         # dk != dv
    (dict(dk=0, dv=0), 1),
    (dict(dt=7), 1),                  # unknown dtype
    (dict(N=-1), 1),
    (dict(B=-2), 1),
    (dict(q=None), 1),                # null input
    (dict(o=FAKE + 8), 1),            # misaligned output
    (dict(s0=FAKE + 4), 1),           # misaligned state
    (dict(chunk=48), 2),              # chunk not available on the tensor-core path
    (dict(dt=1, chunk=128), 2),       # ... nor on the FFMA path
])
def test_prefill_rejects_bad_arguments(lib, kw, status):
    assert _prefill(lib, **kw) == status
    assert lib.la_last_error()


def test_empty_batch_is_noop(lib):
    assert _prefill(lib, B=0) == 0
    assert _prefill(lib, H=0, q=None, k=None, v=None, o=None) == 0


def _varlen(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, cu=FAKE, n_seq=2, T=100, pool=None, n_pool=0, idx=None,
             s_out=None, H=2, dk=128, dv=128, dt=0, chunk=0, ws=FAKE, wsb=256, stream=None)
    a.update(kw)
    return lib.la_prefill_varlen(a["q"], a["k"], a["v"], a["o"], a["cu"], a["n_seq"], a["T"], a["pool"],
                                 a["n_pool"], a["idx"], a["s_out"], a["H"], a["dk"], a["dv"], a["dt"], a["chunk"],
                                 a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(cu=None), 1),
    (dict(cu=FAKE + 2), 1),            # misaligned index array
    (dict(idx=FAKE), 1),               # init_idx without a pool
    (dict(ws=None), 1),                # workspace required on the tensor-core path
    (dict(wsb=8), 1),                  # ... of at least the advertised size
    (dict(n_seq=-1), 1),
    (dict(dk=64, dv=128), 2),
])
def test_varlen_rejects_bad_arguments(lib, kw, status):
    assert _varlen(lib, **kw) == status


def _decode(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, S=FAKE, B=2, H=2, dk=128, dv=128, dt=0, stream=None)
    a.update(kw)
    return lib.la_decode_step(a["q"], a["k"], a["v"], a["o"], a["S"], a["B"], a["H"], a["dk"], a["dv"], a["dt"],
                              a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(S=None), 1), (dict(S=FAKE + 4), 1), (dict(dk=32, dv=32), 2), (dict(B=-1), 1)])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status


def _decode_state(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, S=FAKE, B=2, H=2, dk=128, dv=128, dt=0, sdt=1, phi=0, stream=None)
    a.update(kw)
    return lib.la_decode_step_ex(a["q"], a["k"], a["v"], a["o"], a["S"], a["B"], a["H"], a["dk"], a["dv"],
                                 a["dt"], a["sdt"], a["phi"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(sdt=5), 1), (dict(sdt=-1), 1),   # unknown storage format
    (dict(dt=1, sdt=1), 2),                # a bf16 state needs bf16 inputs
    (dict(dt=1, sdt=2), 2),                # ... as do fp16 and fp8 states
    (dict(dt=1, sdt=3), 2), (dict(dt=1, sdt=4), 2),
    (dict(S=None), 1), (dict(S=FAKE + 8), 1), (dict(B=-1), 1), (dict(dk=64, dv=128), 2),
    (dict(phi=3), 1), (dict(phi=-1), 1)])
def test_decode_state_rejects_bad_arguments(lib, kw, status):
    assert _decode_state(lib, **kw) == status


def _verify(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, S=FAKE, B=2, H=2, m=4, dk=128, dv=128, dt=0, phi=0, stream=None)
    a.update(kw)
    return lib.la_decode_verify(a["q"], a["k"], a["v"], a["o"], a["S"], a["B"], a["H"], a["m"], a["dk"], a["dv"],
                                a["dt"], a["phi"], a["stream"])


def _commit(lib, **kw):
    a = dict(k=FAKE, v=FAKE, S=FAKE, acc=FAKE, B=2, H=2, m=4, dk=128, dv=128, dt=0, phi=0, stream=None)
    a.update(kw)
    return lib.la_decode_commit(a["k"], a["v"], a["S"], a["acc"], a["B"], a["H"], a["m"], a["dk"], a["dv"], a["dt"],
                                a["phi"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(m=0), 1), (dict(m=17), 1), (dict(S=None), 1), (dict(o=FAKE + 8), 1), (dict(B=-1), 1),
    (dict(dk=32, dv=32), 2), (dict(phi=7), 1)])
def test_verify_rejects_bad_arguments(lib, kw, status):
    assert _verify(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(m=0), 1), (dict(m=17), 1), (dict(acc=None), 1), (dict(acc=FAKE + 2), 1), (dict(S=FAKE + 4), 1),
    (dict(dk=64, dv=128), 2)])
def test_commit_rejects_bad_arguments(lib, kw, status):
    assert _commit(lib, **kw) == status


def test_prefill_ex_rejects_unknown_feature_map(lib):
    st = lib.la_prefill_ex(FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 8, 128, 128, 0, 0, 5, None, 0, None)
    assert st == 1


@pytest.mark.parametrize("kw,status", [
    (dict(dq=None), 1), (dict(q=FAKE + 4), 1), (dict(N=-1), 1), (dict(dk=32, dv=32), 2), (dict(dk=64, dv=128), 2)])
def test_backward_rejects_bad_arguments(lib, kw, status):
    a = dict(q=FAKE, k=FAKE, v=FAKE, do=FAKE, s0=None, dsn=None, dq=FAKE, dkk=FAKE, dvv=FAKE, ds0=None, B=1, H=1,
             N=8, dk=128, dv=128, dt=0, stream=None)
    a.update(kw)
    st = lib.la_prefill_backward(a["q"], a["k"], a["v"], a["do"], a["s0"], a["dsn"], a["dq"], a["dkk"], a["dvv"],
                                 a["ds0"], a["B"], a["H"], a["N"], a["dk"], a["dv"], a["dt"], a["stream"])
    assert st == status


def _host(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, s0=None, s_out=None, B=1, H=4, N=64, dk=128, dv=128, dt=0, group=2,
             ws=FAKE, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.la_prefill_host(a["q"], a["k"], a["v"], a["o"], a["s0"], a["s_out"], a["B"], a["H"], a["N"],
                               a["dk"], a["dv"], a["dt"], a["group"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(group=0), 1), (dict(group=-3), 1), (dict(ws=None), 1), (dict(wsb=1000), 1), (dict(ws=FAKE + 8), 1),
    (dict(q=None), 1), (dict(N=-1), 1), (dict(dk=96, dv=96), 2), (dict(dk=64, dv=128), 2)])
def test_host_prefill_rejects_bad_arguments(lib, kw, status):
    assert _host(lib, **kw) == status


def test_host_prefill_workspace_size(lib):
    # two staging buffers, each: q, k, v, o for `group` units and two states
    g, N, d = 8, 4096, 128
    per = 4 * g * N * d * 2 + 2 * g * d * d * 4
    assert lib.la_prefill_host_workspace_size(1, 64, N, d, d, 0, g) == 2 * per
    assert lib.la_prefill_host_workspace_size(1, 3, N, d, d, 0, g) == 2 * (4 * 3 * N * d * 2 + 2 * 3 * d * d * 4)
    assert lib.la_prefill_host_workspace_size(1, 64, N, d, d, 0, 0) == 0


def test_device_status_null(lib):
    assert lib.la_device_status(None, 0) == 1


def test_binding_rejects_cpu_tensors():
    import torch
    import long_context_linear_b200 as la
    x = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        la.prefill(x, x, x)

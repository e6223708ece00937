"""Device-side failure detection without a GPU fault: a bounded wait that can
never be satisfied runs out, the kernel records LA_ERR_TIMEOUT in the device
status word and exits, the host reads it, and the context keeps working."""
import pytest
import torch

import synth
from tests.parity import assert_out

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(oracle_mod):
    import long_context_linear_b200 as la
    from long_context_linear_b200 import _abi
    assert la.device_status(clear=True) == 0
    st = la.lib.la_selftest_wait_timeout(20000, None)   # 20 ms
    assert st == 0
    assert la.device_status(clear=True) == _abi.LA_ERR_TIMEOUT
    assert la.device_status(clear=True) == 0              # cleared
    # the context still runs real work correctly
    q, k, v = synth.dense(1, 2, 300, 128, "bf16", seed=9)
    o, s = la.prefill(q.cuda(), k.cuda(), v.cuda())
    ro, _ = oracle_mod.recurrent(q, k, v)
    assert_out(o.cpu(), ro, torch.bfloat16, 2)
    assert la.device_status() == 0


def test_selftest_rejects_bad_timeouts():
    import long_context_linear_b200 as la
    assert la.lib.la_selftest_wait_timeout(0, None) == 1
    assert la.lib.la_selftest_wait_timeout(2_000_000, None) == 1

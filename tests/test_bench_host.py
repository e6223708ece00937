"""Host-side accounting of bench.py (no GPU): the clock-record rule that
triggers a second measurement, and the byte / FLOP / throughput counts the
JSON line reports, against hand-computed values for the benchmark shapes."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("clocks,bad", [
    (dict(reasons=["sw_power_cap"], sm_mhz=1450.0, sm_max_mhz=1965.0), False),   # the power limit is expected
    (dict(reasons=[], sm_mhz=1965.0, sm_max_mhz=1965.0), False),
    (dict(reasons=["hw_slowdown"], sm_mhz=1900.0, sm_max_mhz=1965.0), True),
    (dict(reasons=["sw_thermal_slowdown", "sw_power_cap"], sm_mhz=1500.0, sm_max_mhz=1965.0), True),
    (dict(reasons=["hw_thermal_slowdown"], sm_mhz=1965.0, sm_max_mhz=1965.0), True),
    (dict(reasons=[], sm_mhz=1000.0, sm_max_mhz=1965.0), True),                  # held low with no reason
    (dict(reasons=["nvidia-smi unavailable"], sm_mhz=None, sm_max_mhz=None), False),
])
def test_bad_clocks_rule(bench, clocks, bad):
    assert bench.bad_clocks(clocks) is bad


def test_prefill_bytes_of_the_long_prefill(bench):
    # Q, K, V read and O written in bf16: 4 x 64 heads x 131072 tokens x 128 x 2 B, plus the fp32 state
    assert bench.prefill_bytes(1, 64, 131072, 128) == 4 * 64 * 131072 * 128 * 2 + 64 * 128 * 128 * 4
    assert bench.prefill_bytes(1, 64, 131072, 128) == 8594128896.0


def test_flop_counts(bench):
    th = 64 * 131072
    assert bench.flops_rec(th, 128) == 4 * 128 * 128 * th
    # two 64-wide value slices, each Q K^T (2*128*128), Q S (2*128*64), P V (2*128*64), K^T V (2*128*64)
    assert bench.flops_issued(th, 128) == th * 2 * (2 * 128 * 128 + 3 * 2 * 128 * 64)


def test_weak_scaling_rate(bench):
    # 131072 tokens per rank on 4 ranks in 2 ms (the slowest rank) -> 262.144 M tokens/s
    assert bench.weak_scaling_rate(131072, 4, 2.0) == pytest.approx(262.144e6)

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


def test_summary_line_is_compact_and_complete(bench):
    cb = dict(value=1.0e4, unit="tokens/s", cores=16, kind="oracle", sample="s" * 200)
    ex = dict(decode=dict(hbm_gbs=6265.1234, frac=0.957123, ms_per_step=0.345123, tokens_per_s=741234.5,
                          workload="w" * 100, cpu_baseline=cb),
              varlen=dict(tokens_per_s=1.1e8, ms_per_step=9.18, hbm_gbs=4012.3, frac=0.61, cpu_baseline=cb),
              prefill_8k=dict(tokens_per_s=1.2e8, ms_per_step=0.27, hbm_gbs=3955.4, frac=0.60, cpu_baseline=cb),
              config1_fp32=dict(us_per_step=48.1, tokens_per_s=5.3e6, tflops_rec=0.02, cpu_baseline=cb),
              backward_8k=dict(ms_per_step=0.69, hbm_gbs=2712.0, frac=0.41))
    import json
    s = bench.summary_line(ex)
    assert set(s) == {"decode_fp32_state", "varlen_resume", "prefill_8k", "config1_fp32", "backward_8k"}
    assert s["decode_fp32_state"]["hbm_gbs"] == 6265.0 and s["decode_fp32_state"]["cpu_cores"] == 16
    assert "workload" not in s["decode_fp32_state"]       # long strings stay on the extras line
    assert len(json.dumps(dict(summary=s))) < 1000       # fits the tail of the output a driver keeps


def test_oracle_baselines_on_tiny_samples(bench):
    import torch
    import synth
    q, k, v = synth.dense(2, 3, 64, 64, "fp32", seed=1)
    r = bench.oracle_dense_baseline(q, k, v, 3, "tiny", reps=2)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    S = torch.zeros(4, 64, 64)
    qs, ks, vs = synth.qkv((5, 4, 64), 64, "bf16", seed=2)
    r = bench.oracle_decode_baseline(S, qs, ks, vs, 2)
    assert r["value"] > 0 and "4 of the 16384" in r["sample"]
    parts = [tuple(x for x in synth.qkv((n, 2, 64), 64, "bf16", seed=n)) for n in (10, 7)]
    pool = torch.zeros(1, 2, 64, 64)
    r = bench.oracle_varlen_baseline(parts, [0, -1], pool)
    assert r["value"] > 0 and "17 tokens" in r["sample"] and "1 resumed" in r["sample"]

#!/usr/bin/env python
"""Benchmark of the causal linear attention hot path on B200.

Headline (one JSON line on rank 0): long prefill, B=1, H=64, N=131072, d=128,
bf16 inputs, fp32 state, zero initial state, returning O and the final S.
One step = one la_prefill call over that batch; value = prefill tokens/s
(B*N tokens per step, all ranks summed).  Inputs (6 GiB) are larger than L2,
so no flush is needed between steps.

Also measured (same timing rules): the batched decode step (B=256, H=64,
d=128, 1024 consecutive steps, achieved HBM GB/s), the ragged varlen prefill
with prefix resume (64 sequences, lengths ~U[1K,32K], H=32), the B=4, H=32,
N=8192 prefill, the fp32 B=1, H=2, N=256, d=64 configuration and further
variants, each beside the fp64 oracle timed on the host cores on a bounded
sample of the same workload.  Their detailed figures go on a line of their own
({"bench_extras": ...}) before the headline line, and the headline line ends
with a compact "summary" of them.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
headline workload instead (rank 0 only).

Multi-GPU: every rank runs the same per-GPU workload on its own inputs
(weak scaling; the units are independent, there is no data-path collective);
times are the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

HEADLINE = dict(B=1, H=64, N=131072, d=128)
DECODE = dict(B=256, H=64, d=128, steps=1024, L_lo=1024, L_hi=65536)
VARLEN = dict(n_seq=64, lo=1024, hi=32768, H=32, d=128, n_resume=32, prefix=4096)
PREFILL8K = dict(B=4, H=32, N=8192, d=128)
FEWHEADS = dict(B=1, H=8, N=131072, d=128)  # under-filled grid: the segment split applies
METRIC = "prefill tokens/s & % bf16 tensor peak at N=128K; decode-step HBM GB/s"

# DRAM traffic of one prefill launch, from one ncu capture (dram__bytes_read.sum
# + dram__bytes_write.sum) of the kernel built from sources with this hash, on
# the H=16, N=32768 case: 517.0 MB for 16*32768 token-heads.  Traffic grows
# with the token-head count, so a launch is scaled by its token-heads.  When the
# kernel sources change the figure no longer applies and is reported as null.
TRAFFIC_SOURCES = ("long_context_linear_b200/csrc/prefill_tc.cuh", "long_context_linear_b200/csrc/sm100.cuh")
TRAFFIC_HASH = "f327651e3f2dcfb9"
TRAFFIC_BYTES_PER_TOKEN_HEAD = (402.712576e6 + 113.398784e6) / (16 * 32768)


# ----------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class Dist:
    """One process per GPU (torchrun env vars); timing reductions over ranks."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cuda"

    def init(self, backend="nccl"):
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist
            self.device = "cuda" if backend == "nccl" else "cpu"

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def _reduce(self, x: float, op) -> float:
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        return x if not self.pg else self._reduce(x, self.pg.ReduceOp.MAX)

    def sum(self, x: float) -> float:
        return x if not self.pg else self._reduce(x, self.pg.ReduceOp.SUM)

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def bad_clocks(c) -> bool:
    """hw_slowdown / hw_thermal_slowdown / sw_thermal_slowdown active, or the
    median SM clock under load below 60 % of its maximum with no reason
    active; sw_power_cap alone is expected under load and kept."""
    reasons = set(c.get("reasons") or [])
    if reasons & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    sm, mx = c.get("sm_mhz"), c.get("sm_max_mhz")
    return bool(sm and mx and not reasons and sm < 0.6 * mx)


class ClockSampler:
    """nvidia-smi clock/throttle samples for one GPU while a region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        try:
            p = torch.cuda.get_device_properties(device_index)
            self.bus = "%04x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            ids = [x.strip() for x in vis.split(",")] if vis else None
            self.bus = ids[device_index] if ids and device_index < len(ids) else str(device_index)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.bus}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.15)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"], samples=0)
        time.sleep(0.05)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 8:
                rows.append(parts)
        if not rows:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["no samples"], samples=0)
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        power = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        # samples under load: SM clock at least half of its max
        load = [s for s in sm if mx and s >= 0.5 * max(mx)] or sm
        return dict(sm_mhz=statistics.median(load) if load else None, sm_max_mhz=max(mx) if mx else None,
                    reasons=reasons, samples=len(rows), power_w_max=max(power) if power else None)


def weak_scaling_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processes its own units_per_rank in the
    timed region, which lasts as long as the slowest rank (max_ms)."""
    return units_per_rank * world / (max_ms / 1e3)


def flops_rec(tokens_heads: float, d: int) -> float:
    """Algorithmic FLOPs of the recurrence: d*d multiply-adds to update S and d*d
    to form o, per token and head (4 d^2)."""
    return 4.0 * d * d * tokens_heads


def flops_issued(tokens_heads: float, d: int, C: int = 128, slice_w: int = 64) -> float:
    """FLOPs the tensor cores execute: per 64-wide value slice, Q K^T (2 C d),
    Q S (2 d w), P V (2 C w) and K^T V (2 d w) per token."""
    n_vs = d // slice_w
    return tokens_heads * n_vs * (2 * C * d + 2 * d * slice_w + 2 * C * slice_w + 2 * d * slice_w)


def measured_traffic(token_heads: float):
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != TRAFFIC_HASH:
        return None
    return TRAFFIC_BYTES_PER_TOKEN_HEAD * token_heads


def prefill_bytes(B, H, N, d) -> float:
    """Algorithmic HBM bytes: read Q, K, V, write O (bf16), write S (fp32)."""
    return 4.0 * B * H * N * d * 2 + B * H * d * d * 4


# ----------------------------------------------------------------- our arm
def timed_launches(fn, steps: int, warmup: int, dist: Dist, stream):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    total_ms = t_all0.elapsed_time(t_all1)
    per_launch = [a.elapsed_time(b) for a, b in ev]
    return total_ms, per_launch


def run_headline(args, dist: Dist, pk, sampler: ClockSampler):
    import long_context_linear_b200 as la
    import synth
    B, H, N, d = HEADLINE["B"], args.heads, args.seq, HEADLINE["d"]
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=3 + 1000 * dist.rank, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        la.prefill(q, k, v, None, out=o, s_out=s)

    sampler.start()
    total_ms, per_launch = timed_launches(step, args.steps, args.warmup, dist, stream)
    clocks = sampler.stop()
    total_ms = dist.max(total_ms)
    launch_ms = dist.max(statistics.fmean(per_launch))
    ms_step = total_ms / args.steps
    tokens = B * N * dist.world
    value = weak_scaling_rate(B * N, dist.world, ms_step)
    if (H, N) != (HEADLINE["H"], HEADLINE["N"]):
        print(f"note: headline workload overridden to H={H} N={N}", file=sys.stderr)
    th = B * H * N
    bytes_launch = prefill_bytes(B, H, N, d)
    achieved_gbs = bytes_launch / (launch_ms / 1e3) / 1e9
    f_rec = flops_rec(th, d) / (launch_ms / 1e3) / 1e12
    f_iss = flops_issued(th, d) / (launch_ms / 1e3) / 1e12

    # end to end through the public host-buffer call (la_prefill_host): pinned
    # host q, k, v in, host O and S out, every copy inside the timed region
    e2e = None
    if args.e2e_steps > 0:
        qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        sh = torch.empty(s.shape, dtype=s.dtype).pin_memory()
        group = 4
        ws = torch.empty(la.lib.la_prefill_host_workspace_size(B, H, N, d, d, 0, group), dtype=torch.uint8,
                         device=dev)

        def e2e_step():
            la.prefill_host(qh, kh, vh, None, group=group, out=oh, s_out=sh, workspace=ws)

        n_e2e = min(args.e2e_steps, args.steps)
        e_total, _ = timed_launches(e2e_step, n_e2e, 1, dist, stream)
        e_total = dist.max(e_total)
        e2e = dict(value=tokens / (e_total / n_e2e / 1e3), unit="tokens/s",
                   h2d_bytes_per_step=3 * q.numel() * q.element_size(),
                   d2h_bytes_per_step=o.numel() * o.element_size() + s.numel() * s.element_size(),
                   steps=n_e2e, call="la_prefill_host, groups of %d heads" % group)
        del qh, kh, vh, oh, sh, ws
    sample = dict(q=q[0, :2, :256].float().cpu(), k=k[0, :2, :256].float().cpu(), v=v[0, :2, :256].float().cpu())
    del q, k, v, o, s
    torch.cuda.empty_cache()
    res = dict(value=value, ms_per_step=ms_step, launch_ms=launch_ms, achieved_gbs=achieved_gbs,
               traffic=measured_traffic(th),
               bytes_launch=bytes_launch, tflops_rec=f_rec, tflops_issued=f_iss, clocks=clocks, e2e=e2e,
               launches=args.steps)
    return res, sample


def run_decode(args, dist: Dist, pk, state_dtype=torch.float32, cpu=False):
    import long_context_linear_b200 as la
    import synth
    c = DECODE
    B, H, d, steps = c["B"], c["H"], c["d"], c["steps"]
    dev = torch.device("cuda", torch.cuda.current_device())
    U = B * H
    L_seq = synth.lengths(B, c["L_lo"], c["L_hi"], seed=41 + dist.rank)
    L = [L_seq[u // H] for u in range(U)]
    S = torch.empty(U, d, d, dtype=torch.float32, device=dev)
    grp = 2048
    for u0 in range(0, U, grp):
        S[u0:u0 + grp] = synth.outer_product_state(min(grp, U - u0), d, d, L[u0:u0 + grp], seed=7 + u0, device=dev)
    S = S.view(B, H, d, d).to(state_dtype)
    qs, ks, vs = synth.qkv((steps, B, H, d), d, "bf16", seed=43 + dist.rank, device=dev)
    os_ = torch.empty_like(vs)
    stream = torch.cuda.current_stream(dev)
    it = [0]
    sample = None
    if cpu and state_dtype == torch.float32:
        # the same starting states and tokens of a seeded sample of units, for the oracle
        units = torch.tensor(synth.choose(U, CPU_DECODE_UNITS, seed=3), device=dev)
        sample = (S.view(U, d, d)[units].cpu(),) + tuple(x.view(steps, U, d)[:, units].cpu() for x in (qs, ks, vs))

    def step():
        t = it[0] % steps
        la.decode_step(qs[t], ks[t], vs[t], S, out=os_[t])
        it[0] += 1

    # warm-up, then time `steps` consecutive decode steps
    total_ms, per = timed_launches(step, steps, max(3, args.warmup), dist, stream)
    total_ms = dist.max(total_ms)
    ms_step = total_ms / steps
    esz = torch.empty(0, dtype=state_dtype).element_size()
    bytes_step = 2.0 * U * d * d * esz + 4.0 * U * d * 2
    gbs = bytes_step / (ms_step / 1e3) / 1e9
    del S, qs, ks, vs, os_
    torch.cuda.empty_cache()
    name = {torch.float32: "fp32", torch.bfloat16: "bf16", torch.float16: "fp16",
            torch.float8_e4m3fn: "fp8_e4m3", torch.float8_e5m2: "fp8_e5m2"}[state_dtype]
    res = dict(workload=f"decode B=256 H=64 d=128 bf16 q/k/v, {name} state, 1024 consecutive steps",
               hbm_gbs=gbs, peak_gbs=pk["hbm"], frac=gbs / pk["hbm"], ms_per_step=ms_step,
               bytes_per_step=bytes_step, tokens_per_s=B * dist.world / (ms_step / 1e3), steps=steps)
    if sample is not None:
        res["cpu_baseline"] = oracle_decode_baseline(*sample, H)
    return res


def run_decode_small_graph(args, dist: Dist, pk):
    """Decode at a small batch (B=4, H=64: 16 MiB of state per step), where a
    step is launch-bound: 1024 eager calls against the same 1024 steps
    captured once in a CUDA graph and replayed."""
    import long_context_linear_b200 as la
    import synth
    B, H, d, steps = 4, 64, 128, 1024
    dev = torch.device("cuda", torch.cuda.current_device())
    S0 = synth.outer_product_state(B * H, d, d, [4096] * (B * H), seed=45 + dist.rank, device=dev).view(B, H, d, d)
    qs, ks, vs = synth.qkv((steps, B, H, d), d, "bf16", seed=47 + dist.rank, device=dev)
    os_ = torch.empty_like(vs)
    S = S0.clone()
    stream = torch.cuda.current_stream(dev)

    def eager():
        for t in range(steps):
            la.decode_step(qs[t], ks[t], vs[t], S, out=os_[t])

    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        eager()
    stream.wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        eager()
    n = 3
    e_ms, _ = timed_launches(eager, n, max(3, args.warmup), dist, stream)
    g_ms, _ = timed_launches(g.replay, n, max(3, args.warmup), dist, stream)
    e_step, g_step = dist.max(e_ms) / (n * steps), dist.max(g_ms) / (n * steps)
    byts = 2.0 * B * H * d * d * 4 + 4.0 * B * H * d * 2
    del g, S, S0, qs, ks, vs, os_
    torch.cuda.empty_cache()
    return dict(workload="decode B=4 H=64 d=128, fp32 state, 1024 steps", eager_us_per_step=e_step * 1e3,
                graph_us_per_step=g_step * 1e3, tokens_per_s_eager=B * dist.world / (e_step / 1e3),
                tokens_per_s_graph=B * dist.world / (g_step / 1e3), hbm_gbs_graph=byts / (g_step / 1e3) / 1e9,
                frac_graph=byts / (g_step / 1e3) / 1e9 / pk["hbm"])


def run_speculative(args, dist: Dist, pk, m: int = 4):
    """Decode B=256, H=64 with m draft tokens per step: one verify and one
    commit of all m drafts, against m plain decode steps (same states)."""
    import long_context_linear_b200 as la
    import synth
    c = DECODE
    B, H, d = c["B"], c["H"], c["d"]
    dev = torch.device("cuda", torch.cuda.current_device())
    U = B * H
    L_seq = synth.lengths(B, c["L_lo"], c["L_hi"], seed=41 + dist.rank)
    L = [L_seq[u // H] for u in range(U)]
    S = torch.empty(U, d, d, dtype=torch.float32, device=dev)
    for u0 in range(0, U, 2048):
        S[u0:u0 + 2048] = synth.outer_product_state(min(2048, U - u0), d, d, L[u0:u0 + 2048], seed=7 + u0, device=dev)
    S = S.view(B, H, d, d)
    rounds = 64
    q, k, v = synth.qkv((rounds, B, H, m, d), d, "bf16", seed=47 + dist.rank, device=dev)
    acc = torch.full((B,), m, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    it = [0]

    def spec():
        r = it[0] % rounds
        la.decode_verify(q[r], k[r], v[r], S)
        la.decode_commit(k[r], v[r], S, acc)
        it[0] += 1

    total_ms, _ = timed_launches(spec, rounds, max(3, args.warmup), dist, stream)
    ms_spec = dist.max(total_ms) / rounds
    it[0] = 0
    o_ver = torch.empty_like(q[0])

    def verify_only():
        r = it[0] % rounds
        la.decode_verify(q[r], k[r], v[r], S, out=o_ver)
        it[0] += 1

    total_ms, _ = timed_launches(verify_only, rounds, max(3, args.warmup), dist, stream)
    ms_verify = dist.max(total_ms) / rounds
    qs, ks, vs = (x.permute(0, 3, 1, 2, 4).contiguous() for x in (q, k, v))  # [rounds, m, B, H, d]
    it[0] = 0

    def steps():
        r = it[0] % rounds
        for t in range(m):
            la.decode_step(qs[r, t], ks[r, t], vs[r, t], S)
        it[0] += 1

    total_ms, _ = timed_launches(steps, rounds, max(3, args.warmup), dist, stream)
    ms_steps = dist.max(total_ms) / rounds
    bytes_spec = 3.0 * U * d * d * 4 + 4.0 * U * m * d * 2
    # verify alone: each state read once, q, k, v read and o written
    bytes_verify = 1.0 * U * d * d * 4 + 4.0 * U * m * d * 2
    del S, q, k, v, qs, ks, vs, o_ver
    torch.cuda.empty_cache()
    return dict(workload=f"speculative decode B=256 H=64 d=128 bf16, fp32 state, m={m} drafts all accepted",
                ms_verify_commit=ms_spec, ms_m_decode_steps=ms_steps,
                tokens_per_s=B * m * dist.world / (ms_spec / 1e3),
                tokens_per_s_decode_steps=B * m * dist.world / (ms_steps / 1e3),
                hbm_gbs=bytes_spec / (ms_spec / 1e3) / 1e9, frac=bytes_spec / (ms_spec / 1e3) / 1e9 / pk["hbm"],
                ms_verify=ms_verify, verify_hbm_gbs=bytes_verify / (ms_verify / 1e3) / 1e9,
                verify_frac=bytes_verify / (ms_verify / 1e3) / 1e9 / pk["hbm"], rounds=rounds)


def run_varlen(args, dist: Dist, pk, cpu=False):
    import long_context_linear_b200 as la
    import synth
    c = VARLEN
    dev = torch.device("cuda", torch.cuda.current_device())
    lens = synth.lengths(c["n_seq"], c["lo"], c["hi"], seed=51 + dist.rank)
    cu = synth.cu_seqlens(lens).to(dev)
    T, H, d = int(cu[-1]), c["H"], c["d"]
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=53 + dist.rank, device=dev)
    resumed = synth.choose(c["n_seq"], c["n_resume"], seed=55)
    pool = synth.outer_product_state(c["n_resume"] * H, d, d, [c["prefix"]] * (c["n_resume"] * H), seed=57,
                                     device=dev).view(c["n_resume"], H, d, d)
    idx = torch.full((c["n_seq"],), -1, dtype=torch.int32)
    for j, n in enumerate(resumed):
        idx[n] = j
    idx = idx.to(dev)
    o = torch.empty_like(v)
    s = torch.empty(c["n_seq"], H, d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(la.prefill_varlen_workspace_size(c["n_seq"], T, H, d, torch.bfloat16), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        la.prefill_varlen(q, k, v, cu, pool, idx, out=o, s_out=s, workspace=ws)

    n = max(3, min(args.steps, 20))
    total_ms, per = timed_launches(step, n, max(3, args.warmup), dist, stream)
    total_ms = dist.max(total_ms)
    ms_step = total_ms / n
    byts = 4.0 * T * H * d * 2 + c["n_seq"] * H * d * d * 4 + c["n_resume"] * H * d * d * 4
    gbs = byts / (ms_step / 1e3) / 1e9
    res = dict(workload="varlen 64 seqs len~U[1K,32K] (T=%d), H=32, d=128, bf16, 32 resumed from fp32 states" % T,
               tokens_per_s=T * dist.world / (ms_step / 1e3), ms_per_step=ms_step, hbm_gbs=gbs,
               frac=gbs / pk["hbm"], tflops_rec=flops_rec(T * H, d) / (ms_step / 1e3) / 1e12, steps=n)
    if cpu:
        seqs = synth.choose(c["n_seq"], CPU_VARLEN_SEQS, seed=4)
        cuh = cu.cpu()
        parts = [(int(cuh[n]), int(cuh[n + 1]), int(idx[n])) for n in seqs]
        sub = [tuple(x[a:b].cpu() for x in (q, k, v)) for a, b, _ in parts]
        res["cpu_baseline"] = oracle_varlen_baseline(sub, [i for _, _, i in parts], pool.cpu())
    del q, k, v, o, s, pool
    torch.cuda.empty_cache()
    return res


def run_prefill8k(args, dist: Dist, pk, phi: str = "identity", d: int = 0, cpu=False):
    import long_context_linear_b200 as la
    import synth
    c = PREFILL8K
    B, H, N = c["B"], c["H"], c["N"]
    d = d or c["d"]
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=61 + dist.rank, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    # the library sizes the workspace: at this shape (full-width kernel) relu
    # and elu + 1 are both mapped on the tiles inside the prefill kernel
    ws_bytes = la.prefill_workspace_size(B, H, N, d, torch.bfloat16, phi)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    n = max(10, min(args.steps, 200))
    total_ms, per = timed_launches(lambda: la.prefill(q, k, v, None, out=o, s_out=s, phi=phi, workspace=ws), n,
                                   max(3, args.warmup), dist, stream)
    total_ms = dist.max(total_ms)
    ms_step = total_ms / n
    byts = prefill_bytes(B, H, N, d)
    gbs = byts / (ms_step / 1e3) / 1e9
    res = dict(workload=f"prefill B=4 H=32 N=8192 d={d} bf16, feature map {phi}",
               tokens_per_s=B * N * dist.world / (ms_step / 1e3),
               ms_per_step=ms_step, hbm_gbs=gbs, frac=gbs / pk["hbm"],
               tflops_rec=flops_rec(B * H * N, d) / (ms_step / 1e3) / 1e12, steps=n,
               l2="inputs (%.0f MiB) larger than L2" % (3 * B * H * N * d * 2 / 2**20))
    if cpu:
        units = torch.tensor(synth.choose(B * H, CPU_8K_UNITS, seed=1), device=dev)
        qs, ks, vs = (x.view(B * H, N, d)[units].cpu() for x in (q, k, v))
        res["cpu_baseline"] = oracle_dense_baseline(qs, ks, vs, H, f"{CPU_8K_UNITS} of the {B * H} (batch, head) "
                                                    f"units of B=4 H=32 N=8192 d={d}, all tokens")
    del q, k, v, o, s, ws
    torch.cuda.empty_cache()
    return res


def run_config1(args, dist: Dist, pk, cpu=False):
    """The fp32 correctness configuration, B=1, H=2, N=256, d=64, chunk 64, zero
    initial state (FFMA path): a latency-bound call, timed back to back."""
    import long_context_linear_b200 as la
    import synth
    B, H, N, d = 1, 2, 256, 64
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = synth.dense(B, H, N, d, "fp32", seed=1 + dist.rank, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    n = 200
    call = lambda: la.prefill(q, k, v, None, out=o, s_out=s, chunk=64)
    total_ms, _ = timed_launches(call, n, max(3, args.warmup), dist, stream)
    ms_step = dist.max(total_ms) / n
    # the same call captured in a CUDA graph (64 calls a replay): the device's
    # own time per call, without the Python binding's per-call host work
    calls = 64
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        call()
    stream.wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            call()
    reps = 10
    g_ms, _ = timed_launches(g.replay, reps, max(3, args.warmup), dist, stream)
    g_step = dist.max(g_ms) / (reps * calls)
    del g
    res = dict(workload="prefill B=1 H=2 N=256 d=64 fp32, chunk 64, zero initial state (FFMA path)",
               us_per_step=ms_step * 1e3, tokens_per_s=B * N * dist.world / (ms_step / 1e3),
               tflops_rec=flops_rec(B * H * N, d) / (ms_step / 1e3) / 1e12, steps=n,
               graph_us_per_call=g_step * 1e3, tokens_per_s_graph=B * N * dist.world / (g_step / 1e3),
               l2="inputs (256 KiB) stay in L2: a latency figure; us_per_step is one Python call back to back, "
                  "graph_us_per_call the device time of a call replayed from a CUDA graph")
    if cpu:
        res["cpu_baseline"] = oracle_dense_baseline(q.cpu(), k.cpu(), v.cpu(), 1, "the whole workload", reps=50)
    del q, k, v, o, s
    torch.cuda.empty_cache()
    return res


def run_varlen_few(args, dist: Dist, pk):
    """A packed batch of two 64K-token sequences with H=8 (32 items on 148
    SMs), with and without the segment split."""
    import long_context_linear_b200 as la
    import synth
    lens, H, d = [65536, 65536], 8, 128
    dev = torch.device("cuda", torch.cuda.current_device())
    cu = synth.cu_seqlens(lens).to(dev)
    T = sum(lens)
    q, k, v = synth.qkv((T, H, d), d, "bf16", seed=87 + dist.rank, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(len(lens), H, d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(la.prefill_varlen_workspace_size(len(lens), T, H, d, torch.bfloat16), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    n = max(10, min(args.steps, 50))
    byts = 4.0 * T * H * d * 2 + len(lens) * H * d * d * 4
    res = dict(workload="varlen 2 sequences x 65536 tokens, H=8, d=128, bf16", workspace_bytes=ws.numel(), steps=n)
    prev = os.environ.get("LA_PREFILL_SEGMENTS")
    try:
        for key, env in (("split", None), ("unsplit", "1")):
            if env is None:
                os.environ.pop("LA_PREFILL_SEGMENTS", None)
            else:
                os.environ["LA_PREFILL_SEGMENTS"] = env
            total_ms, _ = timed_launches(lambda: la.prefill_varlen(q, k, v, cu, out=o, s_out=s, workspace=ws), n,
                                         max(3, args.warmup), dist, stream)
            ms_step = dist.max(total_ms) / n
            res[key] = dict(ms_per_step=ms_step, hbm_gbs=byts / (ms_step / 1e3) / 1e9,
                            frac=byts / (ms_step / 1e3) / 1e9 / pk["hbm"])
    finally:
        if prev is None:
            os.environ.pop("LA_PREFILL_SEGMENTS", None)
        else:
            os.environ["LA_PREFILL_SEGMENTS"] = prev
    del q, k, v, o, s, ws
    torch.cuda.empty_cache()
    return res


def run_backward(args, dist: Dist, pk):
    """Gradients of the 8K prefill (dq, dk, dv, ds0 for a given dO)."""
    import long_context_linear_b200 as la
    import synth
    c = PREFILL8K
    B, H, N, d = c["B"], c["H"], c["N"], c["d"]
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=81 + dist.rank, device=dev)
    _, _, do = synth.dense(B, H, N, d, "bf16", seed=91 + dist.rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    n = max(5, min(args.steps, 20))
    total_ms, _ = timed_launches(lambda: la.prefill_backward(q, k, v, do), n, max(3, args.warmup), dist, stream)
    ms_step = dist.max(total_ms) / n
    # algorithmic bytes: q, k, v, dO read once, dq, dk, dv written once, ds0 written
    byts = 7.0 * B * H * N * d * 2 + B * H * d * d * 4
    gbs = byts / (ms_step / 1e3) / 1e9
    del q, k, v, do
    torch.cuda.empty_cache()
    res = dict(workload="backward of prefill B=4 H=32 N=8192 d=128 bf16 (three tensor-core passes)",
               tokens_per_s=B * N * dist.world / (ms_step / 1e3), ms_per_step=ms_step, hbm_gbs=gbs,
               frac=gbs / pk["hbm"], steps=n)
    # few heads, long sequence: the passes cut into segments, and unsplit
    c = FEWHEADS
    B, H, N, d = c["B"], c["H"], c["N"], c["d"]
    q, k, v = synth.dense(B, H, N, d, "bf16", seed=83 + dist.rank, device=dev)
    _, _, do = synth.dense(B, H, N, d, "bf16", seed=93 + dist.rank, device=dev)
    ws = torch.empty(max(la.lib.la_prefill_backward_workspace_size(B, H, N, d, d, 0), 1), dtype=torch.uint8,
                     device=dev)
    few = dict(workload="backward of prefill B=1 H=8 N=131072 d=128 bf16", workspace_bytes=ws.numel())
    prev = os.environ.get("LA_PREFILL_SEGMENTS")
    try:
        for key, env in (("split", None), ("unsplit", "1")):
            if env is None:
                os.environ.pop("LA_PREFILL_SEGMENTS", None)
            else:
                os.environ["LA_PREFILL_SEGMENTS"] = env
            total_ms, _ = timed_launches(lambda: la.prefill_backward(q, k, v, do, workspace=ws), n,
                                         max(3, args.warmup), dist, stream)
            few[key] = dict(ms_per_step=dist.max(total_ms) / n)
    finally:
        if prev is None:
            os.environ.pop("LA_PREFILL_SEGMENTS", None)
        else:
            os.environ["LA_PREFILL_SEGMENTS"] = prev
    res["few_heads"] = few
    del q, k, v, do, ws
    torch.cuda.empty_cache()
    return res


# FFMA path: fused multiply-adds per token and head at d = 128, C = 64 (scores
# on the diagonal half, outputs, state update: 0.28 M + 1.33 M + 1.05 M per
# 64-token chunk), and the FP32 FFMA peak (148 SMs x 128 lanes x 2 FLOP x
# 1.965 GHz)
FFMA_FMA_PER_TOKEN_HEAD = (0.28e6 + 1.33e6 + 1.05e6) / 64
FFMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_few_heads(args, dist: Dist, pk, dtype: str = "bf16"):
    """Long prefill with too few (batch, head) units to fill the GPU, once with
    the library's segment split and once with it turned off (bf16 on the
    tensor cores; fp32 on the FFMA path, over half the tokens)."""
    import long_context_linear_b200 as la
    import synth
    c = FEWHEADS
    B, H, N, d = c["B"], c["H"], c["N"], c["d"]
    fp32 = dtype == "fp32"
    if fp32:
        N //= 2
    tdt = torch.float32 if fp32 else torch.bfloat16
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = synth.dense(B, H, N, d, dtype, seed=71 + dist.rank, device=dev)
    o = torch.empty_like(v)
    s = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    ws_bytes = la.prefill_workspace_size(B, H, N, d, tdt)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    n = max(10, min(args.steps, 50))
    items = "8 unit items" if fp32 else "16 value-slice items"
    res = dict(workload=f"prefill B={B} H={H} N={N} d={d} {dtype} ({items} on 148 SMs)",
               workspace_bytes=ws_bytes, steps=n)
    byts = prefill_bytes(B, H, N, d) + (4.0 * B * H * N * d * 2 if fp32 else 0)  # fp32 Q, K, V, O: twice the bytes
    prev = os.environ.get("LA_PREFILL_SEGMENTS")
    try:
        for key, env in (("split", None), ("unsplit", "1")):
            if env is None:
                os.environ.pop("LA_PREFILL_SEGMENTS", None)
            else:
                os.environ["LA_PREFILL_SEGMENTS"] = env
            total_ms, _ = timed_launches(lambda: la.prefill(q, k, v, None, out=o, s_out=s, workspace=ws), n,
                                         max(3, args.warmup), dist, stream)
            ms_step = dist.max(total_ms) / n
            gbs = byts / (ms_step / 1e3) / 1e9
            res[key] = dict(ms_per_step=ms_step, tokens_per_s=B * N * dist.world / (ms_step / 1e3), hbm_gbs=gbs,
                            frac=gbs / pk["hbm"])
            if fp32:
                tf = 2 * FFMA_FMA_PER_TOKEN_HEAD * B * H * N / (ms_step / 1e3) / 1e12
                res[key].update(ffma_tflops=tf, ffma_frac=tf / FFMA_PEAK_TFLOPS)
    finally:
        if prev is None:
            os.environ.pop("LA_PREFILL_SEGMENTS", None)
        else:
            os.environ["LA_PREFILL_SEGMENTS"] = prev
    del q, k, v, o, s, ws
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------- oracle arm
def oracle_sample_plan(budget_s: float):
    """Heads x tokens of the headline workload the oracle processes in about
    ``budget_s`` seconds on this host's cores."""
    import oracle
    import synth
    oracle.build()
    threads = oracle.num_threads()
    heads = max(1, min(threads, HEADLINE["H"]))
    q, k, v = synth.dense(1, 1, 2048, HEADLINE["d"], "bf16", seed=0)
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v)
    per_token = (time.perf_counter() - t0) / 2048  # one thread, one head
    tokens = int(budget_s / per_token)
    tokens = max(256, min(HEADLINE["N"], tokens))
    return threads, heads, tokens


def time_oracle(heads, tokens, steps, warmup, seed=3):
    import oracle
    import synth
    q, k, v = synth.dense(1, heads, tokens, HEADLINE["d"], "bf16", seed=seed)
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    for _ in range(warmup):
        oracle.recurrent(qd, kd, vd)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.recurrent(qd, kd, vd)
    dt = (time.perf_counter() - t0) / steps
    equiv_tokens = heads * tokens / HEADLINE["H"]  # headline tokens carry 64 heads each
    return equiv_tokens / dt, dt


def cpu_baseline_line(budget_s=12.0):
    threads, heads, tokens = oracle_sample_plan(budget_s)
    value, dt = time_oracle(heads, tokens, 1, 0)
    return dict(value=value, unit="tokens/s", cores=threads, kind="oracle",
                sample=f"fp64 recurrence on {heads} of 64 heads x first {tokens} tokens of the B=1 H=64 "
                       f"N=131072 d=128 workload ({dt:.1f} s); value in headline tokens (64 heads each)")


CPU_DECODE_UNITS = 256   # (sequence, head) units of the decode batch the oracle follows over all steps
CPU_VARLEN_SEQS = 6      # sequences (all 32 heads) of the packed batch
CPU_8K_UNITS = 16        # (batch, head) units of the 8K prefill


def oracle_dense_baseline(q, k, v, heads_per_token, what, reps=1):
    """The oracle's recurrence on dense host tensors [U, N, d] (or [B, H, N, d]);
    value in workload tokens/s (a token carries ``heads_per_token`` heads)."""
    import oracle
    oracle.build()
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.recurrent(qd, kd, vd)
    dt = (time.perf_counter() - t0) / reps
    th = qd.size / qd.shape[-1]
    return dict(value=th / heads_per_token / dt, unit="tokens/s", cores=oracle.num_threads(), kind="oracle",
                sample=f"fp64 recurrence on {what} ({dt * 1e3:.1f} ms per pass)")


def oracle_decode_baseline(S, q, k, v, H):
    """The oracle's decode step over all steps of a sample of units: S [U, d, d],
    q, k, v [steps, U, d]; value in decode tokens/s (a token carries H heads)."""
    import oracle
    oracle.build()
    Sd = S.double().numpy()
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    steps, U = qd.shape[0], qd.shape[1]
    t0 = time.perf_counter()
    for t in range(steps):
        _, Sd = oracle.decode(qd[t], kd[t], vd[t], Sd)
    dt = time.perf_counter() - t0
    return dict(value=U * steps / H / dt, unit="tokens/s", cores=oracle.num_threads(), kind="oracle",
                sample=f"fp64 decode of {U} of the 16384 (sequence, head) units over all {steps} steps "
                       f"({dt:.1f} s); value in 64-head tokens")


def oracle_varlen_baseline(parts, init, pool):
    """The oracle's packed recurrence on a sample of whole sequences (all heads),
    their resumed states included; value in packed tokens/s."""
    import oracle
    import synth
    oracle.build()
    cu = synth.cu_seqlens([p[0].shape[0] for p in parts])
    q, k, v = (torch.cat([p[j] for p in parts]).double().numpy() for j in range(3))
    idx = torch.tensor(init, dtype=torch.int32)
    t0 = time.perf_counter()
    oracle.varlen(q, k, v, cu, pool, idx)
    dt = time.perf_counter() - t0
    return dict(value=q.shape[0] / dt, unit="tokens/s", cores=oracle.num_threads(), kind="oracle",
                sample=f"fp64 recurrence on {len(parts)} of the 64 sequences ({q.shape[0]} tokens, all 32 heads, "
                       f"{sum(i >= 0 for i in init)} resumed; {dt:.1f} s)")


def _r(x, n=4):
    """Rounded to n significant digits (short JSON)."""
    if x is None or isinstance(x, str):
        return x
    return float(f"{x:.{n}g}")


def summary_line(extras):
    """Compact per-config figures for the end of the headline line."""
    out = {}

    def pick(key, name, fields):
        e = extras.get(key)
        if not e:
            return
        r = {f: _r(e.get(f)) for f in fields if e.get(f) is not None}
        cb = e.get("cpu_baseline")
        if cb:
            r["cpu_tokens_per_s"] = _r(cb["value"])
            r["cpu_cores"] = cb["cores"]
        out[name] = r

    pick("decode", "decode_fp32_state", ("hbm_gbs", "frac", "ms_per_step", "tokens_per_s"))
    pick("varlen", "varlen_resume", ("tokens_per_s", "ms_per_step", "hbm_gbs", "frac"))
    pick("prefill_8k", "prefill_8k", ("tokens_per_s", "ms_per_step", "hbm_gbs", "frac"))
    pick("config1_fp32", "config1_fp32", ("us_per_step", "graph_us_per_call", "tokens_per_s", "tflops_rec"))
    pick("backward_8k", "backward_8k", ("ms_per_step", "hbm_gbs", "frac"))
    pick("speculative_m16", "verify_m16", ("ms_verify", "verify_hbm_gbs", "verify_frac"))
    return out


def reference_arm(args, dist: Dist):
    if dist.rank != 0:
        return 0
    budget = max(0.2, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    threads, heads, tokens = oracle_sample_plan(budget)
    value, dt = time_oracle(heads, tokens, args.steps, args.warmup)
    sample = (f"fp64 oracle recurrence on {heads} of 64 heads x first {tokens} tokens of the headline workload "
              f"per step; value in headline tokens (64 heads each)")
    line = dict(impl="reference", metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=dt * 1e3, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="f64", data="synthetic",
                config=dict(workload="prefill B=1 H=64 N=131072 d=128 (bf16 inputs widened to fp64)",
                            global_batch=1, seq_len=HEADLINE["N"], heads=64, head_dim=128),
                cpu_baseline=dict(value=value, unit="tokens/s", cores=threads, kind="oracle", sample=sample),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                gpu_launches=0)
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-extras", action="store_true", help="headline only (skip decode/varlen/8K)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=HEADLINE["H"], help="headline heads (smaller for profiling)")
    ap.add_argument("--seq", type=int, default=HEADLINE["N"], help="headline tokens (smaller for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    dist = Dist()
    if args.impl == "reference":
        return reference_arm(args, dist)

    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    pk = peaks()
    sampler = ClockSampler(dist.local)
    head, _ = run_headline(args, dist, pk, sampler)
    # a run that saw hardware or thermal slowdown, or SM clocks held far below
    # their maximum with no reason given (a leftover clock lock), is measured
    # once more; every rank takes the same decision
    bad = bad_clocks(head["clocks"])
    if dist.max(1.0 if bad else 0.0) > 0:
        print(f"note: clocks {head['clocks']} -> measuring the headline once more", file=sys.stderr)
        first = head["clocks"]
        head, _ = run_headline(args, dist, pk, sampler)
        head["clocks"]["remeasured_after"] = dict(reasons=first.get("reasons"), sm_mhz=first.get("sm_mhz"))
    extras = {}
    cpu_ok = dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline
    if not args.no_extras:
        extras["config1_fp32"] = run_config1(args, dist, pk, cpu_ok)
        extras["decode"] = run_decode(args, dist, pk, cpu=cpu_ok)
        # state stored in bf16 / fp16, updated in fp32 (the low-precision storage study)
        extras["decode_bf16_state"] = run_decode(args, dist, pk, torch.bfloat16)
        extras["decode_fp16_state"] = run_decode(args, dist, pk, torch.float16)
        extras["decode_fp8_e4m3_state"] = run_decode(args, dist, pk, torch.float8_e4m3fn)
        extras["decode_small_graph"] = run_decode_small_graph(args, dist, pk)
        extras["speculative_m4"] = run_speculative(args, dist, pk, 4)
        extras["speculative_m16"] = run_speculative(args, dist, pk, 16)
        extras["varlen"] = run_varlen(args, dist, pk, cpu_ok)
        extras["varlen_few_long"] = run_varlen_few(args, dist, pk)
        extras["prefill_8k"] = run_prefill8k(args, dist, pk, cpu=cpu_ok)
        extras["prefill_8k_elu1"] = run_prefill8k(args, dist, pk, "elu1")
        extras["prefill_8k_relu"] = run_prefill8k(args, dist, pk, "relu")
        extras["prefill_8k_d64"] = run_prefill8k(args, dist, pk, d=64)
        extras["few_heads"] = run_few_heads(args, dist, pk)
        extras["few_heads_fp32"] = run_few_heads(args, dist, pk, "fp32")
        extras["backward_8k"] = run_backward(args, dist, pk)
    cpu = cpu_baseline_line() if cpu_ok else None
    if dist.rank == 0:
        d = HEADLINE["d"]
        peak_note = "of measured" if pk["source"] == "measured" else "of fallback"
        line = dict(
            metric=METRIC, value=head["value"], unit="tokens/s", n_gpus=dist.world, steps=args.steps,
            warmup=args.warmup, ms_per_step=head["ms_per_step"], higher_is_better=True, scaling="weak",
            vs_baseline=None, dtype="bf16", data="synthetic (seeded N(0,1)/sqrt(d) q,k and N(0,1) v)",
            config=dict(workload=f"long prefill B=1 H={args.heads} N={args.seq} d=128, bf16 in, fp32 state, "
                                 "zero initial state, returns O and final S", global_batch=dist.world,
                        seq_len=args.seq, heads=args.heads, head_dim=d, chunk=128,
                        parallelism=f"replicas x{dist.world}",
                        l2="inputs larger than L2, no flush" if 3 * args.heads * args.seq * d * 2 > 126e6
                        else "inputs fit in L2 (profiling case)"),
            roofline=dict(bound="hbm", achieved=head["achieved_gbs"], peak=pk["hbm"], unit="GB/s",
                          frac=head["achieved_gbs"] / pk["hbm"], traffic=head["traffic"], peak_source=peak_note,
                          algorithmic_bytes_per_launch=head["bytes_launch"], launch_ms=head["launch_ms"]),
            # the launches run back to back for the whole timed region, so the
            # sustained bf16 figure is the one that applies; the burst one is given too
            tensor=dict(tflops_rec=head["tflops_rec"], tflops_issued=head["tflops_issued"],
                        frac_rec=head["tflops_rec"] / pk["bf16_sustained"],
                        frac_issued=head["tflops_issued"] / pk["bf16_sustained"],
                        peak_tflops=pk["bf16_sustained"], peak_kind="sustained",
                        peak_tflops_burst=pk["bf16"], frac_rec_of_burst=head["tflops_rec"] / pk["bf16"],
                        peak_source=peak_note),
            e2e=head["e2e"], gpu_launches=head["launches"], clocks=head["clocks"], cpu_baseline=cpu,
            summary=summary_line(extras))
        # the detailed figures of every other workload on a line of their own,
        # then the headline, whose compact summary closes the output
        if extras:
            print(json.dumps(dict(bench_extras=extras)), flush=True)
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())

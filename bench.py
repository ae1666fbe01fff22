#!/usr/bin/env python
"""Benchmark of the Wall Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (one JSON line on rank 0): fwd+bwd TFLOP/s of the training path at
T = 8192 (B=1, HQ=16, H=4, K=V=128, bf16, decaying gate g = -0.05|N|), one
step = prefix scan + forward + backward (dq, dk, dv, dg with the reverse
scan), counting causal FLOPs: forward 2 * pairs * (K + V) per head,
backward 2.5x that.  The same line carries the decode numbers (B=32,
T_kv=32768, HQ=32, H=8, K=V=128, C=64): GB/s and tokens/s of one decode
step, the cache build and prefix scan GB/s, the 64-token streaming
append loop, and the same 64 positions' queries as one chunk against the
cache (multi-token decode / chunked prefill).

Multi-GPU (one rank per GPU): every rank runs its own replica of the same
workload on its own data (weak scaling, no collective on the data path);
time is the max over ranks, value = all ranks' FLOPs / that time.  Launched
under torchrun (WORLD_SIZE set) the ranks are torchrun's; `--gpus N` with
N > 1 and no WORLD_SIZE starts the N ranks itself through
torch.distributed.run, after checking that N devices are visible.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload, in the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import datetime
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from channel_decay_softmax_b200 import inputs as I  # noqa: E402

METRIC = "fwd+bwd TFLOP/s & % of BF16 peak at T=8192; decode GB/s vs HBM peak"
# DRAM bytes (read + write) of one launch of the key-block backward kernel
# (bwd_tc_kernel) on the T=8192 workload, from the ncu capture summarized in
# profiles/; None once the kernel changed since that capture.
BWD_KEY_TRAFFIC_BYTES = 370527488 + 1171600000
# algorithmic FLOPs of each tensor-core stage per launch, as multiples of the
# forward's 2*N*(K+V): the backward's five contractions are QK^T, dO V^T, dV,
# dK (the key-block kernel) and dq (the query-block kernel, which also
# recomputes S and dP; recomputation is not algorithmic work)
STAGE_FWD_MULT = {"fwd_tc": 1.0, "bwd_keyblock": 2.0, "bwd_dq": 0.5}
# the dominant kernel of the step, timed inside the timed region
ROOF_STAGE = "bwd_keyblock"
TRAIN_CFG = 3
DECODE_CFG = 5
SM_COUNT = 148


# a timed region whose median SM clock is within this fraction of the maximum
# ran at the burst clock: its roofline takes the burst peak
AT_MAX_CLOCK = 0.97
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16, datasheet (for context only)


def pick_peak(peaks, clocks):
    """(peak TFLOP/s, name) for a kernel timed inside the bench's timed
    region: the burst figure when that region ran at the maximum SM clock
    (it is short next to the seconds-long power-capped loop the sustained
    figure comes from), else the sustained one."""
    if clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and \
            clocks["sm_mhz"] >= AT_MAX_CLOCK * clocks["sm_max_mhz"]:
        return peaks["bf16_tflops"], "bf16_tflops (burst)"
    return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    sm_max_mhz=p.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


def train_flops(s: I.Spec, T=None):
    """Algorithmic causal FLOPs of one forward and of forward+backward."""
    T = s.T if T is None else T
    pairs = I.causal_pairs(T, s.window) * s.B * s.HQ
    fwd = 2.0 * pairs * (s.K + s.V)
    return fwd, 3.5 * fwd


def decode_bytes(s: I.Spec, T_kv: int):
    """HBM bytes one decode step must move: k_tilde + v + r_cache + q +
    p_curr + o (+ lse)."""
    esz = 2 if s.dtype == torch.bfloat16 else 4
    kt = s.B * T_kv * s.HQ * s.K * esz
    v = s.B * T_kv * s.H * s.V * esz
    rc = s.B * I.ceil_div(T_kv, s.chunk) * s.HQ * s.K * 4
    small = s.B * s.HQ * (s.K * esz + s.K * 4 + s.V * esz + 4)
    return kt + v + rc + small


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 20 ms; start()
    returns once the first sample is in, mark() brackets the timed region and
    only samples stamped inside it (plus one interval after) are kept.  A
    timed region shorter than the interval may hold none: then the last
    sample before it and the first after it (each within 250 ms) stand in,
    and the record says so ("in_window": 0)."""

    INTERVAL_MS = 20

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        deadline = time.time() + 5.0
        while time.time() < deadline and os.path.getsize(self.file.name) == 0:
            time.sleep(0.02)
        return self

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        parsed = []  # (stamp, sm MHz, max MHz, reasons)
        for r in rows:
            try:
                stamp = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                why = {n for n, val in zip(names, r[6:10]) if "Active" in val and "Not" not in val}
                parsed.append((stamp, float(r[2]), float(r[3]), why))
            except (ValueError, IndexError):
                continue
        chosen, in_window = parsed, len(parsed)
        if self.t0 is not None:
            t1 = self.t1 if self.t1 is not None else float("inf")
            chosen = [x for x in parsed if self.t0 <= x[0] <= t1 + self.INTERVAL_MS * 1e-3]
            in_window = len(chosen)
            if not chosen:
                before = [x for x in parsed if self.t0 - 0.25 <= x[0] < self.t0]
                after = [x for x in parsed if t1 < x[0] <= t1 + 0.25]
                chosen = before[-1:] + after[:1]
        if not chosen:
            return None
        sm = [x[1] for x in chosen]
        smax = max(x[2] for x in chosen)
        reasons = set().union(*(x[3] for x in chosen))
        busy = [x for x in sm if x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "in_window": in_window,
                "interval_ms": self.INTERVAL_MS,
                "window_ms": (self.t1 - self.t0) * 1e3 if self.t0 and self.t1 else None}


# ---------------------------------------------------------------------------
# distributed plumbing

def dist_setup(backend="nccl", timeout_s=300):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE); the
    process group only carries the barrier and the max of the timings (the
    replicas exchange no data).  backend="gloo" runs the same plumbing on
    CPU processes."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        timeout = datetime.timedelta(seconds=timeout_s)
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout,
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=timeout)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(n: int, argv, impl: str) -> int:
    """`--gpus N` (N > 1) outside torchrun: run this script as N ranks on
    this node through torch.distributed.run (rendezvous on 127.0.0.1) and
    return its exit status.  Our arm needs N visible devices and refuses to
    start with fewer; the reference arm runs on the host cores."""
    if impl != "reference":
        have = torch.cuda.device_count()
        if have < n:
            print(f"bench.py: --gpus {n} needs {n} visible CUDA devices, found {have}",
                  file=sys.stderr, flush=True)
            return 2
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *argv]
    return subprocess.run(cmd).returncode


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg: int, rank: int) -> int:
    """Each replica's inputs: the config's seed, offset per rank."""
    return I.CONFIGS[cfg].seed + 7919 * rank


def weak_scaling_value(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


# ---------------------------------------------------------------------------
# our arm

def bench_train(args, world, rank, peaks):
    from channel_decay_softmax_b200 import api

    s = I.spec(TRAIN_CFG, seed=rank_seed(TRAIN_CFG, rank))
    x = I.training_inputs(s, device="cuda")
    q, k, v, g, dO = x["q"], x["k"], x["v"], x["g"], x["dO"]
    fwd_flops, step_flops = train_flops(s)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        # the prefix scan fused into the forward's operand pass; the
        # forward's anchored operands are reused by the backward
        o, lse, P, fws = api.wall_attn_fwd_gate(q, k, v, g, s.scale, return_workspace=True)
        if ev is not None:
            ev[1].record(stream)
        out = api.wall_attn_bwd(dO, q, k, v, P, o, lse, s.scale, fwd_workspace=fws)
        if ev is not None:
            ev[2].record(stream)
        return out

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # Timed region: the library records CUDA events (on the launch stream)
    # around the dominant kernel only, for its roofline; events around every
    # stage would add 0.03-0.07 ms to each step, so the per-stage breakdown
    # comes from a shorter instrumented pass after the timed region.
    api.timing_enable_slots([ROOF_STAGE])
    clocks = ClockSampler(torch.cuda.current_device()).start() if not args.no_clocks else None
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.mark(True)
    t0.record(stream)
    for i in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.mark(False)
    barrier(world)
    roof_stage = api.timing_read()
    api.timing_enable(False)
    clk = clocks.stop() if clocks else None
    ms = t0.elapsed_time(t1) / args.steps
    ms_max = max_over_ranks(ms, world)
    # instrumented pass: every stage's events and the fwd / bwd split
    n_inst = min(args.steps, 20)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_inst)]
    api.timing_enable(True)
    for i in range(n_inst):
        step(evs[i])
    torch.cuda.synchronize()
    stages = api.timing_read()
    api.timing_enable(False)
    stages[ROOF_STAGE] = roof_stage[ROOF_STAGE]
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # launches of this library inside one step (the ncu launch list in
    # profiles/ shows the same 13): forward: prefix chunk sums and carries 2,
    # chunk scans fused with the operand preparation 1, tcgen05 forward 1,
    # the check for units past the anchored range 1; backward (reusing the
    # forward's operands): D pre-pass 1, tcgen05 key-block (dK, dV, dS tiles)
    # 1, tcgen05 query-block dq 1, the units check 1, dk/dv group sums 1,
    # dq/dL finalize with dL's chunk sums 1, reverse-scan carries and chunk
    # scans 2
    launches_per_step = 13
    res = dict(ms=ms_max, value=weak_scaling_value(step_flops, ms_max, world) / 1e12,
               fwd_ms=fwd_ms, bwd_ms=bwd_ms,
               fwd_tflops=fwd_flops / (fwd_ms * 1e-3) / 1e12,
               bwd_tflops=2.5 * fwd_flops / (bwd_ms * 1e-3) / 1e12,
               launches=launches_per_step * args.steps, clocks=clk, spec=s, stages=stages,
               step_flops=step_flops, fwd_flops=fwd_flops)
    if not args.no_e2e:
        res["e2e"] = bench_train_e2e(args, x, s, step_flops, world)
    return res


def bench_train_e2e(args, x, s, step_flops, world):
    """The same step from pinned host buffers: every step uploads its inputs
    (q, k, v, g, dO) and downloads its gradients (dq, dk, dv, dg) inside the
    timed region, as a training input pipeline does: on three streams, the
    upload of step i+1 and the download of step i-1 overlap the compute of
    step i (device inputs and pinned host outputs double-buffered, events
    order each buffer's reuse).  Events on each stream time its own work in
    the timed steps, so the line shows which of the upload, the download and
    the compute bounds the step."""
    from channel_decay_softmax_b200 import api

    names_in = ("q", "k", "v", "g", "dO")
    host_in = {n: x[n].cpu().pin_memory() for n in names_in}
    dev_in = [{n: torch.empty_like(x[n]) for n in names_in} for _ in range(2)]
    host_out = [None, None]
    s_comp = torch.cuda.current_stream()
    s_h2d = torch.cuda.Stream()
    s_d2h = torch.cuda.Stream()
    inputs_free = [torch.cuda.Event(), torch.cuda.Event()]   # compute done with dev_in[b]
    inputs_ready = [torch.cuda.Event(), torch.cuda.Event()]  # upload into dev_in[b] done
    outputs_ready = [torch.cuda.Event(), torch.cuda.Event()]
    for e in inputs_free:
        e.record(s_comp)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    spans = {"h2d": [], "compute": [], "d2h": []}  # per timed step: (start, end) events

    def step(i, timed=False):
        b = i % 2
        d = dev_in[b]
        span = {n: (ev(), ev()) for n in spans} if timed else None
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(inputs_free[b])
            if timed:
                span["h2d"][0].record(s_h2d)
            for n in names_in:
                d[n].copy_(host_in[n], non_blocking=True)
            if timed:
                span["h2d"][1].record(s_h2d)
            inputs_ready[b].record(s_h2d)
        s_comp.wait_event(inputs_ready[b])
        if timed:
            span["compute"][0].record(s_comp)
        o, lse, P, fws = api.wall_attn_fwd_gate(d["q"], d["k"], d["v"], d["g"], s.scale,
                                                return_workspace=True)
        dq, dk, dv, dg, _, _ = api.wall_attn_bwd(d["dO"], d["q"], d["k"], d["v"], P, o, lse,
                                                 s.scale, fwd_workspace=fws)
        if timed:
            span["compute"][1].record(s_comp)
        inputs_free[b].record(s_comp)
        outputs_ready[b].record(s_comp)
        outs = (dq, dk, dv, dg)
        if host_out[b] is None:
            host_out[b] = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(outputs_ready[b])
            if timed:
                span["d2h"][0].record(s_d2h)
            for h, t in zip(host_out[b], outs):
                t.record_stream(s_d2h)  # the allocator keeps it until the copy is done
                h.copy_(t, non_blocking=True)
            if timed:
                span["d2h"][1].record(s_d2h)
        if timed:
            for n in spans:
                spans[n].append(span[n])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_h2d)
    s_comp.wait_stream(s_h2d)
    for i in range(args.steps):
        step(args.warmup + i, timed=True)
    s_d2h.wait_stream(s_comp)
    t1.record(s_d2h)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    busy = {n: statistics.mean(a.elapsed_time(b) for a, b in spans[n]) for n in spans}
    return e2e_record(world, step_flops, ms, h2d, d2h, busy)


def e2e_record(world, step_flops, ms, h2d, d2h, busy):
    """The e2e object: throughput through host buffers, bytes each way per
    step, each stream's busy time per step (its own events) and the copy
    bandwidths they imply, and the stream that bounds the step."""
    limit = max(busy, key=busy.get)
    return {"value": world * step_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "h2d_ms_per_step": busy["h2d"], "d2h_ms_per_step": busy["d2h"],
            "compute_ms_per_step": busy["compute"],
            "h2d_gbs": h2d / (busy["h2d"] * 1e-3) / 1e9,
            "d2h_gbs": d2h / (busy["d2h"] * 1e-3) / 1e9,
            "limit": limit, "limit_share": busy[limit] / ms,
            "pipelined": "3 streams: upload of step i+1 and download of step i-1 overlap "
                         "step i; every step moves its own inputs and gradients"}


def bench_decode(args, rank, peaks):
    from channel_decay_softmax_b200 import _lib as L
    from channel_decay_softmax_b200 import api

    over = {"B": args.decode_batch} if args.decode_batch else {}
    s = I.spec(DECODE_CFG, seed=rank_seed(DECODE_CFG, rank), **over)
    d = I.decode_inputs(s, device="cuda", n_query_rows=64)
    T = s.T
    n_stream = 64
    T0 = T - n_stream
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    out = {}

    def timed(fn, reps=3):
        """ms per call of fn after one warm-up call (outputs preallocated)"""
        fn()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    # prefix scan over the whole cache's gates (B*T*HQ*K elements)
    Bq, Tg, HQ, K = d["g"].shape
    P = torch.empty((Bq, Tg, HQ, K), dtype=torch.float32, device="cuda")
    ms_p = timed(lambda: L.wall_prefix_cumsum(d["g"], P, Bq, Tg, HQ, K))
    n_el = d["g"].numel()
    out["prefix_gbs"] = n_el * (2 + 4) / (ms_p * 1e-3) / 1e9
    # cache build over positions [0, T)
    kt = torch.empty((s.B, T, s.HQ, s.K), dtype=s.dtype, device="cuda")
    rc = torch.empty((s.B, I.ceil_div(T, s.chunk), s.HQ, s.K), dtype=torch.float32, device="cuda")
    ms_cb = timed(lambda: L.wall_build_kv_cache(d["k"], P, s.B, T, s.H, s.HQ, s.K, s.chunk, 0,
                                                kt, rc, T))
    cb_bytes = d["k"].numel() * 2 + P.numel() * 4 + kt.numel() * 2 + rc.numel() * 4
    out["cache_build_gbs"] = cb_bytes / (ms_cb * 1e-3) / 1e9
    p_last = P[:, -1:].contiguous()
    p_tail = P[:, T - n_stream:].contiguous()
    del P
    q_last = d["q_tail"][:, -1:].contiguous()

    def step():
        return api.wall_attn_decode(q_last, d["v"], p_last, kt, rc, scale=s.scale,
                                    cache_chunk_size=s.chunk)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    reps = max(10, args.steps)
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(reps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    nbytes = decode_bytes(s, T)
    gbs = nbytes / (ms * 1e-3) / 1e9
    out.update(decode_ms=ms, decode_gbs=gbs, decode_frac_hbm=gbs / peaks["hbm_gbs"],
               tokens_per_s=s.B / (ms * 1e-3), decode_bytes=nbytes,
               decode_launches_per_step=2)
    # the last 64 positions' queries as one chunk against the full cache
    # (multi-token decode / chunked prefill: row i at position T - 64 + i)

    def chunk():
        return api.wall_attn_decode_chunk(d["q_tail"], d["v"], p_tail, kt, rc, scale=s.scale,
                                          cache_chunk_size=s.chunk)

    for _ in range(max(3, args.warmup)):
        chunk()
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(reps):
        chunk()
    b.record(stream)
    torch.cuda.synchronize()
    ms_c = a.elapsed_time(b) / reps
    esz = 2
    c_bytes = (kt.numel() * esz + d["v"].numel() * esz + rc.numel() * 4 +
               s.B * n_stream * s.HQ * (s.K * esz + s.K * 4 + s.V * esz + 4))
    c_flops = 2.0 * s.B * s.HQ * (s.K + s.V) * sum(t + 1 for t in range(T - n_stream, T))
    out.update(chunk_rows=n_stream, chunk_ms=ms_c,
               chunk_gbs=c_bytes / (ms_c * 1e-3) / 1e9,
               chunk_frac_hbm=c_bytes / (ms_c * 1e-3) / 1e9 / peaks["hbm_gbs"],
               chunk_tokens_per_s=s.B * n_stream / (ms_c * 1e-3),
               chunk_tflops=c_flops / (ms_c * 1e-3) / 1e12, chunk_launches=2)
    del kt, rc
    torch.cuda.empty_cache()
    # streaming append loop: cache of [0, T0) then 64 appended tokens, once
    # with the one-launch fused step and once with the three-call path
    # (prefix scan, cache build + value copy, decode) from the same prefill
    cache = api.WallDecodeCache(s.B, s.H, s.HQ, s.K, s.V, capacity=T, chunk_size=s.chunk,
                                dtype=s.dtype, device="cuda", scale=s.scale)
    cache.append(d["k"][:, :T0], d["v"][:, :T0], d["g"][:, :T0])
    carry0 = cache.carry.clone()
    torch.cuda.synchronize()

    def stream_loop(fused):
        cache.length = T0
        cache.carry = carry0.clone()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(stream)
        for t in range(T0, T):
            cache.step(d["q_tail"][:, t - T0:t - T0 + 1], d["k"][:, t:t + 1],
                       d["v"][:, t:t + 1], d["g"][:, t:t + 1], fused=fused)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n_stream

    stream_loop(True)  # warm-up of both paths
    stream_loop(False)
    ms_tok = stream_loop(True)
    ms_tok3 = stream_loop(False)
    stream_bytes = sum(decode_bytes(s, t + 1) for t in range(T0, T)) / n_stream
    out.update(stream_ms_per_token=ms_tok, stream_tokens_per_s=s.B / (ms_tok * 1e-3),
               stream_gbs=stream_bytes / (ms_tok * 1e-3) / 1e9, stream_launches_per_token=1,
               stream_three_call_ms_per_token=ms_tok3,
               stream_three_call_launches_per_token=7)
    del cache, d
    torch.cuda.empty_cache()
    out["workload"] = (f"decode B={s.B} T_kv={T} HQ={s.HQ} H={s.H} K=V={s.K} C={s.chunk} bf16, "
                       f"g=-0.02|N|")
    return out


def config_fwd_flops(s: I.Spec, lengths) -> float:
    """Algorithmic forward FLOPs of a (possibly packed) batch: 2 (K + V) per
    visible (query, key) pair, summed over sequences and query heads."""
    return 2.0 * sum(I.causal_pairs(int(n), s.window) for n in lengths) * s.HQ * (s.K + s.V)


def bench_configs(args, world, rank):
    """fwd+bwd TFLOP/s of the two other training workloads, L2 flushed before
    every timed step (their working sets are near or below the 126 MB L2),
    per step (events around it) and per kernel time (the library's stage
    events, one rank's):
    config 2 (B=2, T=1024, HQ=8, H=4, K=V=64), eagerly and replayed from a
    CUDA graph (one rank's time), and config 4 (8 packed sequences of
    512-4096 rows, HQ=16, H=2, K=V=128, g_scalar, sink with dsink, window
    1024), both through the fused gate call with the backward reusing its
    operands (the autograd function's path).  Median over the timed steps,
    max over ranks; config 4 also reports its per-stage kernel times."""
    from channel_decay_softmax_b200 import api

    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = {}
    for cfg in (2, 4):
        ms, err, info = -1.0, None, {}
        try:
            s = I.spec(cfg, seed=rank_seed(cfg, rank))
            x = I.training_inputs(s, device="cuda")
            cu = x["cu_seqlens"]
            lengths = (cu[1:] - cu[:-1]).tolist() if cu is not None else [x["T"]] * x["B"]
            fwd = config_fwd_flops(s, lengths)
            kw = dict(g_scalar=x["g_scalar"], sink_bias=x["sink_bias"],
                      window_size=x["window_size"], cu_seqlens=cu)
            q, k, v, g, dO = x["q"], x["k"], x["v"], x["g"], x["dO"]
            want_dsink = x["sink_bias"] is not None

            def step():
                o, lse, P, fws = api.wall_attn_fwd_gate(q, k, v, g, s.scale,
                                                        return_workspace=True, **kw)
                api.wall_attn_bwd(dO, q, k, v, P, o, lse, s.scale, fwd_workspace=fws,
                                  want_dsink=want_dsink, **kw)
            path = "fused gate forward + backward reusing its operands" + \
                (" (with dsink)" if want_dsink else "")
            for _ in range(max(3, args.warmup)):
                step()
            n = min(max(args.steps, 10), 30)
            evs = [(ev(), ev()) for _ in range(n)]
            # the library's stage events give the device time of its own
            # kernels; the events around each step also hold any time the
            # GPU waits for the host to issue the step's launches
            api.timing_enable(True)
            try:
                for a, b in evs:
                    flush.zero_()
                    a.record(stream)
                    step()
                    b.record(stream)
                torch.cuda.synchronize()
                stages = api.timing_read()
            finally:
                api.timing_enable(False)
            ms = statistics.median(a.elapsed_time(b) for a, b in evs)
            kernel_ms = sum(t for _, t in stages.values()) / n
            graph = {}
            if cfg == 2 and world > 1:
                # no capture next to a live process group, whose watchdog
                # thread may touch CUDA while the stream is capturing
                graph = {"graph": "single-rank runs only"}
            elif cfg == 2:
                # the same step captured once in a CUDA graph and replayed:
                # one launch per step instead of the host issuing eleven
                try:
                    sg = api.WallAttnStepGraph(q, k, v, g, dO, s.scale, **kw)
                    gevs = [(ev(), ev()) for _ in range(n)]
                    for a, b in gevs:
                        flush.zero_()
                        a.record(stream)
                        sg.graph.replay()
                        b.record(stream)
                    torch.cuda.synchronize()
                    gms = statistics.median(a.elapsed_time(b) for a, b in gevs)
                    graph = dict(graph_ms_per_step=gms,
                                 graph_tflops=3.5 * fwd / (gms * 1e-3) / 1e12)
                    del sg
                except Exception as e:  # reported; the eager numbers stand
                    graph = {"graph_error": f"{type(e).__name__}: {e}"[:200]}
            info = dict(workload=f"{s.name}: B={x['B']} T={x['T']} HQ={s.HQ} H={s.H} "
                                 f"K=V={s.K}" + (f", {len(lengths)} packed sequences"
                                                 if cu is not None else "")
                                 + (f", window {s.window}" if s.window else ""),
                        path=path, fwd_bwd_flop=3.5 * fwd, timed_steps=n,
                        kernel_ms_per_step=kernel_ms,
                        stage_ms_per_step={name: t / n for name, (c, t) in stages.items() if c},
                        l2="flushed (256 MB write) before every timed step", **graph)
        except Exception as e:  # reported in the line; the headline stands
            err = f"{type(e).__name__}: {e}"[:200]
        ms = max_over_ranks(ms, world)
        if err is None and ms > 0:
            fl = info["fwd_bwd_flop"]
            info.update(ms_per_step=ms, tflops=world * fl / (ms * 1e-3) / 1e12,
                        kernel_tflops=fl / (info["kernel_ms_per_step"] * 1e-3) / 1e12)
            out[f"config{cfg}"] = info
        else:
            out[f"config{cfg}"] = {"error": err or "failed on another rank"}
    del flush
    try:
        torch.cuda.empty_cache()
    except Exception:  # a failed config above may have left the context unusable
        pass
    return out


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline leg and the reference arm)

def oracle_sample_tflops(T_sample: int):
    """fp64 oracle forward+backward on the first T_sample rows of the
    T=8192 workload (all 16 heads); returns (TFLOP/s in the bench's unit,
    seconds, threads)."""
    from oracle import wall_oracle as wo

    s = I.spec(TRAIN_CFG, T=T_sample)
    x = I.training_inputs(s)
    threads = wo.default_threads()
    t = time.perf_counter()
    wo.backward(x["q"], x["k"], x["v"], x["g"], x["dO"], scale=s.scale, nthreads=threads)
    sec = time.perf_counter() - t
    _, flops = train_flops(s)
    return flops / sec / 1e12, sec, threads


def run_reference(args, world, rank):
    if rank != 0:
        return
    T_sample = int(os.environ.get("WALL_REF_T", "768"))
    vals = []
    for _ in range(args.warmup):
        oracle_sample_tflops(T_sample)
    for _ in range(args.steps):
        vals.append(oracle_sample_tflops(T_sample))
    v = statistics.mean(x[0] for x in vals)
    sec = statistics.mean(x[1] for x in vals)
    threads = vals[0][2]
    sample = (f"fp64 oracle fwd+bwd on rows [0,{T_sample}) of the T=8192 workload, "
              f"all 16 heads, per step")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(), "sample": sample},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_name():
    s = I.spec(TRAIN_CFG)
    return (f"wall_attn fwd+bwd B={s.B} T={s.T} HQ={s.HQ} H={s.H} K=V={s.K} bf16 causal, "
            f"g=-0.05|N| (prefix scan + forward + backward incl. dg)")


def assemble_line(args, world, tr, dec, peaks, configs=None):
    """The JSON line of our arm (without the cpu_baseline leg): headline,
    per-stage table, the dominant kernel's roofline, clocks, e2e, decode.
    `tr["stages"]` maps stage names to (launches, total ms) as
    api.timing_read returns them."""
    # per-stage device time from the library's events; the dominant stage's
    # roofline uses its algorithmic FLOPs per launch over its average launch
    # time (timed inside the timed region), against the measured burst bf16
    # peak when that region ran at the maximum clock, else the sustained one
    peak, peak_name = pick_peak(peaks, tr.get("clocks"))
    stage_rows = {}
    for name, (n, ms) in tr["stages"].items():
        if n == 0:
            continue
        row = {"launches": n, "ms_per_launch": ms / n}
        if name in STAGE_FWD_MULT:
            fl = STAGE_FWD_MULT[name] * tr["fwd_flops"]
            row["algorithmic_tflop"] = fl / 1e12
            row["tflops"] = fl / (ms / n * 1e-3) / 1e12
        stage_rows[name] = row
    dom = ROOF_STAGE
    d = stage_rows[dom]
    roof = {"kernel": "bwd_tc_kernel (key-block dK, dV; also stores the dS tiles)",
            "bound": "tensor", "achieved": d["tflops"], "peak": peak, "unit": "TFLOP/s",
            "frac": d["tflops"] / peak,
            "frac_of_sustained": d["tflops"] / peaks["bf16_tflops_sustained"],
            "frac_of_nominal": d["tflops"] / NOMINAL_BF16_TFLOPS,
            "traffic": BWD_KEY_TRAFFIC_BYTES if dom == "bwd_keyblock" else None,
            "peak_source": f"{peak_name} of {peaks['source']} peaks (timed region at "
                           f"{(tr.get('clocks') or {}).get('sm_mhz')} MHz); nominal "
                           f"{NOMINAL_BF16_TFLOPS:g} TFLOP/s dense bf16 for context",
            "ms_per_launch": d["ms_per_launch"],
            "timed": "CUDA events around this kernel only, on its launch stream, over the "
                     "timed region",
            "algorithmic": "%.3g FLOP per launch = %g x the forward's 2*N*(K+V) summed "
                           "over (b,h)" % (d["algorithmic_tflop"] * 1e12, STAGE_FWD_MULT[dom])}
    line = {"metric": METRIC, "value": tr["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tr["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_name(),
                       "l2": "per-step working set ~0.45 GB > 126 MB L2 (no flush)",
                       "parallelism": f"replicas x{world}"},
            "frac_bf16_peak": tr["value"] / world / peak,
            "frac_bf16_peak_of": peak_name,
            "frac_bf16_sustained": tr["value"] / world / peaks["bf16_tflops_sustained"],
            "frac_bf16_nominal": tr["value"] / world / NOMINAL_BF16_TFLOPS,
            "fwd_tflops": tr["fwd_tflops"], "bwd_tflops": tr["bwd_tflops"],
            "roofline": roof, "stages": stage_rows, "gpu_launches": tr["launches"],
            "peaks": {k: peaks[k] for k in ("hbm_gbs", "bf16_tflops",
                                             "bf16_tflops_sustained", "source")}}
    if tr.get("clocks"):
        line["clocks"] = tr["clocks"]
    if "e2e" in tr:
        line["e2e"] = tr["e2e"]
    if dec is not None:
        line["decode"] = dec
    if configs is not None:
        line["configs"] = configs
    return line


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    # a smaller decode batch, for profiler captures (the reported decode line
    # is the full workload only without this flag)
    ap.add_argument("--decode-batch", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv), args.impl)
    if "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={os.environ['WORLD_SIZE']}; "
              f"the ranks are torchrun's", file=sys.stderr, flush=True)

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return 0

    world, rank, local = dist_setup()
    peaks = load_peaks()
    tr = bench_train(args, world, rank, peaks)
    dec = None
    if not args.no_decode:
        dec = bench_decode(args, rank, peaks)
    cfgs = None if args.no_configs else bench_configs(args, world, rank)
    barrier(world)
    if rank == 0:
        line = assemble_line(args, world, tr, dec, peaks, cfgs)
        if world == 1 and not args.no_cpu:
            # about 10-15 s of host work (the cost grows with the square of
            # the sampled rows)
            v, sec, threads = oracle_sample_tflops(int(os.environ.get("WALL_CPU_T", "4608")))
            line["cpu_baseline"] = {
                "value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                "seconds": sec,
                "sample": "fp64 oracle fwd+bwd on rows [0,%s) of the T=8192 workload, all 16 "
                          "heads" % os.environ.get("WALL_CPU_T", "4608")}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

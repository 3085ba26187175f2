#!/usr/bin/env python
"""Throughput of the TRACE capture + guided NVFP4 fake-quant hot path on B200.

One step = one pass of the whole path over one synthetic activation site:
  rollout capture of x_roll  (3 launches: zero accumulators, grid amax, quantise
                              -> FP4 codes + compact cache of mantissa bits and scales)
  guided fake-quant forward of x_train with that cache (bf16 out + STE mask)
  masked straight-through backward of an upstream gradient
  round-to-nearest fake-quant forward of x_train (the vanilla-QAT comparator)

Workload: the Qwen3-30B-A3B-shaped attention-input site, bf16 [16384, 2048],
lognormal channel scales, 1% outlier channels x100, 0.5% relative training
noise (seeded, synthetic).  L2 is flushed (256 MiB write) before every step.

The reported value is algorithmic bytes / time (GB/s): every input read once
and every output written once per kernel, x_roll read twice by capture (its
two passes).  Per-element bytes: capture 4.6875, guided 4.3125, backward
4.125, RTN 4.1875 (+4 bytes per group).  elem/s and the fraction of the
measured HBM copy bandwidth are reported beside it.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl trace|reference]
                       [--config 1..5]
--config picks another of the five workloads for the same measurement (a step
then covers every tensor of the workload; the headline is --config 2, the
default).  Under torchrun every rank runs its own sites (weak scaling, no
collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "capture & guided fake-quant fwd GB/s (elem/s) and % of B200 HBM roofline"
ROWS, COLS = 16384, 2048
WORKLOAD = "attn_in [16384 x 2048] bf16, Qwen3-30B-A3B-shaped attention-input site"
BYTES_PER_ELEM = {"capture": 4.6875, "guided_fwd": 4.3125, "ste_bwd": 4.125, "rtn_fwd": 4.1875}
KERNEL_NAMES = {"capture": "k_amax + k_capture", "guided_fwd": "k_fake_quant<1> (1-bit guided)",
                "ste_bwd": "k_ste_bwd", "rtn_fwd": "k_fake_quant<0> (round to nearest)"}
LAUNCHES_PER_STEP = 6  # zero + amax + capture, guided, bwd, rtn
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
CSRC_DIR = os.path.join(ROOT, "fp4_quantization_aware_trace_b200", "csrc")


def source_hash() -> str:
    """sha256/16 over the CUDA sources (every file of csrc/, by name)."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC_DIR)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            with open(os.path.join(CSRC_DIR, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]
PROFILE_DIR = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["trace", "reference"], default="trace")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="row chunks of the host-to-host step (copies overlap compute)")
    ap.add_argument("--eager", action="store_true",
                    help="time the step as separate launches instead of a CUDA-graph replay")
    ap.add_argument("--one-stream", action="store_true",
                    help="capture the graph on one stream (by default the round-to-nearest "
                         "comparator runs on a second stream beside the guided forward and "
                         "backward, which depend on capture only as it does)")
    ap.add_argument("--lanes", type=int, default=2,
                    help="independent sites of a multi-site workload run on this many "
                         "stream pairs inside the graph (1: one after another)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work budget of the oracle baseline leg")
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5],
                    help="workload: 1 single activation, 2 attention input (default, the "
                         "headline), 3 MoE experts, 4 KV cache, 5 later-half layer sweep")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def traffic_from_profiles(kernel_key: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or
    None when the summary is missing or the source changed since."""
    src_hash = source_hash()
    path = os.path.join(PROFILE_DIR, f"{kernel_key}_attn_in_16384x2048.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", txt)
    if not h or not t or h.group(1) != src_hash:
        return None
    return int(t.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(values, pg, device):
    """Element-wise max of per-rank device timings (one all-reduce after the
    timed region; identity with a single process)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_gbs(world: int, n_per_rank: int, bytes_per_elem: float, ms_per_step: float) -> float:
    """Whole-job algorithmic GB/s: every rank processes its own site of
    n_per_rank elements per step; the step time is the slowest rank's."""
    return world * n_per_rank * bytes_per_elem / (ms_per_step * 1e-3) / 1e9


def site_seed(rank: int) -> int:
    """Seed of rank r's site: rank 0 is the workload's own seed (1)."""
    return 1 + 1000 * rank


def make_site(rank: int, device):
    from fp4_quantization_aware_trace_b200 import inputs
    return inputs.attention_input(seed=site_seed(rank), rows=ROWS, cols=COLS, device=device)


def make_workload(cfg: int, rank: int, device):
    """(workload name, sites) of a configuration; rank r shifts every seed."""
    from fp4_quantization_aware_trace_b200 import inputs
    off = 1000 * rank
    if cfg == 1:
        return ("single activation [256 x 2048] bf16, 8 outlier channels x50",
                [inputs.single_activation(0 + off, device=device)])
    if cfg == 2:
        return WORKLOAD, [make_site(rank, device)]
    if cfg == 3:
        return ("MoE experts: 128 experts x 512 tokens, up-proj input [65536 x 2048] and "
                "down-proj input [65536 x 768] bf16, one group per expert",
                [inputs.moe_experts(2 + off, cols=2048, device=device, name="expert_up_in"),
                 inputs.moe_experts(12 + off, cols=768, device=device, name="expert_down_in")])
    if cfg == 4:
        return ("FP4 KV cache: K and V [32768 tokens, 4 heads, 128] bf16 as [131072 x 128]",
                [inputs.kv_cache(3 + off, device=device, which="k"),
                 inputs.kv_cache(3 + off, device=device, which="v")])
    sites = [inputs.layer_sweep_site(layer, k, device=device)
             for layer in (20, 21) for k in range(4)]
    if rank:
        sites = [inputs.layer_sweep_site(20 + 2 * rank + layer % 2, k, device=device)
                 for layer in (20, 21) for k in range(4)]
    return ("later-half layer sweep: 8 of the 80 sites (layers 20-21 x qkv-in, o-in, up-in, "
            "down-in), each [65536 x 4096] bf16", sites)


# ---------------------------------------------------------------------------
# CPU oracle legs (reported baseline / reference arm)
# ---------------------------------------------------------------------------

def oracle_step(oracle, xr, xt, g):
    codes, mbits, scales, gscale = oracle.capture(xr)
    out, mask = oracle.guided_fwd(xt, mbits, scales, gscale)
    oracle.fq_bwd(g, mask)
    oracle.rtn_fwd(xt, scales, gscale)


def cpu_oracle_rate(site, budget_s: float, rows: int | None = None):
    """Time the oracle, as it stands, on host copies of the workload (or its
    first `rows` rows); returns (GB/s, elem/s, seconds, sample text)."""
    import oracle
    from fp4_quantization_aware_trace_b200 import inputs
    oracle.build()
    xr, xt, g = (inputs.bits(t) for t in (site.x_roll, site.x_train, site.grad))
    if rows is not None:
        xr, xt, g = xr[:rows].copy(), xt[:rows].copy(), g[:rows].copy()
    n = xr.size
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle_step(oracle, xr, xt, g)
        passes += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    per = el / passes
    bpe = sum(BYTES_PER_ELEM.values())
    sample = (f"{passes} full step(s) (capture+guided+bwd+rtn) over the first {xr.shape[0]} of "
              f"{ROWS} rows [{xr.shape[0]} x {COLS}] of the same site, single-threaded C oracle")
    return n * bpe / per / 1e9, n / per, per, sample


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    site = make_site(0, "cpu")
    import oracle
    from fp4_quantization_aware_trace_b200 import inputs
    oracle.build()
    sample_rows = 4096
    xr, xt, g = (inputs.bits(t)[:sample_rows].copy() for t in (site.x_roll, site.x_train, site.grad))
    n = xr.size
    for _ in range(args.warmup):
        oracle_step(oracle, xr, xt, g)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(oracle, xr, xt, g)
    el = time.perf_counter() - t0
    bpe = sum(BYTES_PER_ELEM.values())
    value = n * bpe * args.steps / el / 1e9
    sample = f"each step: the first {sample_rows} of {ROWS} rows [{sample_rows} x {COLS}]"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "elem_per_s": round(n * args.steps / el, 1),
        "config": {"workload": WORKLOAD, "rows": sample_rows, "cols": COLS, "groups": 1,
                   "step": "capture + guided fwd + STE bwd + RTN fwd", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_trace(args):
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
        pg = dist

    from fp4_quantization_aware_trace_b200 import ops
    ops.library()

    workload, sites = make_workload(args.config, rank, dev)
    work = []
    for site in sites:
        R, C = site.x_roll.shape
        offs = None if site.offsets is None else site.offsets.to(dev)
        cap, ws = ops.alloc_capture(R, C, site.num_groups, dev, offs)
        w = dict(site=site, xr=site.x_roll.contiguous(), xt=site.x_train.contiguous(),
                 g=site.grad.contiguous(), offs=offs, cap=cap, ws=ws,
                 out=torch.empty_like(site.x_train), gin=torch.empty_like(site.grad),
                 out_r=torch.empty_like(site.x_train),
                 mask=torch.empty(R * C // 32, dtype=torch.int32, device=dev),
                 mask_r=torch.empty(R * C // 32, dtype=torch.int32, device=dev))
        work.append(w)
    n = sum(w["xr"].numel() for w in work)
    groups = [w["site"].num_groups for w in work]
    shapes = [list(w["xr"].shape) for w in work]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def one_site(w, e, d, s, s2):
        """capture -> guided fwd -> STE bwd on stream s; the RTN comparator on
        s2 after the capture (its only input besides x_train), or on s after
        the backward when s2 is None.  e / d: optional event lists for the
        per-kernel breakdown and the dominant kernel."""
        if e: e[0].record(s)
        ops.capture(w["xr"], w["offs"], w["cap"], w["ws"], s)
        if e: e[1].record(s)
        if s2 is not None:
            captured = torch.cuda.Event()
            captured.record(s)
            s2.wait_event(captured)
            ops.rtn_fq_fwd(w["xt"], w["cap"].scales, w["cap"].gscale, w["offs"], w["out_r"],
                           w["mask_r"], s2)
        if d: d[0].record(s)
        ops.guided_fq_fwd(w["xt"], w["cap"], w["out"], w["mask"], s)
        if e: e[2].record(s)
        if d: d[1].record(s)
        ops.fq_bwd(w["g"], w["mask"], w["gin"], s)
        if e: e[3].record(s)
        if s2 is None:
            ops.rtn_fq_fwd(w["xt"], w["cap"].scales, w["cap"].gscale, w["offs"], w["out_r"],
                           w["mask_r"], s)
        if e: e[4].record(s)

    def step(ev=None, dom=None, s=None, s2=None, lanes=None):
        """One step over every site.  Sites run one after another on s, each
        with its RTN comparator on s2 when given; with lanes (a list of (main,
        side) stream pairs) site i runs on lanes[i % len] instead, since the
        sites are independent.  Every stream used joins s at the end."""
        s = stream if s is None else s
        if lanes:
            for m, sd in lanes:
                m.wait_stream(s)  # fork
                if sd is not None:
                    sd.wait_stream(s)
            for i, w in enumerate(work):
                m, sd = lanes[i % len(lanes)]
                one_site(w, None, None, m, sd)
            for m, sd in lanes:
                s.wait_stream(m)  # join
                if sd is not None:
                    s.wait_stream(sd)
            return
        if s2 is not None:
            s2.wait_stream(s)
        for i, w in enumerate(work):
            one_site(w, ev[i] if ev else None, dom[i] if dom else None, s, s2)
        if s2 is not None:
            s.wait_stream(s2)

    for i in range(max(args.warmup, 3)):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()

    # the step captured once as a CUDA graph (all sites, every kernel of the
    # path) and replayed per step: one graph launch instead of 6 launches per
    # site, and no per-launch submission gap between the kernels
    gph, graph_error = None, None
    if not args.eager:
        try:
            gph = torch.cuda.CUDAGraph()
            cs = torch.cuda.Stream()
            cs.wait_stream(stream)
            side = None if args.one_stream else torch.cuda.Stream()
            nl = min(max(args.lanes, 1), len(work))
            lanes = ([(torch.cuda.Stream(), None if args.one_stream else torch.cuda.Stream())
                      for _ in range(nl)] if nl > 1 else None)
            # thread-local: other threads' CUDA calls (e.g. a process group's
            # watchdog) must not invalidate the capture
            with torch.cuda.graph(gph, stream=cs, capture_error_mode="thread_local"):
                if lanes:
                    step(s=cs, lanes=lanes)
                else:
                    step(s=cs, s2=side)
            torch.cuda.synchronize()
            for _ in range(max(args.warmup, 3)):
                gph.replay()
            torch.cuda.synchronize()
        except Exception as exc:  # fall back to separate launches, and say so
            gph, graph_error = None, f"{type(exc).__name__}: {exc}"[:200]

    # timed region: one event pair around every step (nothing between the
    # kernels, so each launch can overlap the tail of the previous one)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    # the dominant kernel (guided forward) is also bracketed inside the timed
    # steps, for the roofline's achieved bandwidth
    dom_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in work] for _ in range(args.steps)]
    # per-kernel breakdown: events between the calls (which can delay the
    # next launch a little, so these durations are slightly pessimistic)
    kern_ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in work]
               for _ in range(args.steps)]
    eager_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        # timed region 1 (the value): the step, graph-replayed (or eager)
        if pg: pg.barrier()
        torch.cuda.synchronize()
        for k in range(args.steps):
            flush.fill_((k + 7) & 0xFF)
            step_ev[k][0].record(stream)
            if gph is not None:
                gph.replay()
            else:
                step(dom=dom_ev[k])
            step_ev[k][1].record(stream)
        torch.cuda.synchronize()
        if pg: pg.barrier()
        # timed region 2: the same step as separate launches, with the
        # dominant kernel bracketed by events on its stream (the roofline)
        if gph is not None:
            if pg: pg.barrier()
            torch.cuda.synchronize()
            for k in range(args.steps):
                flush.fill_((k + 5) & 0xFF)
                eager_ev[k][0].record(stream)
                step(dom=dom_ev[k])
                eager_ev[k][1].record(stream)
            torch.cuda.synchronize()
            if pg: pg.barrier()
    clocks = clk.summary()
    if gph is not None:
        del gph
    for k in range(args.steps):          # breakdown pass, outside the timed region
        flush.fill_((k + 11) & 0xFF)
        step(kern_ev[k])
    torch.cuda.synchronize()

    # the next row built beyond the step: full-information guidance (the
    # cache keeps the rollout's whole codes), timed alone the same way
    full_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in work] for _ in range(args.steps)]
    for w in work:  # untimed: the first launch of a kernel also loads it
        ops.full_guided_fq_fwd(w["xt"], w["cap"], w["out"], w["mask"], stream)
    for k in range(args.steps):
        flush.fill_((k + 13) & 0xFF)
        for i, w in enumerate(work):
            full_ev[k][i][0].record(stream)
            ops.full_guided_fq_fwd(w["xt"], w["cap"], w["out"], w["mask"], stream)
            full_ev[k][i][1].record(stream)
    torch.cuda.synchronize()
    full_ms = max_over_ranks([sum(a.elapsed_time(b) for per in full_ev for a, b in per)], pg, dev)[0]

    # the mismatch diagnostic (ladder distance of RTN / 1-bit guided / full
    # guided codes from the rollout's), one histogram over all sites
    hist = torch.zeros(3, 15, dtype=torch.int64, device=dev)
    hist_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in work] for _ in range(args.steps)]
    for w in work:  # untimed warm-up launch
        ops.mismatch_histogram(w["xt"], w["cap"], hist, stream)
    for k in range(args.steps):
        flush.fill_((k + 29) & 0xFF)
        hist.zero_()
        for i, w in enumerate(work):
            hist_ev[k][i][0].record(stream)
            ops.mismatch_histogram(w["xt"], w["cap"], hist, stream)
            hist_ev[k][i][1].record(stream)
    torch.cuda.synchronize()
    hist_ms = max_over_ranks([sum(a.elapsed_time(b) for per in hist_ev for a, b in per)], pg, dev)[0]
    hist_counts = hist.cpu().tolist()

    # the cache tier: every site's compact cache captured into one record and
    # copied to pinned host memory on a copy stream while the compute stream
    # goes on; timed from the first capture to the end of the last copy
    from fp4_quantization_aware_trace_b200 import cache_tier
    # one device record per site: a smaller ring throttles the captures to
    # the copy engine (its back-pressure), which is not what is timed here
    tier = cache_tier.CacheTier(num_layers=1, keep=1, device=dev, ring=len(work))
    for i, w in enumerate(work):  # untimed: allocates records and host buffers
        tier.capture(("site", i), 0, w["xr"], w["offs"], w["cap"].codes, stream)
    torch.cuda.synchronize()
    tier_ev = []
    for k in range(args.steps):
        # each step starts with an idle copy engine (no backlog from the last)
        torch.cuda.synchronize()
        flush.fill_((k + 41) & 0xFF)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        for i, w in enumerate(work):
            tier.capture(("site", i), 0, w["xr"], w["offs"], w["cap"].codes, stream)
        ev[1].record(stream)
        ev[2].record(tier.copy_stream)
        tier_ev.append(ev)
    torch.cuda.synchronize()
    tier_compute_ms = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in tier_ev)], pg, dev)[0]
    tier_total_ms = max_over_ranks([sum(e[0].elapsed_time(e[2]) for e in tier_ev)], pg, dev)[0]
    rec_bytes = sum(cache_tier.RecordLayout.of(*w["xr"].shape, w["site"].num_groups).nbytes
                    for w in work)
    del tier

    # the MXFP4 variant on the same sites: capture, 1-bit guided, RTN and
    # full-guided forwards, each launch timed on its own
    mxc = [ops.mx_capture(w["xr"], stream=stream) for w in work]
    mx_hist = torch.zeros(3, 15, dtype=torch.int64, device=dev)

    def mx_pass(evs):
        for i, w in enumerate(work):
            ev = evs[i] if evs is not None else None
            if ev: ev[0].record(stream)
            ops.mx_capture(w["xr"], mxc[i], stream)
            if ev: ev[1].record(stream)
            ops.mx_guided_fq_fwd(w["xt"], mxc[i], w["out"], w["mask"], stream)
            if ev: ev[2].record(stream)
            ops.mx_rtn_fq_fwd(w["xt"], mxc[i].scales, w["out_r"], w["mask_r"], stream)
            if ev: ev[3].record(stream)
            ops.mx_full_guided_fq_fwd(w["xt"], mxc[i], w["out"], w["mask"], stream)
            if ev: ev[4].record(stream)
            ops.mx_mismatch_histogram(w["xt"], mxc[i], mx_hist, stream)
            if ev: ev[5].record(stream)

    # capture and guided forward with the scales in the 128 x 4 tiled layout
    # of a block-scaled FP4 GEMM
    tcap = [ops.capture_tiled(w["xr"], w["offs"], stream) for w in work]
    tws = [w["ws"] for w in work]

    def tiled_pass(evs):
        for i, w in enumerate(work):
            R, C = w["xr"].shape
            G = w["site"].num_groups
            ev = evs[i] if evs is not None else None
            if ev: ev[0].record(stream)
            ops.trace_capture_ex(w["xr"], R, C, G, w["offs"], tcap[i].codes, tcap[i].mbits,
                                 tcap[i].scales, tcap[i].gscale, tws[i], tws[i].numel(),
                                 ops.TRACE_SCALES_TILED_128x4, stream)
            if ev: ev[1].record(stream)
            ops.fq_fwd_tiled(ops.TRACE_RULE_GUIDED, w["xt"], tcap[i], w["out"], w["mask"], stream)
            if ev: ev[2].record(stream)

    tiled_pass(None)
    tl_ev = []
    for k in range(args.steps):
        flush.fill_((k + 67) & 0xFF)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in work]
        tiled_pass(evs)
        tl_ev.append(evs)
    torch.cuda.synchronize()
    tl_ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for evs in tl_ev for i in range(len(work)))
             for j in range(2)]
    tl_ms = max_over_ranks(tl_ms, pg, dev)

    # W4A8 (E4M3 activations, MX scales) on the same sites
    m8c = [ops.mx8_capture(w["xr"], stream=stream) for w in work]

    def mx8_pass(evs):
        for i, w in enumerate(work):
            ev = evs[i] if evs is not None else None
            if ev: ev[0].record(stream)
            ops.mx8_capture(w["xr"], m8c[i], stream)
            if ev: ev[1].record(stream)
            ops.mx8_guided_fq_fwd(w["xt"], m8c[i], w["out"], w["mask"], stream)
            if ev: ev[2].record(stream)
            ops.mx8_rtn_fq_fwd(w["xt"], m8c[i].scales, w["out_r"], w["mask_r"], stream)
            if ev: ev[3].record(stream)
            ops.mx8_full_guided_fq_fwd(w["xt"], m8c[i], w["out"], w["mask"], stream)
            if ev: ev[4].record(stream)

    mx8_pass(None)
    m8_ev = []
    for k in range(args.steps):
        flush.fill_((k + 97) & 0xFF)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in work]
        mx8_pass(evs)
        m8_ev.append(evs)
    torch.cuda.synchronize()
    m8_ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for evs in m8_ev for i in range(len(work)))
             for j in range(4)]
    m8_ms = max_over_ranks(m8_ms, pg, dev)
    del m8c

    mx_pass(None)  # untimed: first launches
    mx_ev = []
    for k in range(args.steps):
        flush.fill_((k + 53) & 0xFF)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in work]
        mx_pass(evs)
        mx_ev.append(evs)
    torch.cuda.synchronize()
    mx_ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for evs in mx_ev for i in range(len(work)))
             for j in range(5)]
    mx_ms = max_over_ranks(mx_ms, pg, dev)

    names = ["capture", "guided_fwd", "ste_bwd", "rtn_fwd"]
    per_kernel = {nm: 0.0 for nm in names}
    total_ms = sum(a.elapsed_time(b) for a, b in step_ev)
    eager_ms = (sum(a.elapsed_time(b) for a, b in eager_ev) if graph_error is None and not args.eager
                else total_ms)
    eager_ms = max_over_ranks([eager_ms], pg, dev)[0]
    dom_ms = sum(a.elapsed_time(b) for per in dom_ev for a, b in per)
    for per in kern_ev:
        for ev in per:
            for i, nm in enumerate(names):
                per_kernel[nm] += ev[i].elapsed_time(ev[i + 1])
    t_max = max_over_ranks([total_ms, dom_ms] + [per_kernel[nm] for nm in names], pg, dev)
    total_ms, dom_ms = t_max[0], t_max[1]
    per_kernel = {nm: t_max[i + 2] for i, nm in enumerate(names)}

    ms_step = total_ms / args.steps
    bpe = sum(BYTES_PER_ELEM.values())
    value = job_gbs(world, n, bpe, ms_step)
    hbm, peak_kind = measured_peaks()
    kern = {}
    for nm in names:
        ms = per_kernel[nm] / args.steps
        kern[nm] = {"kernel": KERNEL_NAMES[nm], "us": round(ms * 1e3, 2),
                    "gbs": round(n * BYTES_PER_ELEM[nm] / (ms * 1e-3) / 1e9, 1),
                    "elem_per_s": round(n / (ms * 1e-3), 1)}
        kern[nm]["frac_of_hbm"] = round(kern[nm]["gbs"] / hbm, 4)
    fms = full_ms / args.steps
    next_rows = {"full_guided_fwd": {
        "kernel": "k_fake_quant<kFull>", "us": round(fms * 1e3, 2),
        "gbs": round(n * 4.6875 / (fms * 1e-3) / 1e9, 1),
        "frac_of_hbm": round(n * 4.6875 / (fms * 1e-3) / 1e9 / hbm, 4),
        "bytes_per_elem": 4.6875}}
    hms = hist_ms / args.steps
    tot = max(1, sum(hist_counts[0]))
    next_rows["mismatch_histogram"] = {
        "kernel": "k_mismatch_hist", "us": round(hms * 1e3, 2),
        "gbs": round(n * 2.5625 / (hms * 1e-3) / 1e9, 1),
        "frac_of_hbm": round(n * 2.5625 / (hms * 1e-3) / 1e9 / hbm, 4),
        "bytes_per_elem": 2.5625,
        "rules": list(ops.MISMATCH_RULES),
        "disagree_frac": [round(1.0 - r[0] / tot, 6) for r in hist_counts],
        "adjacent_frac_of_disagreements": [round(r[1] / max(1, tot - r[0]), 6) for r in hist_counts],
        "counts": hist_counts}
    mx_rows = {}
    for j, (nm, kn, b_k) in enumerate([("capture", "k_mx_capture", 2.65625),
                                       ("guided_fwd", "k_mx_fake_quant<1>", 4.28125),
                                       ("rtn_fwd", "k_mx_fake_quant<0>", 4.15625),
                                       ("full_guided_fwd", "k_mx_fake_quant<2>", 4.65625),
                                       ("mismatch_histogram", "k_mismatch_hist<true>", 2.53125)]):
        ms = mx_ms[j] / args.steps
        mx_rows[nm] = {"kernel": kn, "us": round(ms * 1e3, 2), "bytes_per_elem": b_k,
                       "gbs": round(n * b_k / (ms * 1e-3) / 1e9, 1),
                       "frac_of_hbm": round(n * b_k / (ms * 1e-3) / 1e9 / hbm, 4)}
    next_rows["mxfp4"] = mx_rows
    m8_rows = {}
    for j, (nm, kn, b_k) in enumerate([("capture", "k_mx8_capture", 3.15625),
                                       ("guided_fwd", "k_mx8_fake_quant<1>", 4.28125),
                                       ("rtn_fwd", "k_mx8_fake_quant<0>", 4.15625),
                                       ("full_guided_fwd", "k_mx8_fake_quant<2>", 5.15625)]):
        ms = m8_ms[j] / args.steps
        m8_rows[nm] = {"kernel": kn, "us": round(ms * 1e3, 2), "bytes_per_elem": b_k,
                       "gbs": round(n * b_k / (ms * 1e-3) / 1e9, 1),
                       "frac_of_hbm": round(n * b_k / (ms * 1e-3) / 1e9 / hbm, 4)}
    next_rows["w4a8"] = m8_rows
    next_rows["tiled_scales"] = {
        nm: {"kernel": kn, "us": round(tl_ms[j] / args.steps * 1e3, 2), "bytes_per_elem": b_k,
             "gbs": round(n * b_k / (tl_ms[j] / args.steps * 1e-3) / 1e9, 1),
             "frac_of_hbm": round(n * b_k / (tl_ms[j] / args.steps * 1e-3) / 1e9 / hbm, 4)}
        for j, (nm, kn, b_k) in enumerate([("capture", "k_amax + k_capture<true>", 4.6875),
                                           ("guided_fwd", "k_fake_quant<1, true>", 4.3125)])}
    cms, tms = tier_compute_ms / args.steps, tier_total_ms / args.steps
    next_rows["cache_tier"] = {
        "what": "capture of every site into one compact record + one D2H copy per site to pinned "
                "host memory on a copy stream",
        "record_bytes_per_step": rec_bytes, "ring_slots": len(work),
        "bits_per_elem": round(8 * rec_bytes / n, 4),
        "capture_only_us": round(per_kernel["capture"] * 1e3 / args.steps, 2),
        "compute_stream_us": round(cms * 1e3, 2),
        "until_last_copy_us": round(tms * 1e3, 2),
        "d2h_gbs": round(rec_bytes / (tms * 1e-3) / 1e9, 2)}
    # dominant kernel: the guided forward (the largest single launch of the
    # step), timed inside the timed steps
    dom = "guided_fwd"
    dom_bytes = n * BYTES_PER_ELEM[dom]
    dom_us = dom_ms / args.steps * 1e3
    achieved = round(dom_bytes / (dom_us * 1e-6) / 1e9, 1)
    traffic = traffic_from_profiles("k_fake_quant_guided")

    # --- yardstick: the library's plain copy kernel on the same bytes -------
    ny = max(w["xr"].numel() for w in work)
    ysrc = torch.empty(ny, dtype=torch.bfloat16, device=dev).fill_(1.0)
    ydst = torch.empty_like(ysrc)
    yev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(3):
        flush.fill_(i)
        ops.trace_copy_bf16(ysrc, ydst, ny, stream)
    for k in range(args.steps):
        flush.fill_((k + 3) & 0xFF)
        yev[k][0].record(stream)
        ops.trace_copy_bf16(ysrc, ydst, ny, stream)
        yev[k][1].record(stream)
    torch.cuda.synchronize()
    y_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in yev) / args.steps], pg, dev)[0]
    yardstick = {"kernel": "k_copy", "bytes": 4 * ny, "us": round(y_ms * 1e3, 2),
                 "gbs": round(4 * ny / (y_ms * 1e-3) / 1e9, 1)}
    del ysrc, ydst

    # --- end-to-end through the C ABI with pinned host buffers -------------
    e2e = None
    if not args.no_e2e and args.config == 2:
        # through the public host-to-host API: inputs from pinned host memory,
        # every output back to it, the copies overlapped with the kernels in
        # row chunks (host_step.HostStep)
        from fp4_quantization_aware_trace_b200 import host_step
        hs = []
        for w in work:
            R, C = w["xr"].shape
            offs_h = None if w["offs"] is None else w["offs"].cpu()
            h = host_step.HostStep(R, C, offs_h, chunks=args.e2e_chunks, device=dev)
            hs.append((h, [w[k].cpu().pin_memory() for k in ("xr", "xt", "g")], h.alloc_host()))
        ins = [t for _, i, _ in hs for t in i]
        outs = [t for _, _, o in hs for t in o.values()]

        def e2e_step():
            for h, (xr_h, xt_h, g_h), out_h in hs:
                h.run(xr_h, xt_h, g_h, out_h, stream)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if pg: pg.barrier()
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], pg, dev)[0] / args.steps
        h2d = sum(t.numel() * t.element_size() for t in ins)
        d2h = sum(t.numel() * t.element_size() for t in outs)
        e2e = {"value": round(job_gbs(world, n, bpe, e2e_ms), 3), "unit": "GB/s",
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": f"host_step.HostStep.run, {len(hs[0][0].cuts)} row chunks",
               "elem_per_s": round(world * n / (e2e_ms * 1e-3), 1)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == 2:
        gbs, eps, per, sample = cpu_oracle_rate(work[0]["site"], args.cpu_seconds)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": sample, "elem_per_s": round(eps, 1), "s_per_step": round(per, 3)}

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "elem_per_s": round(world * n / (ms_step * 1e-3), 1),
        "frac_of_hbm": round(value / world / hbm, 4),
        "config": {"workload": workload, "shapes": shapes, "groups": groups,
                   "step": "capture + guided fwd + STE bwd + RTN fwd",
                   "l2": "flushed before every step (256 MiB write)",
                   "launch": (("CUDA graph of the whole step, captured once and replayed"
                               + ("" if args.one_stream else
                                  "; the RTN comparator on a second stream beside the guided "
                                  "forward and the backward")
                              + (f"; sites on {min(max(args.lanes, 1), len(work))} stream lanes"
                                 if min(max(args.lanes, 1), len(work)) > 1 else ""))
                              if graph_error is None and not args.eager else
                              "separate launches (programmatic stream serialization)"),
                   "parallelism": f"{world} independent sites, one per GPU (no collective)"},
        "kernels": kern,
        "yardstick": yardstick,
        "next_rows": next_rows,
        "roofline": {"bound": "hbm", "kernel": KERNEL_NAMES[dom], "achieved": achieved,
                     "us_per_launch": round(dom_us, 2),
                     "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": traffic,
                     "algorithmic_bytes": int(dom_bytes)},
        "cpu_baseline": cpu,
        "e2e": e2e,
        # the graph replays launch the same kernels as separate steps do;
        # with the graph there is also the eager pass for the roofline
        "gpu_launches": LAUNCHES_PER_STEP * len(work) * args.steps *
                        (2 if graph_error is None and not args.eager else 1),
        "eager_ms_per_step": round(eager_ms / args.steps, 5),
        "graph_error": graph_error,
        "timing": ("value: events around each step (graph replay) only; roofline: events around "
                   "the guided forward in a second timed pass of eager steps; kernels: a third, "
                   "untimed pass with events between the calls"),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_trace(args)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of the TRACE capture + guided NVFP4 fake-quant hot path on B200.

One step = one pass of the whole path over every site of the workload:
  rollout capture of x_roll  (grid amax, grid barrier, then quantise -> FP4
                              codes + compact cache of mantissa bits and
                              scales; one cooperative launch)
  guided fake-quant forward of x_train with that cache (bf16 out + STE mask)
  masked straight-through backward of an upstream gradient
  round-to-nearest fake-quant forward of x_train (the vanilla-QAT comparator)

Default workload (the headline): the later-half layer sweep, all 80 sites --
layers 20..39 of 40 x {qkv-in, o-in, expert up-in, expert down-in}, each
[65536, 4096] bf16, lognormal channel scales, 1% outlier channels x100, 0.5%
relative training noise (seeded, synthetic).  All 80 sites' x_roll, x_train
and grad (120 GiB) stay resident in HBM; every input is read from HBM once
per step (far larger than the 126 MB L2, so no flush is needed between
steps).  The attention-input site [16384, 2048], the MoE expert inputs and
the KV cache follow as secondary lines (`secondary`), with L2 flushed before
every step.

The value is algorithmic bytes / time (GB/s): every input read once and every
output written once per kernel, x_roll read twice by capture (its amax and
quantising phases).  Per-element bytes: capture 4.6875, guided 4.3125, backward 4.125,
RTN 4.1875 (+4 bytes per group).  elem/s is reported beside it, and
`algo_bytes_over_copy_peak` divides the step's algorithmic GB/s by the
measured copy bandwidth -- not a DRAM fraction: reads that hit L2 count too.
The per-kernel `roofline` is the HBM fraction of the dominant kernel.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl trace|reference]
                       [--config 1..5]
--config picks one of the five workloads (1 single activation, 2 attention
input, 3 MoE experts, 4 KV cache, 5 the layer sweep: default).  --gpus N > 1
without torchrun starts N ranks itself (torch.distributed.run on 127.0.0.1);
every rank runs its own draw of the workload (weak scaling, no collective on
the data path) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import socket
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "capture & guided fake-quant fwd GB/s (elem/s) and % of B200 HBM roofline"
HEADLINE_CONFIG = 5
SECONDARY_CONFIGS = (2, 3, 4)
BYTES_PER_ELEM = {"capture": 4.6875, "guided_fwd": 4.3125, "ste_bwd": 4.125, "rtn_fwd": 4.1875}
STEP_BYTES_PER_ELEM = sum(BYTES_PER_ELEM.values())
KERNEL_NAMES = {"capture": "k_capture_coop (amax, grid barrier, quantise)",
                "guided_fwd": "k_fake_quant<1> (1-bit guided)",
                "ste_bwd": "k_ste_bwd", "rtn_fwd": "k_fake_quant<0> (round to nearest)"}
# kernels of the library launched per site and step: capture (one
# cooperative launch), guided forward, backward, RTN
LAUNCHES_PER_SITE = 4
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 * 10 ** 6
CSRC_DIR = os.path.join(ROOT, "fp4_quantization_aware_trace_b200", "csrc")
PROFILE_DIR = os.path.join(ROOT, "profiles")
# row windows of the CPU legs (whole rows; about 80 M elements for the
# baseline leg, 20 M per step for the reference arm)
CPU_SAMPLE_ELEMS = 80 * 2 ** 20
REF_SAMPLE_ELEMS = 20 * 2 ** 20


def source_hash() -> str:
    """sha256/16 over the CUDA sources (every file of csrc/, by name)."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC_DIR)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            with open(os.path.join(CSRC_DIR, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["trace", "reference"], default="trace")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="row chunks of the host-to-host step (copies overlap compute)")
    ap.add_argument("--e2e-steps", type=int, default=2,
                    help="timed end-to-end steps (each covers every site)")
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
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the secondary lines (attention input, MoE experts, KV cache) "
                         "after the headline")
    ap.add_argument("--next-sites", type=int, default=8,
                    help="sites of the workload the next-row legs (full guidance, "
                         "histogram, MXFP4, W4A8, tiled scales, cache tier) run on")
    ap.add_argument("--sites", type=int, default=0,
                    help="run only the first N sites of the workload (0: all; for profiling "
                         "one site of the layer sweep)")
    ap.add_argument("--plumbing-only", action="store_true",
                    help="run only the multi-rank plumbing (launch, process group over gloo, "
                         "max over ranks) on CPU, without any GPU work; prints one JSON line")
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG, choices=[1, 2, 3, 4, 5],
                    help="workload: 1 single activation, 2 attention input, 3 MoE experts, "
                         "4 KV cache, 5 later-half layer sweep (default, the headline)")
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_launch_cmd(argv: list[str], gpus: int, port: int) -> list[str]:
    """Command that runs this script on `gpus` ranks of one node (one
    process per GPU) with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1",
            f"--master-port={port}", os.path.abspath(__file__), *argv]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def traffic_from_profiles(kernel_key: str, tag: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary
    `profiles/<kernel_key>_<tag>.md`, or None when the summary is missing or
    the source changed since."""
    path = os.path.join(PROFILE_DIR, f"{kernel_key}_{tag}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", txt)
    if not h or not t or h.group(1) != source_hash():
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
        self.lines = []

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
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines += [l for l in out.splitlines() if l.strip()]

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
    """Whole-job algorithmic GB/s: every rank processes its own draw of the
    workload (n_per_rank elements per step); the step time is the slowest
    rank's."""
    return world * n_per_rank * bytes_per_elem / (ms_per_step * 1e-3) / 1e9


def site_seed(rank: int) -> int:
    """Seed of rank r's attention-input site: rank 0 is the workload's own seed (1)."""
    return 1 + 1000 * rank


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------

WORKLOAD_NAMES = {
    1: "single activation [256 x 2048] bf16, 8 outlier channels x50",
    2: "attn_in [16384 x 2048] bf16, Qwen3-30B-A3B-shaped attention-input site",
    3: ("MoE experts: 128 experts x 512 tokens, up-proj input [65536 x 2048] and down-proj "
        "input [65536 x 768] bf16, one group per expert"),
    4: "FP4 KV cache: K and V [32768 tokens, 4 heads, 128] bf16 as [131072 x 128]",
    5: ("later-half layer sweep: all 80 sites (layers 20-39 of 40 x qkv-in, o-in, up-in, "
        "down-in), each [65536 x 4096] bf16"),
}
WORKLOAD_TAGS = {1: "single_256x2048", 2: "attn_in_16384x2048", 3: "moe_experts_g128",
                 4: "kv_cache_131072x128", 5: "layer_sweep_65536x4096"}


def workload_shapes(cfg: int) -> list[tuple[int, int]]:
    """[rows, cols] of every site of a configuration (without drawing it)."""
    return {1: [(256, 2048)], 2: [(16384, 2048)], 3: [(65536, 2048), (65536, 768)],
            4: [(131072, 128)] * 2, 5: [(65536, 4096)] * 80}[cfg]


def workload_sites(cfg: int, rank: int, device):
    """The sites of a configuration, generated one at a time (a generator);
    rank r draws its own copy of the recipe (every seed shifted)."""
    from fp4_quantization_aware_trace_b200 import inputs
    off = 1000 * rank
    if cfg == 1:
        yield inputs.single_activation(0 + off, device=device)
    elif cfg == 2:
        yield inputs.attention_input(seed=site_seed(rank), device=device)
    elif cfg == 3:
        yield inputs.moe_experts(2 + off, cols=2048, device=device, name="expert_up_in")
        yield inputs.moe_experts(12 + off, cols=768, device=device, name="expert_down_in")
    elif cfg == 4:
        yield inputs.kv_cache(3 + off, device=device, which="k")
        yield inputs.kv_cache(3 + off, device=device, which="v")
    else:
        for layer in range(20, 40):
            for k in range(len(inputs.LAYER_SWEEP_SITES)):
                yield inputs.layer_sweep_site(layer, k, device=device, seed_offset=off)


# ---------------------------------------------------------------------------
# CPU oracle legs (reported baseline / reference arm)
# ---------------------------------------------------------------------------

def site_sample(site, rows_per_site: int, index: int):
    """Host copies of a window of whole rows of a site plus the global scale
    of each of those rows, taken from the whole tensor's per-group amax (so
    the window is quantised exactly as it is inside the whole tensor).
    The window starts at a seeded row; the amax is taken with torch on the
    tensor's own device, the global scale with the oracle."""
    import numpy as np

    import oracle
    from fp4_quantization_aware_trace_b200 import inputs
    R, C = site.x_roll.shape
    k = min(R, max(1, rows_per_site))
    a = int(np.random.default_rng(1234 + index).integers(0, R - k + 1))
    offs = None if site.offsets is None else site.offsets.cpu().numpy()
    mags = site.x_roll.abs()
    if offs is None:
        amax = [float(mags.max())]
    else:
        amax = [float(mags[int(offs[g]):int(offs[g + 1])].max()) if offs[g + 1] > offs[g] else 0.0
                for g in range(len(offs) - 1)]
    gs = np.array([oracle.global_scale(m) for m in amax], np.float32)
    if offs is None:
        rg = np.full(k, gs[0], np.float32)
    else:
        rg = np.repeat(gs, np.diff(offs)).astype(np.float32)[a:a + k].copy()
    xr, xt, g = (inputs.bits(t[a:a + k]) for t in (site.x_roll, site.x_train, site.grad))
    return {"xr": xr, "xt": xt, "g": g, "rg": rg}


def oracle_sample_step(samples, threads: int):
    """The oracle's whole step on every sample, threaded over row chunks:
    amax pass, capture, guided forward, backward, round-to-nearest forward."""
    import oracle.threaded as ot
    for s in samples:
        ot.group_amax_mt(s["xr"], threads=threads)
        codes, mbits, scales = ot.capture_rows_mt(s["xr"], s["rg"], threads)
        _, mask = ot.fake_quant_rows_mt(s["xt"], s["rg"], scales, mbits, threads)
        ot.fq_bwd_mt(s["g"], mask, threads)
        ot.fake_quant_rows_mt(s["xt"], s["rg"], scales, None, threads)


def rows_per_site(cfg: int, shapes, budget_elems: int) -> int:
    n_sites = len(shapes)
    cols = max(c for _, c in shapes)
    return max(1, budget_elems // (n_sites * cols))


def cpu_baseline_leg(cfg: int, sites, budget_elems: int = CPU_SAMPLE_ELEMS, repeats: int = 2):
    """The oracle, as it stands, threaded over every core of this process,
    on a window of rows of every site; returns the cpu_baseline object."""
    import oracle
    import oracle.threaded as ot
    oracle.build()
    shapes = [tuple(s.x_roll.shape) for s in sites]
    rps = rows_per_site(cfg, shapes, budget_elems)
    samples = [site_sample(s, rps, i) for i, s in enumerate(sites)]
    n = sum(s["xr"].size for s in samples)
    threads = ot.cores()
    oracle_sample_step(samples[:1], threads)  # untimed: library load, pool start
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle_sample_step(samples, threads)
    per = (time.perf_counter() - t0) / repeats
    return {"value": round(n * STEP_BYTES_PER_ELEM / per / 1e9, 4), "unit": "GB/s",
            "cores": threads, "host_cores": os.cpu_count(), "kind": "oracle",
            "elem_per_s": round(n / per, 1), "s_per_step": round(per, 3),
            "sample": (f"{repeats} passes of the whole step (amax, capture, guided fwd, STE bwd, "
                       f"RTN fwd) over a window of {min(rps, shapes[0][0])} whole rows of each of "
                       f"the {len(sites)} sites ({n} elements), each window quantised with its "
                       f"tensor's whole-tensor global scale; the C oracle threaded over row "
                       f"chunks on {threads} cores")}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    import oracle
    import oracle.threaded as ot
    oracle.build()
    # the inputs are drawn where the GPU arm draws them (same values), one
    # site at a time; only each site's row window is kept, on the host
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dev = torch.device("cuda", local)
    else:
        dev = torch.device("cpu")
    shapes = workload_shapes(args.config)
    # the row window per site is fixed by the step budget and the shapes
    rps = rows_per_site(args.config, shapes, REF_SAMPLE_ELEMS)
    samples = []
    for i, site in enumerate(workload_sites(args.config, 0, dev)):
        samples.append(site_sample(site, rps, i))
        del site
    if dev.type == "cuda":
        torch.cuda.empty_cache()
    n = sum(s["xr"].size for s in samples)
    threads = ot.cores()
    for _ in range(args.warmup):
        oracle_sample_step(samples, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(samples, threads)
    el = time.perf_counter() - t0
    value = n * STEP_BYTES_PER_ELEM * args.steps / el / 1e9
    sample = (f"each step: the oracle's whole step over a window of {min(rps, shapes[0][0])} "
              f"whole rows of each of the {len(shapes)} sites ({n} elements), each window "
              f"quantised with its tensor's whole-tensor global scale; threaded over row "
              f"chunks on {threads} cores")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "elem_per_s": round(n * args.steps / el, 1),
        "config": {"workload": WORKLOAD_NAMES[args.config], "shapes": [list(s) for s in shapes],
                   "rows_per_site": min(rps, shapes[0][0]),
                   "step": "capture + guided fwd + STE bwd + RTN fwd", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def _ev():
    return torch.cuda.Event(enable_timing=True)


def _pair():
    return (_ev(), _ev())


class Workload:
    """The sites of a configuration resident on the device, with what the
    step writes: each site keeps its compact cache (mantissa bits, scales,
    global scales); the FP4 codes and the forward / backward outputs live in
    one set of buffers per stream lane (sites on one lane run in order)."""

    def __init__(self, cfg: int, rank: int, dev, lanes: int, max_sites: int = 0):
        from fp4_quantization_aware_trace_b200 import ops
        self.cfg, self.dev = cfg, dev
        self.sites = []
        for site in workload_sites(cfg, rank, dev):
            self.sites.append(site)
            if max_sites and len(self.sites) >= max_sites:
                break
        self.nl = max(1, min(lanes, len(self.sites)))
        nmax = max(s.x_roll.numel() for s in self.sites)
        i32, bf = torch.int32, torch.bfloat16
        self.lane_buf = [dict(codes=torch.empty(nmax // 2, dtype=torch.uint8, device=dev),
                              out=torch.empty(nmax, dtype=bf, device=dev),
                              gin=torch.empty(nmax, dtype=bf, device=dev),
                              out_r=torch.empty(nmax, dtype=bf, device=dev),
                              mask=torch.empty(nmax // 32, dtype=i32, device=dev),
                              mask_r=torch.empty(nmax // 32, dtype=i32, device=dev))
                         for _ in range(self.nl)]
        self.work = []
        for i, site in enumerate(self.sites):
            R, C = site.x_roll.shape
            n = R * C
            lb = self.lane_buf[i % self.nl]
            offs = None if site.offsets is None else site.offsets.to(dev)
            G = site.num_groups
            cap = ops.Capture(codes=lb["codes"][:n // 2],
                              mbits=torch.empty(n // 32, dtype=i32, device=dev),
                              scales=torch.empty(R, C // 16, dtype=torch.uint8, device=dev),
                              gscale=torch.empty(G, dtype=torch.float32, device=dev),
                              offsets=offs)
            ws = torch.zeros(max(ops.trace_capture_workspace_bytes(R, C, G), 256),
                             dtype=torch.uint8, device=dev)
            self.work.append(dict(
                site=site, xr=site.x_roll, xt=site.x_train, g=site.grad, offs=offs, cap=cap, ws=ws,
                lane=i % self.nl, out=lb["out"][:n].view(R, C), gin=lb["gin"][:n].view(R, C),
                out_r=lb["out_r"][:n].view(R, C), mask=lb["mask"][:n // 32],
                mask_r=lb["mask_r"][:n // 32]))
        self.n = sum(w["xr"].numel() for w in self.work)
        self.shapes = [list(w["xr"].shape) for w in self.work]
        self.groups = [w["site"].num_groups for w in self.work]
        self.resident_bytes = sum(3 * w["xr"].numel() * 2 for w in self.work)

    def large(self) -> bool:
        """Inputs far beyond L2 (a step streams many times the L2 through
        it before any input comes round again): no flush between steps."""
        return self.resident_bytes > 16 * L2_BYTES


def one_site(w, e, d, s, s2):
    """capture -> guided fwd -> STE bwd on stream s; the RTN comparator on s2
    after the capture (its only input besides x_train), or on s after the
    backward when s2 is None.  e / d: optional event lists for the
    per-kernel breakdown and the dominant kernel."""
    from fp4_quantization_aware_trace_b200 import ops
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
    if d: d[1].record(s)
    if e: e[2].record(s)
    ops.fq_bwd(w["g"], w["mask"], w["gin"], s)
    if e: e[3].record(s)
    if s2 is None:
        ops.rtn_fq_fwd(w["xt"], w["cap"].scales, w["cap"].gscale, w["offs"], w["out_r"],
                       w["mask_r"], s)
    if e: e[4].record(s)


def run_step(work, stream, ev=None, dom=None, s=None, s2=None, lanes=None):
    """One step over every site.  Sites run one after another on s, each with
    its RTN comparator on s2 when given; with lanes (a list of (main, side)
    stream pairs) site i runs on lanes[i % len] instead -- the sites are
    independent, and site i's output buffers belong to that lane.  Every
    stream used joins s at the end."""
    s = stream if s is None else s
    if lanes:
        for m, sd in lanes:
            m.wait_stream(s)  # fork
            if sd is not None:
                sd.wait_stream(s)
        for w in work:
            m, sd = lanes[w["lane"] % len(lanes)]
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


class L2Flush:
    """L2 flush between timed iterations: a 256 MiB write (every line of
    the 126 MB L2 replaced), then a read of another 256 MiB buffer, which
    writes the flush's dirty lines back to HBM before the next timed kernel
    starts instead of during it.  `fill_(v)` runs both on the current
    stream."""

    def __init__(self, dev):
        self.wr = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.rd = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        self.sink = torch.empty((), dtype=torch.int64, device=dev)

    def fill_(self, v: int):
        self.wr.fill_(v)
        torch.sum(self.rd, dim=0, out=self.sink)


def measure_step(args, wl: Workload, pg, dev, clk, flush):
    """Time the step over a resident workload: (1) graph-replayed steps (the
    value), (2) the same steps as separate launches with events around the
    dominant kernel (the roofline), (3) an untimed pass with events between
    every call (the per-kernel breakdown).  Returns a dict of max-over-rank
    milliseconds."""
    work = wl.work
    stream = torch.cuda.current_stream()
    do_flush = not wl.large()

    def flush_l2(k):
        if do_flush:
            flush.fill_(k & 0xFF)

    for i in range(max(args.warmup, 3)):
        flush_l2(i)
        run_step(work, stream)
    torch.cuda.synchronize()

    gph, graph_error = None, None
    nl = wl.nl
    if not args.eager:
        try:
            gph = torch.cuda.CUDAGraph()
            cs = torch.cuda.Stream()
            cs.wait_stream(stream)
            side = None if args.one_stream else torch.cuda.Stream()
            lanes = ([(torch.cuda.Stream(), None if args.one_stream else torch.cuda.Stream())
                      for _ in range(nl)] if nl > 1 else None)
            # thread-local: other threads' CUDA calls (e.g. a process group's
            # watchdog) must not invalidate the capture
            with torch.cuda.graph(gph, stream=cs, capture_error_mode="thread_local"):
                if lanes:
                    run_step(work, stream, s=cs, lanes=lanes)
                else:
                    run_step(work, stream, s=cs, s2=side)
            torch.cuda.synchronize()
            for _ in range(max(args.warmup, 3)):
                gph.replay()
            torch.cuda.synchronize()
        except Exception as exc:  # fall back to separate launches, and say so
            gph, graph_error = None, f"{type(exc).__name__}: {exc}"[:200]

    K = args.steps
    step_ev = [_pair() for _ in range(K)]
    dom_ev = [[_pair() for _ in work] for _ in range(K)]
    kern_ev = [[[_ev() for _ in range(5)] for _ in work] for _ in range(K)]
    eager_ev = [_pair() for _ in range(K)]
    with clk:
        # timed region 1 (the value): the step, graph-replayed (or eager)
        if pg: pg.barrier()
        torch.cuda.synchronize()
        for k in range(K):
            flush_l2(k + 7)
            step_ev[k][0].record(stream)
            if gph is not None:
                gph.replay()
            else:
                run_step(work, stream, dom=dom_ev[k])
            step_ev[k][1].record(stream)
        torch.cuda.synchronize()
        if pg: pg.barrier()
        # timed region 2: the same steps as separate launches, with the
        # dominant kernel bracketed by events on its stream (the roofline)
        if gph is not None:
            if pg: pg.barrier()
            torch.cuda.synchronize()
            for k in range(K):
                flush_l2(k + 5)
                eager_ev[k][0].record(stream)
                run_step(work, stream, dom=dom_ev[k])
                eager_ev[k][1].record(stream)
            torch.cuda.synchronize()
            if pg: pg.barrier()
    if gph is not None:
        del gph
    for k in range(K):  # breakdown pass, outside the timed region
        flush_l2(k + 11)
        run_step(work, stream, ev=kern_ev[k])
    torch.cuda.synchronize()

    names = ["capture", "guided_fwd", "ste_bwd", "rtn_fwd"]
    total = sum(a.elapsed_time(b) for a, b in step_ev)
    eager = (sum(a.elapsed_time(b) for a, b in eager_ev) if graph_error is None and not args.eager
             else total)
    dom = sum(a.elapsed_time(b) for per in dom_ev for a, b in per)
    per_kernel = {nm: 0.0 for nm in names}
    for per in kern_ev:
        for e in per:
            for i, nm in enumerate(names):
                per_kernel[nm] += e[i].elapsed_time(e[i + 1])
    t = max_over_ranks([total, eager, dom] + [per_kernel[nm] for nm in names], pg, dev)
    launch = (("CUDA graph of the whole step, captured once and replayed"
               + ("" if args.one_stream else
                  "; the RTN comparator on a second stream beside the guided forward and the "
                  "backward")
               + (f"; sites on {nl} stream lanes" if nl > 1 else ""))
              if graph_error is None and not args.eager else
              "separate launches (programmatic stream serialization)")
    return {"total_ms": t[0], "eager_ms": t[1], "dom_ms": t[2],
            "per_kernel_ms": {nm: t[3 + i] for i, nm in enumerate(names)},
            "graph_error": graph_error, "launch": launch, "flushed": do_flush,
            "timed_passes": 2 if graph_error is None and not args.eager else 1}


def step_summary(args, wl: Workload, m, world, hbm, peak_kind):
    """The step's value, per-kernel table and roofline from measure_step."""
    K = args.steps
    n = wl.n
    ms_step = m["total_ms"] / K
    value = job_gbs(world, n, STEP_BYTES_PER_ELEM, ms_step)
    kern = {}
    for nm, ms_tot in m["per_kernel_ms"].items():
        ms = ms_tot / K
        gbs = n * BYTES_PER_ELEM[nm] / (ms * 1e-3) / 1e9
        kern[nm] = {"kernel": KERNEL_NAMES[nm], "us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
                    "elem_per_s": round(n / (ms * 1e-3), 1), "frac_of_hbm": round(gbs / hbm, 4)}
    dom = "guided_fwd"
    launches = len(wl.work)
    dom_bytes = n * BYTES_PER_ELEM[dom] / launches          # per launch (average site)
    dom_us = m["dom_ms"] / (K * launches) * 1e3              # average launch duration
    achieved = round(dom_bytes / (dom_us * 1e-6) / 1e9, 1)
    roofline = {"bound": "hbm", "kernel": KERNEL_NAMES[dom], "achieved": achieved,
                "us_per_launch": round(dom_us, 2), "launches_timed": K * launches,
                "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "traffic": traffic_from_profiles("k_fake_quant_guided", WORKLOAD_TAGS[wl.cfg]),
                "algorithmic_bytes": int(dom_bytes)}
    return {"value": value, "ms_per_step": ms_step,
            "elem_per_s": world * n / (ms_step * 1e-3),
            "algo_bytes_over_copy_peak": value / world / hbm,
            "kernels": kern, "roofline": roofline,
            "eager_ms_per_step": m["eager_ms"] / K}


def yardstick_leg(args, wl, pg, dev, flush):
    """The library's copy kernels on the largest tensor of the workload: the
    plain one (32-byte loads straight to registers, the kernels' own access
    pattern) and the one with its reads staged through shared memory by the
    bulk-copy engine (cp.async.bulk + mbarrier, four 16 KiB tiles in flight
    per CTA).  Both are checked to have copied every byte."""
    from fp4_quantization_aware_trace_b200 import ops
    stream = torch.cuda.current_stream()
    ny = max(w["xr"].numel() for w in wl.work)
    ysrc = torch.randn(ny, device=dev).to(torch.bfloat16)
    ydst = torch.empty_like(ysrc)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out = {}
    for name, fn in (("k_copy", lambda: ops.trace_copy_bf16(ysrc, ydst, ny, stream)),
                     ("k_copy_staged", lambda: ops.trace_copy_bf16_staged(ysrc, ydst, ny, err,
                                                                          stream))):
        yev = [_pair() for _ in range(args.steps)]
        for i in range(3):
            flush.fill_(i)
            fn()
        ydst.zero_()
        for k in range(args.steps):
            flush.fill_((k + 3) & 0xFF)
            yev[k][0].record(stream)
            fn()
            yev[k][1].record(stream)
        torch.cuda.synchronize()
        ok = bool(torch.equal(ydst, ysrc)) and int(err.item()) == 0
        y_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in yev) / args.steps], pg, dev)[0]
        out[name] = {"bytes": 4 * ny, "us": round(y_ms * 1e3, 2),
                     "gbs": round(4 * ny / (y_ms * 1e-3) / 1e9, 1), "copied_ok": ok}
    out["l2"] = "flushed before each launch"
    return out


def next_rows_leg(args, wl: Workload, pg, dev, flush, hbm):
    """The rows built beyond the step, each timed alone over the first
    `--next-sites` sites: full-information guidance, the mismatch
    histogram, the cache tier, MXFP4, W4A8 and the tiled scale layout."""
    from fp4_quantization_aware_trace_b200 import cache_tier, ops
    stream = torch.cuda.current_stream()
    work = wl.work[:max(1, args.next_sites)]
    K = args.steps
    n = sum(w["xr"].numel() for w in work)
    caps = [ops.capture(w["xr"], w["offs"], stream=stream) for w in work]  # own codes per site

    def rate(ms_total, b):
        ms = ms_total / K
        gbs = n * b / (ms * 1e-3) / 1e9
        return {"us": round(ms * 1e3, 2), "bytes_per_elem": b, "gbs": round(gbs, 1),
                "frac_of_hbm": round(gbs / hbm, 4)}

    def timed(fn, nev, seed):
        fn(None)  # untimed: first launches
        evs_all = []
        for k in range(K):
            flush.fill_((k + seed) & 0xFF)
            evs = [[_ev() for _ in range(nev)] for _ in work]
            fn(evs)
            evs_all.append(evs)
        torch.cuda.synchronize()
        ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for evs in evs_all
                  for i in range(len(work))) for j in range(nev - 1)]
        return max_over_ranks(ms, pg, dev)

    def full_pass(evs):
        for i, w in enumerate(work):
            if evs: evs[i][0].record(stream)
            ops.full_guided_fq_fwd(w["xt"], caps[i], w["out"], w["mask"], stream)
            if evs: evs[i][1].record(stream)

    rows = {"sites": len(work)}
    rows["full_guided_fwd"] = dict(kernel="k_fake_quant<kFull>",
                                   **rate(timed(full_pass, 2, 13)[0], 4.6875))

    hist = torch.zeros(3, 15, dtype=torch.int64, device=dev)

    def hist_pass(evs):
        hist.zero_()
        for i, w in enumerate(work):
            if evs: evs[i][0].record(stream)
            ops.mismatch_histogram(w["xt"], caps[i], hist, stream)
            if evs: evs[i][1].record(stream)

    hr = rate(timed(hist_pass, 2, 29)[0], 2.5625)
    counts = hist.cpu().tolist()
    tot = max(1, sum(counts[0]))
    rows["mismatch_histogram"] = dict(
        kernel="k_mismatch_hist", **hr, rules=list(ops.MISMATCH_RULES),
        disagree_frac=[round(1.0 - r[0] / tot, 6) for r in counts],
        adjacent_frac_of_disagreements=[round(r[1] / max(1, tot - r[0]), 6) for r in counts],
        counts=counts)

    # the cache tier: every site's compact cache captured into one record and
    # copied to pinned host memory on a copy stream while the compute stream
    # goes on; timed from the first capture to the end of the last copy
    tier = cache_tier.CacheTier(num_layers=1, keep=1, device=dev, ring=len(work))
    for i, w in enumerate(work):  # untimed: allocates records and host buffers
        tier.capture(("site", i), 0, w["xr"], w["offs"], caps[i].codes, stream)
    torch.cuda.synchronize()
    tier_ev = []
    for k in range(K):
        torch.cuda.synchronize()  # each step starts with an idle copy engine
        flush.fill_((k + 41) & 0xFF)
        ev = [_ev() for _ in range(3)]
        ev[0].record(stream)
        for i, w in enumerate(work):
            tier.capture(("site", i), 0, w["xr"], w["offs"], caps[i].codes, stream)
        ev[1].record(stream)
        ev[2].record(tier.copy_stream)
        tier_ev.append(ev)
    torch.cuda.synchronize()
    t_c, t_t = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in tier_ev),
                               sum(e[0].elapsed_time(e[2]) for e in tier_ev)], pg, dev)
    rec_bytes = sum(cache_tier.RecordLayout.of(*w["xr"].shape, w["site"].num_groups).nbytes
                    for w in work)
    del tier
    rows["cache_tier"] = {
        "what": "capture of every site into one compact record + one D2H copy per site to "
                "pinned host memory on a copy stream",
        "record_bytes_per_step": rec_bytes, "ring_slots": len(work),
        "bits_per_elem": round(8 * rec_bytes / n, 4),
        "compute_stream_us": round(t_c / K * 1e3, 2),
        "until_last_copy_us": round(t_t / K * 1e3, 2),
        "d2h_gbs": round(rec_bytes / (t_t / K * 1e-3) / 1e9, 2)}

    # capture and guided forward with the scales in the 128 x 4 tiled layout
    tcap = [ops.capture_tiled(w["xr"], w["offs"], stream) for w in work]

    def tiled_pass(evs):
        for i, w in enumerate(work):
            R, C = w["xr"].shape
            G = w["site"].num_groups
            if evs: evs[i][0].record(stream)
            ops.trace_capture_ex(w["xr"], R, C, G, w["offs"], tcap[i].codes, tcap[i].mbits,
                                 tcap[i].scales, tcap[i].gscale, w["ws"], w["ws"].numel(),
                                 ops.TRACE_SCALES_TILED_128x4, stream)
            if evs: evs[i][1].record(stream)
            ops.fq_fwd_tiled(ops.TRACE_RULE_GUIDED, w["xt"], tcap[i], w["out"], w["mask"], stream)
            if evs: evs[i][2].record(stream)

    tl = timed(tiled_pass, 3, 67)
    rows["tiled_scales"] = {
        "capture": dict(kernel="k_capture_coop<true>", **rate(tl[0], 4.6875)),
        "guided_fwd": dict(kernel="k_fake_quant<1, true>", **rate(tl[1], 4.3125))}
    del tcap

    # W4A8 (E4M3 activations, MX scales)
    m8c = [ops.mx8_capture(w["xr"], stream=stream) for w in work]

    def mx8_pass(evs):
        for i, w in enumerate(work):
            if evs: evs[i][0].record(stream)
            ops.mx8_capture(w["xr"], m8c[i], stream)
            if evs: evs[i][1].record(stream)
            ops.mx8_guided_fq_fwd(w["xt"], m8c[i], w["out"], w["mask"], stream)
            if evs: evs[i][2].record(stream)
            ops.mx8_rtn_fq_fwd(w["xt"], m8c[i].scales, w["out_r"], w["mask_r"], stream)
            if evs: evs[i][3].record(stream)
            ops.mx8_full_guided_fq_fwd(w["xt"], m8c[i], w["out"], w["mask"], stream)
            if evs: evs[i][4].record(stream)

    m8 = timed(mx8_pass, 5, 97)
    rows["w4a8"] = {nm: dict(kernel=kn, **rate(m8[j], b)) for j, (nm, kn, b) in enumerate(
        [("capture", "k_mx8_capture", 3.15625), ("guided_fwd", "k_mx8_fake_quant<1>", 4.28125),
         ("rtn_fwd", "k_mx8_fake_quant<0>", 4.15625),
         ("full_guided_fwd", "k_mx8_fake_quant<2>", 5.15625)])}
    del m8c

    # MXFP4 (W4A4, E8M0 scales, 32-element blocks)
    mxc = [ops.mx_capture(w["xr"], stream=stream) for w in work]
    mx_hist = torch.zeros(3, 15, dtype=torch.int64, device=dev)

    def mx_pass(evs):
        for i, w in enumerate(work):
            if evs: evs[i][0].record(stream)
            ops.mx_capture(w["xr"], mxc[i], stream)
            if evs: evs[i][1].record(stream)
            ops.mx_guided_fq_fwd(w["xt"], mxc[i], w["out"], w["mask"], stream)
            if evs: evs[i][2].record(stream)
            ops.mx_rtn_fq_fwd(w["xt"], mxc[i].scales, w["out_r"], w["mask_r"], stream)
            if evs: evs[i][3].record(stream)
            ops.mx_full_guided_fq_fwd(w["xt"], mxc[i], w["out"], w["mask"], stream)
            if evs: evs[i][4].record(stream)
            ops.mx_mismatch_histogram(w["xt"], mxc[i], mx_hist, stream)
            if evs: evs[i][5].record(stream)

    mx = timed(mx_pass, 6, 53)
    rows["mxfp4"] = {nm: dict(kernel=kn, **rate(mx[j], b)) for j, (nm, kn, b) in enumerate(
        [("capture", "k_mx_capture", 2.65625), ("guided_fwd", "k_mx_fake_quant<1>", 4.28125),
         ("rtn_fwd", "k_mx_fake_quant<0>", 4.15625),
         ("full_guided_fwd", "k_mx_fake_quant<2>", 4.65625),
         ("mismatch_histogram", "k_mismatch_hist<true>", 2.53125)])}
    del mxc, caps
    torch.cuda.synchronize()
    return rows


def e2e_leg(args, wl: Workload, pg, dev, world):
    """The step end to end through the public host-to-host API
    (host_step.HostStep): every site's x_roll, x_train and grad go up from
    pinned host memory and every output comes back to it, the copies
    overlapped with the kernels in row chunks.  A pinned input set is filled
    from the site's resident tensors before its timed segment (untimed); each
    e2e step covers every site, and the segments' device times add up."""
    from fp4_quantization_aware_trace_b200 import host_step
    stream = torch.cuda.current_stream()
    hs = {}
    for w in wl.work:
        R, C = w["xr"].shape
        key = (R, C, None if w["offs"] is None else tuple(w["offs"].cpu().tolist()))
        if key not in hs:
            offs_h = None if w["offs"] is None else w["offs"].cpu()
            h = host_step.HostStep(R, C, offs_h, chunks=args.e2e_chunks, device=dev)
            hs[key] = (h, [torch.empty((R, C), dtype=torch.bfloat16, pin_memory=True)
                           for _ in range(3)], h.alloc_host())
        w["e2e_key"] = key

    def segment(w, ev):
        h, ins, outs = hs[w["e2e_key"]]
        for dst, src in zip(ins, (w["xr"], w["xt"], w["g"])):
            dst.copy_(src)  # untimed: fill the pinned inputs (synchronous)
        if ev: ev[0].record(stream)
        h.run(ins[0], ins[1], ins[2], outs, stream)
        if ev: ev[1].record(stream)
        return h, ins, outs

    segment(wl.work[0], None)  # untimed: first launches, host buffers touched
    torch.cuda.synchronize()
    steps = max(1, args.e2e_steps)
    evs = []
    if pg: pg.barrier()
    h2d = d2h = 0
    for _ in range(steps):
        for w in wl.work:
            ev = _pair()
            h, ins, outs = segment(w, ev)
            evs.append(ev)
            if _ == 0:
                h2d += sum(t.numel() * t.element_size() for t in ins)
                d2h += sum(t.numel() * t.element_size() for t in outs.values())
    torch.cuda.synchronize()
    if pg: pg.barrier()
    ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in evs)], pg, dev)[0] / steps
    chunks = {len(h.cuts) for h, _, _ in hs.values()}
    return {"value": round(job_gbs(world, wl.n, STEP_BYTES_PER_ELEM, ms), 3), "unit": "GB/s",
            "ms_per_step": round(ms, 3), "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": f"host_step.HostStep.run per site, {sorted(chunks)} row chunks",
            "elem_per_s": round(world * wl.n / (ms * 1e-3), 1),
            "timing": "events around each site's host-to-host step, summed over the sites; "
                      "the pinned inputs are filled before each segment, outside it"}


def run_trace(args):
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one process per GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
        pg = dist

    from fp4_quantization_aware_trace_b200 import ops
    ops.library()
    hbm, peak_kind = measured_peaks()
    flush = L2Flush(dev)
    clk = ClockSampler(local)

    wl = Workload(args.config, rank, dev, args.lanes, args.sites)
    m = measure_step(args, wl, pg, dev, clk, flush)
    head = step_summary(args, wl, m, world, hbm, peak_kind)
    yard = yardstick_leg(args, wl, pg, dev, flush)
    next_rows = next_rows_leg(args, wl, pg, dev, flush, hbm)
    e2e = None if args.no_e2e else e2e_leg(args, wl, pg, dev, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_leg(args.config, [w["site"] for w in wl.work])
    n_sites = len(wl.work)
    name = WORKLOAD_NAMES[args.config]
    if args.sites and n_sites < len(workload_shapes(args.config)):
        name = f"the first {n_sites} site(s) of: {name}"
    config = {"workload": name, "sites": n_sites, "shapes": wl.shapes
              if n_sites <= 8 else [wl.shapes[0], f"x{n_sites}"], "groups": sorted(set(wl.groups)),
              "step": "capture + guided fwd + STE bwd + RTN fwd",
              "resident_input_bytes": wl.resident_bytes,
              "l2": ("inputs far larger than L2 (each read from HBM once per step): no flush"
                     if not m["flushed"] else "flushed before every step (256 MiB write, then a 256 MiB read that writes the dirty lines back outside the timed region)"),
              "launch": m["launch"],
              "parallelism": f"{world} GPU(s), each its own draw of the workload (no collective)"}
    gpu_launches = LAUNCHES_PER_SITE * n_sites * args.steps * m["timed_passes"]
    del wl
    torch.cuda.empty_cache()

    secondary = None
    if not args.no_secondary and args.config == HEADLINE_CONFIG:
        secondary = {}
        for cfg2 in SECONDARY_CONFIGS:
            wl2 = Workload(cfg2, rank, dev, args.lanes)
            m2 = measure_step(args, wl2, pg, dev, clk, flush)
            s2 = step_summary(args, wl2, m2, world, hbm, peak_kind)
            secondary[WORKLOAD_TAGS[cfg2]] = {
                "workload": WORKLOAD_NAMES[cfg2], "shapes": wl2.shapes,
                "value": round(s2["value"], 3), "unit": "GB/s",
                "ms_per_step": round(s2["ms_per_step"], 5),
                "eager_ms_per_step": round(s2["eager_ms_per_step"], 5),
                "elem_per_s": round(s2["elem_per_s"], 1),
                "algo_bytes_over_copy_peak": round(s2["algo_bytes_over_copy_peak"], 4),
                "kernels": s2["kernels"], "roofline": s2["roofline"],
                "yardstick": yardstick_leg(args, wl2, pg, dev, flush),
                "l2": "flushed before every step (256 MiB write, then a 256 MiB read that writes the dirty lines back outside the timed region)", "launch": m2["launch"]}
            gpu_launches += LAUNCHES_PER_SITE * len(wl2.work) * args.steps * m2["timed_passes"]
            del wl2
            torch.cuda.empty_cache()

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(head["value"], 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(head["ms_per_step"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "elem_per_s": round(head["elem_per_s"], 1),
        "algo_bytes_over_copy_peak": round(head["algo_bytes_over_copy_peak"], 4),
        "config": config,
        "kernels": head["kernels"],
        "roofline": head["roofline"],
        "yardstick": yard,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": gpu_launches,
        "eager_ms_per_step": round(head["eager_ms_per_step"], 5),
        "graph_error": m["graph_error"],
        "secondary": secondary,
        "next_rows": next_rows,
        "timing": ("value: events around each step (graph replay) only; roofline: events around "
                   "every guided-forward launch in a second timed pass of eager steps, averaged "
                   "over the launches; kernels: a third, untimed pass with events between the "
                   "calls"),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_plumbing(args):
    """The multi-rank plumbing alone, on CPU: every rank joins a gloo process
    group (127.0.0.1), the per-rank values reduce to their max, and rank 0
    prints what it saw."""
    import datetime
    import torch.distributed as dist
    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
    try:
        got = max_over_ranks([1.0 + rank, 10.0 - rank], dist if world > 1 else None, "cpu")
        ranks = [torch.zeros(1) for _ in range(world)]
        if world > 1:
            dist.all_gather(ranks, torch.tensor([float(rank)]))
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"plumbing": True, "n_gpus": world, "ranks": [int(r) for r in ranks],
                          "max_over_ranks": got,
                          "master_addr": os.environ.get("MASTER_ADDR", "")}), flush=True)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        if args.impl == "reference" and not args.plumbing_only:
            run_reference(args)  # one process: rank 0 alone runs the oracle
            return 0
        r = subprocess.run(rank_launch_cmd(argv, args.gpus, _free_port()))
        return r.returncode
    if args.plumbing_only:
        run_plumbing(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_trace(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())

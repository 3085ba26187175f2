"""The JSON line bench.py prints: the keys and invariants of the contract,
for the reference arm (the oracle on the host: runs anywhere) and for the
library on a GPU."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"}


def _run(*args, timeout=900):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def _metric():
    sys.path.insert(0, ROOT)
    import bench
    return bench.METRIC


def test_reference_arm_line():
    # the attention-input workload: drawn on the CPU here in seconds (the
    # layer sweep is drawn on the GPU where there is one)
    d = _run("--impl", "reference", "--config", "2", "--steps", "1", "--warmup", "0")
    assert BASE_KEYS <= set(d) and d["impl"] == "reference"
    assert d["metric"] == _metric() and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["n_gpus"] == 1 and d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_gpus_n_starts_n_ranks():
    """--gpus 2 without torchrun starts two ranks itself (torch.distributed.run
    on 127.0.0.1); with --plumbing-only they join a gloo group on the CPU and
    rank 0 prints one line that counts both."""
    d = _run("--gpus", "2", "--plumbing-only", timeout=300)
    assert d["plumbing"] is True and d["n_gpus"] == 2 and d["ranks"] == [0, 1]
    assert d["max_over_ranks"] == [2.0, 10.0] and d["master_addr"] == "127.0.0.1"


def test_rank_launch_command():
    sys.path.insert(0, ROOT)
    import bench
    cmd = bench.rank_launch_cmd(["--gpus", "4", "--steps", "3"], 4, 29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr" in cmd and "127.0.0.1" in cmd
    assert cmd[-3:] == ["4", "--steps", "3"] and cmd[-5].endswith("bench.py")


@pytest.mark.gpu
def test_headline_line_is_the_whole_layer_sweep():
    """The default line: all 80 sites of the later-half layer sweep resident,
    with the roofline of the dominant kernel and the end-to-end number."""
    d = _run("--steps", "2", "--warmup", "3", "--e2e-steps", "1", "--no-cpu-baseline",
             "--no-secondary", "--next-sites", "1", timeout=1500)
    assert d["config"]["sites"] == 80 and "80 sites" in d["config"]["workload"]
    n = 80 * 65536 * 4096
    assert abs(d["value"] - n * 17.3125 / (d["ms_per_step"] * 1e-3) / 1e9) < 0.01 * d["value"]
    r = d["roofline"]
    assert r["launches_timed"] == 160 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] == 80 * 3 * 65536 * 4096 * 2


@pytest.mark.gpu
def test_trace_arm_line():
    d = _run("--config", "2", "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    assert BASE_KEYS <= set(d) and "impl" not in d
    assert d["metric"] == _metric() and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 3 and d["warmup"] >= 3 and d["scaling"] == "weak"
    assert d["config"]["workload"] and d["data"] == "synthetic"
    r = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["frac"] < 1.5
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] > 0
    c = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(c)
    # the value is the whole step's algorithmic bytes over the step time
    n = 16384 * 2048
    assert abs(d["value"] - n * 17.3125 / (d["ms_per_step"] * 1e-3) / 1e9) < 0.01 * d["value"]

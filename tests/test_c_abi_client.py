"""The C ABI from plain C: tests/c_abi_client.c (no Python, no torch) is
compiled with gcc against include/trace_fp4.h and libtrace_fp4.so; on a GPU
it runs the path and its outputs are compared bit for bit with the oracle on
the inputs it wrote."""
from __future__ import annotations

import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fp4_quantization_aware_trace_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path) -> str:
    if not os.path.exists(os.path.join(PKG, "libtrace_fp4.so")):
        pytest.skip("libtrace_fp4.so is not built")
    exe = str(tmp_path / "c_abi_client")
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi_client.c"),
           "-L", PKG, "-ltrace_fp4", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{PKG}:{os.path.join(CUDA, 'lib64')}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_client_compiles_and_links(tmp_path):
    """The header is valid C11 and the library links from C (no GPU needed)."""
    assert os.path.exists(_build(tmp_path))


@pytest.mark.gpu
def test_c_client_matches_oracle(tmp_path, oracle_mod):
    exe = _build(tmp_path)
    out_file = tmp_path / "client.bin"
    r = subprocess.run([exe, str(out_file)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    buf = out_file.read_bytes()
    pos = 0

    def take(dtype, count):
        nonlocal pos
        a = np.frombuffer(buf, dtype=dtype, count=count, offset=pos)
        pos += a.nbytes
        return a

    rows, cols = (int(v) for v in take(np.int64, 2))
    G = int(take(np.int32, 1)[0])
    offs = take(np.int64, G + 1).copy()
    n = rows * cols
    xr = take(np.uint16, n).reshape(rows, cols)
    xt = take(np.uint16, n).reshape(rows, cols)
    g = take(np.uint16, n).reshape(rows, cols)
    got = dict(codes=take(np.uint8, n // 2), mbits=take(np.uint32, n // 32),
               scales=take(np.uint8, n // 16), gscale=take(np.float32, G),
               out=take(np.uint16, n), mask=take(np.uint32, n // 32), grad_in=take(np.uint16, n),
               out_rtn=take(np.uint16, n), mask_rtn=take(np.uint32, n // 32))
    assert pos == len(buf)
    codes, mbits, scales, gscale = oracle_mod.capture(xr, G, offs)
    out, mask = oracle_mod.guided_fwd(xt, mbits, scales, gscale, G, offs)
    out_r, mask_r = oracle_mod.rtn_fwd(xt, scales, gscale, G, offs)
    gin = oracle_mod.fq_bwd(g, mask)
    ref = dict(codes=codes, mbits=mbits, scales=scales, gscale=gscale, out=out, mask=mask,
               grad_in=gin, out_rtn=out_r, mask_rtn=mask_r)
    for k, v in ref.items():
        a, b = np.asarray(got[k]).reshape(-1), np.asarray(v).reshape(-1)
        if a.dtype == np.float32:
            a, b = a.view(np.uint32), b.view(np.uint32)
        assert np.array_equal(a, b), k

"""Static checks of the CUDA sources (no GPU).

Out-of-line (__noinline__) device functions must not use the 32-byte vector
load / store forms (`ld_block_stream`, `st_block`, any `.v8` asm): with
them, ptxas 12.9 crashed (load) or, depending on the rest of the module,
emitted a store of wrong data (found by the seeded fuzz parity cases).  Those
functions use the 16-byte `ld_block_ro` / `st_block_plain` instead."""
from __future__ import annotations

import glob
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "fp4_quantization_aware_trace_b200", "csrc")


def _noinline_bodies(text: str):
    for m in re.finditer(r"__noinline__[^{;]*\{", text):
        depth, i = 1, m.end()
        while depth and i < len(text):
            depth += {"{": 1, "}": -1}.get(text[i], 0)
            i += 1
        yield text[m.start():i]


def test_no_wide_vector_access_in_out_of_line_functions():
    files = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.cu"))
    bodies = [b for f in files for b in _noinline_bodies(open(f).read())]
    assert len(bodies) >= 3  # the three exact-path functions
    for b in bodies:
        name = b.split("(")[0].split()[-1]
        for bad in ("ld_block_stream(", "st_block(", ".v8."):
            assert bad not in b, f"{name} uses {bad}"

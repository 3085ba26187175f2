"""CPU oracle for TRACE rollout-guided NVFP4 rounding -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``fp4_quantization_aware_trace_b200``) never imports it, and it
never imports the product path.

The arithmetic lives in ``trace_oracle.c`` (plain C, one IEEE binary32
operation per step, built with ``-ffp-contract=off``); this module only
builds it with gcc and marshals numpy arrays through ctypes.

Method: the rcap.io post "TRACE: Rollout-Guided Quantization-Aware Training
for FP4" -- sections "rollout-guided rounding" and "compact cache" and the
pseudocode listing (rollout capture; QAT forward).  Every function is pinned
by tests against brute force, library routines and closed forms; see the
header of ``trace_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "trace_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
             "-fno-finite-math-only", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = f32
        lib.oracle_f32_to_bf16.argtypes = [f32]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f32.restype = f32
        lib.oracle_f32_to_e4m3.argtypes = [f32]
        lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        lib.oracle_e2m1_rtn.argtypes = [f32]
        lib.oracle_e2m1_rtn.restype = ctypes.c_int
        lib.oracle_e2m1_bracket.argtypes = [f32, ctypes.POINTER(ctypes.c_int),
                                            ctypes.POINTER(ctypes.c_int)]
        lib.oracle_e2m1_bracket.restype = None
        lib.oracle_guided_code.argtypes = [f32, ctypes.c_int]
        lib.oracle_guided_code.restype = ctypes.c_int
        lib.oracle_dequant_bf16.argtypes = [ctypes.c_int, ctypes.c_int, f32, f32]
        lib.oracle_dequant_bf16.restype = ctypes.c_uint16
        lib.oracle_global_scale.argtypes = [f32]
        lib.oracle_global_scale.restype = f32
        lib.oracle_block_scale.argtypes = [f32, f32]
        lib.oracle_block_scale.restype = ctypes.c_uint8
        lib.oracle_capture.argtypes = [P, i64, i64, i32, P, P, P, P, P]
        lib.oracle_capture.restype = None
        lib.oracle_guided_fwd.argtypes = [P, i64, i64, i32, P, P, P, P, P, P]
        lib.oracle_guided_fwd.restype = None
        lib.oracle_rtn_fwd.argtypes = [P, i64, i64, i32, P, P, P, P, P]
        lib.oracle_rtn_fwd.restype = None
        lib.oracle_fq_bwd.argtypes = [P, P, i64, P]
        lib.oracle_fq_bwd.restype = None
        lib.oracle_group_amax.argtypes = [P, i64, i64, i32, P, P]
        lib.oracle_group_amax.restype = None
        lib.oracle_capture_rows.argtypes = [P, i64, i64, P, P, P, P]
        lib.oracle_capture_rows.restype = None
        lib.oracle_fake_quant_rows.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.oracle_fake_quant_rows.restype = None
        lib.oracle_fake_quant_codes.argtypes = [P, i64, i64, i32, P, P, P, P, P]
        lib.oracle_fake_quant_codes.restype = None
        lib.oracle_full_guided_code.argtypes = [f32, ctypes.c_int]
        lib.oracle_full_guided_code.restype = ctypes.c_int
        lib.oracle_full_guided_fwd.argtypes = [P, i64, i64, i32, P, P, P, P, P, P]
        lib.oracle_full_guided_fwd.restype = None
        lib.oracle_full_guided_codes.argtypes = [P, i64, i64, i32, P, P, P, P, P]
        lib.oracle_full_guided_codes.restype = None
        lib.oracle_full_guided_rows.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.oracle_full_guided_rows.restype = None
        lib.oracle_mismatch_histogram.argtypes = [P, i64, i64, i32, P, P, P, P, P]
        lib.oracle_mismatch_histogram.restype = None
        lib.oracle_e8m0_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e8m0_to_f32.restype = ctypes.c_float
        lib.oracle_mx_scale.argtypes = [ctypes.c_float]
        lib.oracle_mx_scale.restype = ctypes.c_uint8
        lib.oracle_mx_capture.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_mx_capture.restype = None
        lib.oracle_mx_guided_fwd.argtypes = [P, i64, i64, P, P, P, P]
        lib.oracle_mx_guided_fwd.restype = None
        lib.oracle_mx_rtn_fwd.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_mx_rtn_fwd.restype = None
        lib.oracle_mx_full_guided_fwd.argtypes = [P, i64, i64, P, P, P, P]
        lib.oracle_mx_full_guided_fwd.restype = None
        lib.oracle_mx_fake_quant_codes.argtypes = [P, i64, i64, P, P, P, P, ctypes.c_int]
        lib.oracle_mx_fake_quant_codes.restype = None
        lib.oracle_mx8_scale.argtypes = [ctypes.c_float]
        lib.oracle_mx8_scale.restype = ctypes.c_uint8
        lib.oracle_e4m3_bracket.argtypes = [ctypes.c_float, P, P]
        lib.oracle_e4m3_bracket.restype = None
        lib.oracle_e4m3_guided_code.argtypes = [ctypes.c_float, ctypes.c_int]
        lib.oracle_e4m3_guided_code.restype = ctypes.c_int
        lib.oracle_e4m3_full_guided_code.argtypes = [ctypes.c_float, ctypes.c_int]
        lib.oracle_e4m3_full_guided_code.restype = ctypes.c_int
        lib.oracle_mx8_capture.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_mx8_capture.restype = None
        lib.oracle_mx8_guided_fwd.argtypes = [P, i64, i64, P, P, P, P]
        lib.oracle_mx8_guided_fwd.restype = None
        lib.oracle_mx8_rtn_fwd.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_mx8_rtn_fwd.restype = None
        lib.oracle_mx8_full_guided_fwd.argtypes = [P, i64, i64, P, P, P, P]
        lib.oracle_mx8_full_guided_fwd.restype = None
        lib.oracle_mx8_fake_quant_codes.argtypes = [P, i64, i64, P, P, P, P, ctypes.c_int]
        lib.oracle_mx8_fake_quant_codes.restype = None
        lib.oracle_mx_mismatch_histogram.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_mx_mismatch_histogram.restype = None
        lib.oracle_e4m3_sweep.argtypes = [ctypes.c_uint32, ctypes.c_uint32, P]
        lib.oracle_e4m3_sweep.restype = None
        lib.oracle_swizzled_scale_bytes.argtypes = [i64, i64]
        lib.oracle_swizzled_scale_bytes.restype = i64
        lib.oracle_swizzle_scales.argtypes = [P, i64, i64, P]
        lib.oracle_swizzle_scales.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_bf16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16 and x.ndim == 2, "bf16 bits as uint16 [rows, cols]"
    return x


def _offsets(offsets, G: int, rows: int):
    if offsets is None:
        assert G == 1
        return None
    o = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    assert o.shape == (G + 1,) and o[0] == 0 and o[-1] == rows
    return o


# -- scalar helpers (used by the pin tests) ---------------------------------

def bf16_to_f32(h: int) -> float:
    return _load().oracle_bf16_to_f32(h)


def f32_to_bf16(f: float) -> int:
    return _load().oracle_f32_to_bf16(f)


def e4m3_to_f32(b: int) -> float:
    return _load().oracle_e4m3_to_f32(b)


def f32_to_e4m3(t: float) -> int:
    return _load().oracle_f32_to_e4m3(t)


def e2m1_rtn(a: float) -> int:
    return _load().oracle_e2m1_rtn(a)


def e2m1_bracket(a: float) -> tuple[int, int]:
    lo, hi = ctypes.c_int(), ctypes.c_int()
    _load().oracle_e2m1_bracket(a, ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value


def guided_code(a: float, bit: int) -> int:
    return _load().oracle_guided_code(a, bit)


def dequant_bf16(code: int, negative: bool, sbv: float, s_g: float) -> int:
    return _load().oracle_dequant_bf16(code, int(negative), sbv, s_g)


def global_scale(amax: float) -> float:
    return _load().oracle_global_scale(amax)


def block_scale(bmax: float, s_g: float) -> int:
    return _load().oracle_block_scale(bmax, s_g)


# -- the four operations ----------------------------------------------------

def capture(x, num_groups: int = 1, offsets=None):
    """Rollout capture.  Returns (codes u8[N/2], mbits u32[N/32],
    scales u8[rows, cols/16], gscale f32[G])."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    n = rows * cols
    codes = np.zeros(n // 2, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros((rows, cols // 16), np.uint8)
    gscale = np.zeros(num_groups, np.float32)
    _load().oracle_capture(_ptr(x), rows, cols, num_groups, _ptr(o), _ptr(codes),
                           _ptr(mbits), _ptr(scales), _ptr(gscale))
    return codes, mbits, scales, gscale


def guided_fwd(x_train, mbits, scales, gscale, num_groups: int = 1, offsets=None):
    """Guided QAT forward.  Returns (out bf16 bits u16[rows, cols], mask u32[N/32])."""
    x = _as_bf16_bits(x_train)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    mbits = np.ascontiguousarray(mbits, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    gscale = np.ascontiguousarray(gscale, dtype=np.float32)
    assert mbits.size == rows * cols // 32 and scales.size == rows * cols // 16
    assert gscale.size == num_groups
    out = np.zeros((rows, cols), np.uint16)
    mask = np.zeros(rows * cols // 32, np.uint32)
    _load().oracle_guided_fwd(_ptr(x), rows, cols, num_groups, _ptr(o), _ptr(mbits),
                              _ptr(scales), _ptr(gscale), _ptr(out), _ptr(mask))
    return out, mask


def rtn_fwd(x, scales, gscale, num_groups: int = 1, offsets=None):
    """Round-to-nearest fake-quant with given scales.  Returns (out, mask)."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    gscale = np.ascontiguousarray(gscale, dtype=np.float32)
    assert scales.size == rows * cols // 16 and gscale.size == num_groups
    out = np.zeros((rows, cols), np.uint16)
    mask = np.zeros(rows * cols // 32, np.uint32)
    _load().oracle_rtn_fwd(_ptr(x), rows, cols, num_groups, _ptr(o), _ptr(scales),
                           _ptr(gscale), _ptr(out), _ptr(mask))
    return out, mask


def fq_bwd(grad_out, mask):
    """Masked straight-through backward.  Returns grad_in bits (same shape)."""
    g = np.ascontiguousarray(grad_out, dtype=np.uint16)
    mask = np.ascontiguousarray(mask, dtype=np.uint32)
    assert g.size % 32 == 0 and mask.size == g.size // 32
    out = np.zeros_like(g)
    _load().oracle_fq_bwd(_ptr(g), _ptr(mask), g.size, _ptr(out))
    return out


# -- row-level entry points (sampled checks on tensors too big for the
#    whole-tensor oracle) -----------------------------------------------------

def group_amax(x, num_groups: int = 1, offsets=None) -> np.ndarray:
    """max |x| over the rows of each group (f32[G])."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    amax = np.zeros(num_groups, np.float32)
    _load().oracle_group_amax(_ptr(x), rows, cols, num_groups, _ptr(o), _ptr(amax))
    return amax


def capture_rows(x, row_gscale):
    """Capture steps 3-6 for rows whose global scale is given per row.
    Returns (codes, mbits, scales)."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    rg = np.ascontiguousarray(row_gscale, dtype=np.float32)
    assert rg.shape == (rows,)
    n = rows * cols
    codes = np.zeros(n // 2, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros((rows, cols // 16), np.uint8)
    _load().oracle_capture_rows(_ptr(x), rows, cols, _ptr(rg), _ptr(codes),
                                _ptr(mbits), _ptr(scales))
    return codes, mbits, scales


def fake_quant_rows(x, row_gscale, scales, mbits=None):
    """Guided (mbits given) or round-to-nearest (mbits None) fake-quant for
    rows whose global scale is given per row.  Returns (out, mask)."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    rg = np.ascontiguousarray(row_gscale, dtype=np.float32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    assert rg.shape == (rows,) and scales.size == rows * cols // 16
    if mbits is not None:
        mbits = np.ascontiguousarray(mbits, dtype=np.uint32)
        assert mbits.size == rows * cols // 32
    out = np.zeros((rows, cols), np.uint16)
    mask = np.zeros(rows * cols // 32, np.uint32)
    _load().oracle_fake_quant_rows(_ptr(x), rows, cols, _ptr(rg), _ptr(mbits),
                                   _ptr(scales), _ptr(out), _ptr(mask))
    return out, mask


def fake_quant_codes(x, scales, gscale, mbits=None, num_groups: int = 1, offsets=None):
    """Signed code (sign<<3 | magnitude) picked at every site by the guided
    forward (mbits given) or by round-to-nearest (mbits None): u8[rows, cols]."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    gscale = np.ascontiguousarray(gscale, dtype=np.float32)
    if mbits is not None:
        mbits = np.ascontiguousarray(mbits, dtype=np.uint32)
    sites = np.zeros((rows, cols), np.uint8)
    _load().oracle_fake_quant_codes(_ptr(x), rows, cols, num_groups, _ptr(o), _ptr(mbits),
                                    _ptr(scales), _ptr(gscale), _ptr(sites))
    return sites


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """Packed nibbles -> one signed code per element (layout helper)."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.size * 2, np.uint8)
    out[0::2] = c & 0xF
    out[1::2] = c >> 4
    return out


def unpack_bits(words: np.ndarray) -> np.ndarray:
    """Packed u32 bit words -> one 0/1 byte per element (layout helper)."""
    w = np.asarray(words, dtype=np.uint32).view(np.uint8)
    return np.unpackbits(w, bitorder="little")


# -- full-information guidance (the cache keeps the whole rollout code) ------

def full_guided_code(z: float, roll_code: int) -> int:
    """Magnitude code of q* for unclipped z and a signed rollout code."""
    return _load().oracle_full_guided_code(z, roll_code)


def full_guided_fwd(x_train, rcodes, scales, gscale, num_groups: int = 1, offsets=None):
    """Full-information guided forward.  Returns (out, mask)."""
    x = _as_bf16_bits(x_train)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    rcodes = np.ascontiguousarray(rcodes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    gscale = np.ascontiguousarray(gscale, dtype=np.float32)
    assert rcodes.size == rows * cols // 2 and scales.size == rows * cols // 16
    out = np.zeros((rows, cols), np.uint16)
    mask = np.zeros(rows * cols // 32, np.uint32)
    _load().oracle_full_guided_fwd(_ptr(x), rows, cols, num_groups, _ptr(o), _ptr(rcodes),
                                   _ptr(scales), _ptr(gscale), _ptr(out), _ptr(mask))
    return out, mask


def full_guided_codes(x, rcodes, scales, gscale, num_groups: int = 1, offsets=None):
    """Signed code picked at every site by full-information guidance."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    sites = np.zeros((rows, cols), np.uint8)
    _load().oracle_full_guided_codes(_ptr(x), rows, cols, num_groups, _ptr(o),
                                     _ptr(np.ascontiguousarray(rcodes, dtype=np.uint8)),
                                     _ptr(np.ascontiguousarray(scales, dtype=np.uint8)),
                                     _ptr(np.ascontiguousarray(gscale, dtype=np.float32)),
                                     _ptr(sites))
    return sites


def full_guided_rows(x, row_gscale, scales, rcodes):
    """Full-information guided forward for rows with known global scales."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    rg = np.ascontiguousarray(row_gscale, dtype=np.float32)
    out = np.zeros((rows, cols), np.uint16)
    mask = np.zeros(rows * cols // 32, np.uint32)
    _load().oracle_full_guided_rows(_ptr(x), rows, cols, _ptr(rg),
                                    _ptr(np.ascontiguousarray(rcodes, dtype=np.uint8)),
                                    _ptr(np.ascontiguousarray(scales, dtype=np.uint8)),
                                    _ptr(out), _ptr(mask))
    return out, mask


# -- mismatch diagnostic ------------------------------------------------------

def mismatch_histogram(x_train, rcodes, scales, gscale, num_groups: int = 1, offsets=None):
    """uint64[3, 15]: ladder distance from the rollout code of the training
    side's RTN (row 0), 1-bit guided (row 1) and full-information guided
    (row 2) codes."""
    x = _as_bf16_bits(x_train)
    rows, cols = x.shape
    o = _offsets(offsets, num_groups, rows)
    hist = np.zeros(45, np.uint64)
    _load().oracle_mismatch_histogram(_ptr(x), rows, cols, num_groups, _ptr(o),
                                      _ptr(np.ascontiguousarray(rcodes, dtype=np.uint8)),
                                      _ptr(np.ascontiguousarray(scales, dtype=np.uint8)),
                                      _ptr(np.ascontiguousarray(gscale, dtype=np.float32)),
                                      _ptr(hist))
    return hist.reshape(3, 15)


# -- MXFP4 variant ------------------------------------------------------------

def e8m0_to_f32(b: int) -> float:
    return float(_load().oracle_e8m0_to_f32(int(b)))


def mx_scale(amax: float) -> int:
    return int(_load().oracle_mx_scale(float(amax)))


def mx_capture(x_roll):
    """(codes uint8[N/2], mbits uint32[N/32], scales uint8[rows, cols/32])."""
    x = _as_bf16_bits(x_roll)
    rows, cols = x.shape
    n = rows * cols
    codes = np.zeros(n // 2, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros((rows, cols // 32), np.uint8)
    _load().oracle_mx_capture(_ptr(x), rows, cols, _ptr(codes), _ptr(mbits), _ptr(scales))
    return codes, mbits, scales


def _mx_fwd(fn, x, extra, scales):
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    out = np.zeros((rows, cols), np.uint16)
    mask = np.zeros(rows * cols // 32, np.uint32)
    args = [_ptr(x), rows, cols]
    if extra is not None:
        args.append(_ptr(extra))
    args += [_ptr(np.ascontiguousarray(scales, dtype=np.uint8)), _ptr(out), _ptr(mask)]
    fn(*args)
    return out, mask


def mx_guided_fwd(x_train, mbits, scales):
    return _mx_fwd(_load().oracle_mx_guided_fwd, x_train,
                   np.ascontiguousarray(mbits, dtype=np.uint32), scales)


def mx_rtn_fwd(x, scales):
    return _mx_fwd(_load().oracle_mx_rtn_fwd, x, None, scales)


def mx_full_guided_fwd(x_train, rcodes, scales):
    return _mx_fwd(_load().oracle_mx_full_guided_fwd, x_train,
                   np.ascontiguousarray(rcodes, dtype=np.uint8), scales)


def mx_fake_quant_codes(x, scales, mbits=None, rcodes=None):
    """Signed code per element: RTN (both None), 1-bit guided (mbits) or
    full-information guided (rcodes)."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    sites = np.zeros(rows * cols, np.uint8)
    mode = 1 if mbits is not None else (2 if rcodes is not None else 0)
    mb = None if mbits is None else np.ascontiguousarray(mbits, dtype=np.uint32)
    rc = None if rcodes is None else np.ascontiguousarray(rcodes, dtype=np.uint8)
    _load().oracle_mx_fake_quant_codes(_ptr(x), rows, cols, _ptr(mb), _ptr(rc),
                                       _ptr(np.ascontiguousarray(scales, dtype=np.uint8)),
                                       _ptr(sites), mode)
    return sites.reshape(rows, cols)


# -- block-scale layout of a block-scaled FP4 GEMM ------------------------------

def swizzled_scale_bytes(rows: int, scols: int) -> int:
    return int(_load().oracle_swizzled_scale_bytes(rows, scols))


def swizzle_scales(scales) -> np.ndarray:
    """Row-major scales [rows, scols] (uint8) -> the 128 x 4 tiled layout
    (uint8, padding bytes 0)."""
    lin = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, scols = lin.shape
    out = np.zeros(swizzled_scale_bytes(rows, scols), np.uint8)
    _load().oracle_swizzle_scales(_ptr(lin), rows, scols, _ptr(out))
    return out


# -- W4A8: E4M3 activations with MX scales --------------------------------------

def mx8_scale(amax: float) -> int:
    return int(_load().oracle_mx8_scale(float(amax)))


def e4m3_bracket(a: float) -> tuple[int, int]:
    lo, hi = ctypes.c_int(0), ctypes.c_int(0)
    _load().oracle_e4m3_bracket(float(a), ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value


def e4m3_guided_code(a: float, bit: int) -> int:
    return int(_load().oracle_e4m3_guided_code(float(a), int(bit)))


def e4m3_full_guided_code(z: float, roll_code: int) -> int:
    return int(_load().oracle_e4m3_full_guided_code(float(z), int(roll_code)))


def mx8_capture(x_roll):
    """(codes uint8[N], mbits uint32[N/32], scales uint8[rows, cols/32])."""
    x = _as_bf16_bits(x_roll)
    rows, cols = x.shape
    n = rows * cols
    codes = np.zeros(n, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros((rows, cols // 32), np.uint8)
    _load().oracle_mx8_capture(_ptr(x), rows, cols, _ptr(codes), _ptr(mbits), _ptr(scales))
    return codes, mbits, scales


def mx8_guided_fwd(x_train, mbits, scales):
    return _mx_fwd(_load().oracle_mx8_guided_fwd, x_train,
                   np.ascontiguousarray(mbits, dtype=np.uint32), scales)


def mx8_rtn_fwd(x, scales):
    return _mx_fwd(_load().oracle_mx8_rtn_fwd, x, None, scales)


def mx8_full_guided_fwd(x_train, rcodes, scales):
    return _mx_fwd(_load().oracle_mx8_full_guided_fwd, x_train,
                   np.ascontiguousarray(rcodes, dtype=np.uint8), scales)


def mx8_fake_quant_codes(x, scales, mbits=None, rcodes=None):
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    sites = np.zeros(rows * cols, np.uint8)
    mode = 1 if mbits is not None else (2 if rcodes is not None else 0)
    mb = None if mbits is None else np.ascontiguousarray(mbits, dtype=np.uint32)
    rc = None if rcodes is None else np.ascontiguousarray(rcodes, dtype=np.uint8)
    _load().oracle_mx8_fake_quant_codes(_ptr(x), rows, cols, _ptr(mb), _ptr(rc),
                                        _ptr(np.ascontiguousarray(scales, dtype=np.uint8)),
                                        _ptr(sites), mode)
    return sites.reshape(rows, cols)


def e4m3_sweep(first_bits: int, count: int) -> np.ndarray:
    """E4M3 codes of the fp32 values with bit patterns first_bits + i."""
    out = np.zeros(count, np.uint8)
    _load().oracle_e4m3_sweep(first_bits, count, _ptr(out))
    return out


def mx_mismatch_histogram(x_train, rcodes, scales):
    """uint64[3, 15] as mismatch_histogram, with MXFP4 (E8M0) scales."""
    x = _as_bf16_bits(x_train)
    rows, cols = x.shape
    hist = np.zeros(45, np.uint64)
    _load().oracle_mx_mismatch_histogram(_ptr(x), rows, cols,
                                         _ptr(np.ascontiguousarray(rcodes, dtype=np.uint8)),
                                         _ptr(np.ascontiguousarray(scales, dtype=np.uint8)),
                                         _ptr(hist))
    return hist.reshape(3, 15)

"""Brute-force restatement of the NVFP4 rounding decisions, for pinning the
oracle on tiny inputs.

Nothing here shares an algorithm with ``oracle/trace_oracle.c``: every
rounding decision is an exhaustive search over the candidate values in exact
rational arithmetic (``fractions.Fraction``), where the oracle uses threshold
comparisons and exponent/mantissa arithmetic.  The fp32 operations the format
prescribes (a division, a product) are taken from numpy float32 arithmetic,
which is IEEE-754 binary32 with round-to-nearest-even; fp32 -> bf16 is
torch's CPU conversion (round to nearest even).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

# The signed E2M1 grid as (value, magnitude code).  The mantissa bit of a
# codeword is the lowest bit of its magnitude code.
_MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
         Fraction(3), Fraction(4), Fraction(6)]
SIGNED_GRID = sorted({(s * m, c) for c, m in enumerate(_MAGS) for s in (1, -1)},
                     key=lambda t: t[0])
# +0 and -0 are one point of the grid.
SIGNED_GRID = [g for i, g in enumerate(SIGNED_GRID) if i == 0 or g[0] != SIGNED_GRID[i - 1][0]]


def e4m3_value(byte: int) -> Fraction:
    """Exact value of a non-negative finite E4M3 (fn) byte 0x00..0x7E."""
    assert 0 <= byte <= 0x7E
    e, m = byte >> 3, byte & 7
    if e == 0:
        return Fraction(m, 512)
    return Fraction(8 + m, 8) * (Fraction(2) ** (e - 7))


E4M3_TABLE = [(e4m3_value(b), b) for b in range(0x7F)]


def brute_e4m3(t: float) -> int:
    """Nearest E4M3 byte to t >= 0 by exhaustive search; ties to the even
    mantissa; values beyond 448 saturate to 448."""
    tq = Fraction(float(np.float32(t)))
    best = None
    for v, b in E4M3_TABLE:
        d = abs(tq - v)
        if best is None or d < best[0] or (d == best[0] and (b & 1) == 0):
            best = (d, b)
    return best[1]


def brute_rtn(z: Fraction) -> tuple[Fraction, int]:
    """Clip z to [-6,6], then nearest signed codeword by exhaustive search;
    ties go to the codeword whose mantissa bit is 0."""
    zc = max(Fraction(-6), min(Fraction(6), z))
    best = None
    for v, c in SIGNED_GRID:
        d = abs(zc - v)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, v, c)
    return best[1], best[2]


def brute_bracket(z: Fraction) -> tuple[tuple[Fraction, int], tuple[Fraction, int]]:
    """The two signed codewords around clip(z): the largest <= and the
    smallest >=, by exhaustive search."""
    zc = max(Fraction(-6), min(Fraction(6), z))
    below = max((g for g in SIGNED_GRID if g[0] <= zc), key=lambda g: g[0])
    above = min((g for g in SIGNED_GRID if g[0] >= zc), key=lambda g: g[0])
    return below, above


def brute_guided(z: Fraction, bit: int) -> tuple[Fraction, int]:
    """Of the bracket around clip(z), the member whose mantissa bit equals
    ``bit``; a collapsed bracket gives its single member."""
    lo, hi = brute_bracket(z)
    if lo[0] == hi[0]:
        return lo
    return lo if (lo[1] & 1) == bit else hi


def f32(x) -> np.float32:
    return np.float32(x)


def bf16_bits_to_float(h: int) -> float:
    return float(np.array([h << 16], dtype=np.uint32).view(np.float32)[0])


def float_to_bf16_bits(v: np.float32) -> int:
    t = torch.tensor([float(v)], dtype=torch.float32).to(torch.bfloat16)
    return int(t.view(torch.int16).item()) & 0xFFFF


def _signed_code(value: Fraction, mag_code: int, z_negative: bool) -> int:
    neg = value < 0 or (value == 0 and z_negative)
    return (8 if neg else 0) | mag_code


def brute_pipeline(x_roll: np.ndarray, x_train: np.ndarray, grad: np.ndarray):
    """Capture on x_roll, guided and RTN fake-quant on x_train, STE backward,
    for one group, by brute force.  Inputs are bf16 bit arrays [rows, cols].
    Returns a dict of the same arrays the oracle produces."""
    rows, cols = x_roll.shape
    n = rows * cols
    xr = [bf16_bits_to_float(int(h)) for h in x_roll.reshape(-1)]
    xt = [bf16_bits_to_float(int(h)) for h in x_train.reshape(-1)]
    amax = max(abs(v) for v in xr)
    s_g = f32(1.0) if amax == 0 else f32(amax) / f32(2688.0)
    den6 = f32(6.0) * s_g
    codes = np.zeros(n // 2, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros(n // 16, np.uint8)
    out_g = np.zeros(n, np.uint16)
    out_r = np.zeros(n, np.uint16)
    mask = np.zeros(n // 32, np.uint32)

    def zval(x: float, d: np.float32) -> tuple[Fraction, bool]:
        if d == 0:
            return Fraction(0), np.signbit(np.float32(x))
        z = f32(x) / d
        return Fraction(float(z)), bool(np.signbit(z))

    def deq(value: Fraction, z_negative: bool, sbv: Fraction) -> int:
        exact = abs(value) * sbv * Fraction(float(s_g))
        v = f32(float(exact))          # exact product has <= 30 bits: one rounding
        if value < 0 or (value == 0 and z_negative):
            v = -v
        return float_to_bf16_bits(v)

    for b in range(n // 16):
        blk = range(16 * b, 16 * b + 16)
        bmax = max(abs(xr[i]) for i in blk)
        t = f32(bmax) / den6
        sb = brute_e4m3(float(t))
        scales[b] = sb
        sbv = e4m3_value(sb)
        d = s_g * f32(float(sbv))
        for i in blk:
            z, neg = zval(xr[i], d)
            v, c = brute_rtn(z)
            codes[i // 2] |= _signed_code(v, c, neg) << (4 * (i & 1))
            mbits[i // 32] |= (c & 1) << (i & 31)
    for b in range(n // 16):
        sbv = e4m3_value(int(scales[b]))
        d = s_g * f32(float(sbv))
        for i in range(16 * b, 16 * b + 16):
            z, neg = zval(xt[i], d)
            if abs(z) <= 6:
                mask[i // 32] |= 1 << (i & 31)
            bit = (int(mbits[i // 32]) >> (i & 31)) & 1
            vg, _ = brute_guided(z, bit)
            vr, _ = brute_rtn(z)
            out_g[i] = deq(vg, neg, sbv)
            out_r[i] = deq(vr, neg, sbv)
    g = grad.reshape(-1)
    gin = np.array([g[i] if (mask[i // 32] >> (i & 31)) & 1 else 0 for i in range(n)],
                   dtype=np.uint16)
    return dict(codes=codes, mbits=mbits, scales=scales.reshape(rows, cols // 16),
                gscale=np.array([s_g], np.float32), out_guided=out_g.reshape(rows, cols),
                out_rtn=out_r.reshape(rows, cols), mask=mask,
                grad_in=gin.reshape(rows, cols))


def brute_full_guided(z: Fraction, roll_value: Fraction) -> tuple[Fraction, int]:
    """Of the bracket around clip(z), the member nearest to the rollout
    codeword value, by exhaustive comparison (no tie can occur)."""
    lo, hi = brute_bracket(z)
    dl, dh = abs(lo[0] - roll_value), abs(hi[0] - roll_value)
    assert lo[0] == hi[0] or dl != dh
    return hi if dh < dl else lo


# ---------------------------------------------------------------------------
# MXFP4 variant: 32-element blocks, E8M0 power-of-two scales, no global scale
# ---------------------------------------------------------------------------

def e8m0_value(byte: int) -> Fraction:
    assert 0 <= byte <= 254
    return Fraction(2) ** (byte - 127)


def brute_mx_scale(amax: Fraction) -> int:
    """The E8M0 byte whose value X puts amax / X in [4, 8) (the binade of
    E2M1's largest value), by search over all bytes; the smallest byte when
    amax is too small for any (or zero)."""
    if amax == 0:
        return 0
    hits = [b for b in range(255) if 4 <= amax / e8m0_value(b) < 8]
    assert len(hits) <= 1
    return hits[0] if hits else 0


def brute_mx_pipeline(x_roll: np.ndarray, x_train: np.ndarray):
    """MX capture on x_roll, then 1-bit guided, round-to-nearest and full
    guided fake-quant of x_train, by brute force (bf16 bit arrays)."""
    rows, cols = x_roll.shape
    n = rows * cols
    xr = [bf16_bits_to_float(int(h)) for h in x_roll.reshape(-1)]
    xt = [bf16_bits_to_float(int(h)) for h in x_train.reshape(-1)]
    codes = np.zeros(n // 2, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros(n // 32, np.uint8)
    outs = {k: np.zeros(n, np.uint16) for k in ("out_guided", "out_rtn", "out_full")}
    mask = np.zeros(n // 32, np.uint32)

    def zval(x: float, X: np.float32):
        z = f32(x) / X
        return Fraction(float(z)), bool(np.signbit(z))

    def deq(value: Fraction, neg: bool, X: Fraction) -> int:
        v = f32(float(abs(value) * X))   # exact
        if value < 0 or (value == 0 and neg):
            v = -v
        return float_to_bf16_bits(v)

    for b in range(n // 32):
        blk = range(32 * b, 32 * b + 32)
        sb = brute_mx_scale(max(Fraction(abs(xr[i])) for i in blk))
        scales[b] = sb
        Xq = e8m0_value(sb)
        X = f32(float(Xq))
        for i in blk:
            z, neg = zval(xr[i], X)
            v, c = brute_rtn(z)
            codes[i // 2] |= _signed_code(v, c, neg) << (4 * (i & 1))
            mbits[i // 32] |= (c & 1) << (i & 31)
        for i in blk:
            z, neg = zval(xt[i], X)
            if abs(z) <= 6:
                mask[i // 32] |= 1 << (i & 31)
            bit = (int(mbits[i // 32]) >> (i & 31)) & 1
            rc = (int(codes[i // 2]) >> (4 * (i & 1))) & 0xF
            rv = _MAGS[rc & 7] * (-1 if rc & 8 else 1)
            outs["out_guided"][i] = deq(brute_guided(z, bit)[0], neg, Xq)
            outs["out_rtn"][i] = deq(brute_rtn(z)[0], neg, Xq)
            outs["out_full"][i] = deq(brute_full_guided(z, rv)[0], neg, Xq)
    return dict(codes=codes, mbits=mbits, scales=scales.reshape(rows, cols // 32), mask=mask,
                **{k: v.reshape(rows, cols) for k, v in outs.items()})


# ---------------------------------------------------------------------------
# W4A8: E4M3 (FP8) activations with MX scales
# ---------------------------------------------------------------------------

def brute_mx8_scale(amax: Fraction) -> int:
    """The E8M0 byte putting amax / X in [256, 512) (E4M3's top binade), by
    search over all bytes; the smallest byte when none does (or amax = 0)."""
    if amax == 0:
        return 0
    hits = [b for b in range(255) if 256 <= amax / e8m0_value(b) < 512]
    assert len(hits) <= 1
    return hits[0] if hits else 0


def brute_e4m3_rtn(a: Fraction) -> int:
    """Nearest E4M3 magnitude code to clip(a, 448), ties to the even code."""
    a = min(a, Fraction(448))
    best = None
    for v, b in E4M3_TABLE:
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and (b & 1) == 0):
            best = (d, b)
    return best[1]


def brute_e4m3_bracket(a: Fraction) -> tuple[int, int]:
    a = min(a, Fraction(448))
    lo = max((t for t in E4M3_TABLE if t[0] <= a), key=lambda t: t[0])[1]
    hi = min((t for t in E4M3_TABLE if t[0] >= a), key=lambda t: t[0])[1]
    return lo, hi


def brute_mx8_pipeline(x_roll: np.ndarray, x_train: np.ndarray):
    """MXFP8 capture on x_roll, then guided / RTN / full-guided forwards of
    x_train, by exhaustive searches over the E4M3 values."""
    rows, cols = x_roll.shape
    n = rows * cols
    xr = [bf16_bits_to_float(int(h)) for h in x_roll.reshape(-1)]
    xt = [bf16_bits_to_float(int(h)) for h in x_train.reshape(-1)]
    codes = np.zeros(n, np.uint8)
    mbits = np.zeros(n // 32, np.uint32)
    scales = np.zeros(n // 32, np.uint8)
    outs = {k: np.zeros(n, np.uint16) for k in ("out_guided", "out_rtn", "out_full")}
    mask = np.zeros(n // 32, np.uint32)

    def deq(code: int, neg: bool, X: Fraction) -> int:
        v = f32(float(e4m3_value(code) * X))      # exact
        return float_to_bf16_bits(-v if neg else v)

    for b in range(n // 32):
        blk = range(32 * b, 32 * b + 32)
        sb = brute_mx8_scale(max(Fraction(abs(xr[i])) for i in blk))
        scales[b] = sb
        Xq = e8m0_value(sb)
        X = f32(float(Xq))
        for i in blk:
            z = f32(xr[i]) / X
            c = brute_e4m3_rtn(Fraction(float(abs(z))))
            codes[i] = (0x80 if np.signbit(z) else 0) | c
            mbits[i // 32] |= (c & 1) << (i & 31)
        for i in blk:
            z = f32(xt[i]) / X
            neg = bool(np.signbit(z))
            a = Fraction(float(abs(z)))
            if a <= 448:
                mask[i // 32] |= 1 << (i & 31)
            lo, hi = brute_e4m3_bracket(a)
            bit = (int(mbits[i // 32]) >> (i & 31)) & 1
            g = lo if lo == hi or (lo & 1) == bit else hi
            rc = int(codes[i])
            rv = e4m3_value(rc & 0x7F) * (-1 if rc & 0x80 else 1)
            s = -1 if neg else 1
            dl, dh = abs(s * e4m3_value(lo) - rv), abs(s * e4m3_value(hi) - rv)
            full = hi if dh < dl else lo
            outs["out_guided"][i] = deq(g, neg, Xq)
            outs["out_rtn"][i] = deq(brute_e4m3_rtn(a), neg, Xq)
            outs["out_full"][i] = deq(full, neg, Xq)
    return dict(codes=codes, mbits=mbits, scales=scales.reshape(rows, cols // 32), mask=mask,
                **{k: v.reshape(rows, cols) for k, v in outs.items()})

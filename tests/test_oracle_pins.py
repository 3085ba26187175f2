"""Pins for the CPU oracle: brute force, library routines, closed forms and
the worked example.  None of these runs the CUDA path.

Sources: the rcap.io post "TRACE: Rollout-Guided Quantization-Aware Training
for FP4" -- the rounding-boundary example, the section on rollout-guided
rounding (the per-site guarantee), the compact-cache section (1 mantissa bit
plus scales; ~6x smaller) and the pseudocode listing.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import _bruteforce as bf
from fp4_quantization_aware_trace_b200 import inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
MIDS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def _nextafter(x, n):
    x = np.float32(x)
    for _ in range(abs(n)):
        x = np.nextafter(x, np.float32(np.inf if n > 0 else -np.inf), dtype=np.float32)
    return x


def _lattice(points, ulps=(-2, -1, 0, 1, 2)):
    out = []
    for p in points:
        for u in ulps:
            out.append(float(_nextafter(p, u)))
    return out


def _z_lattice():
    pts = E2M1 + MIDS + [6.0, 7.0, 1e30]
    vals = _lattice(pts) + [float(v) for v in np.random.default_rng(5).uniform(0, 7, 400)]
    vals += [0.0, 1e-45, 1e-38, 0.1]
    return sorted(v for v in vals if v >= 0.0)


# --------------------------------------------------------------------------
# bf16 <-> fp32 (library: torch's CPU conversion, round to nearest even)
# --------------------------------------------------------------------------

def test_bf16_decode_all_patterns(oracle_mod):
    pats = np.arange(1 << 16, dtype=np.uint32)
    exp = (pats >> 7) & 0xFF
    finite = pats[exp != 0xFF]
    ref = torch.from_numpy(finite.astype(np.int32).astype(np.int16)).view(torch.bfloat16).float()
    got = np.array([oracle_mod.bf16_to_f32(int(h)) for h in finite], np.float32)
    assert np.array_equal(got.view(np.uint32), ref.numpy().view(np.uint32))


def test_bf16_encode_vs_torch(oracle_mod):
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 0x7F7FFFFF, 20000, dtype=np.uint32)
    # exact ties, ties +- 1, near-overflow, subnormals
    ties = (rng.integers(0, 0x7F7F, 2000, dtype=np.uint32) << 16) | 0x8000
    extra = np.concatenate([ties, ties + 1, ties - 1,
                            np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7F8001, 0x00008000,
                                      0x00018000, 0x00000001, 0x007FFFFF], np.uint32)])
    allbits = np.concatenate([bits, extra])
    allbits = np.concatenate([allbits, allbits | 0x80000000])
    f = allbits.view(np.float32)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.f32_to_bf16(float(v)) for v in f], np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------
# E4M3 (brute force in exact rationals; library: torch float8_e4m3fn)
# --------------------------------------------------------------------------

def test_e4m3_decode_all_bytes(oracle_mod):
    for b in range(0x7F):
        assert Fraction(oracle_mod.e4m3_to_f32(b)) == bf.e4m3_value(b)
    ref = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle_mod.e4m3_to_f32(b) for b in range(0x7F)], np.float32)
    assert np.array_equal(got, ref)
    assert math.isnan(oracle_mod.e4m3_to_f32(0x7F))


def _e4m3_lattice():
    vals = [float(v) for v, _ in bf.E4M3_TABLE]
    mids = [float((a + b) / 2) for (a, _), (b, _) in zip(bf.E4M3_TABLE, bf.E4M3_TABLE[1:])]
    pts = _lattice(vals + mids + [464.0, 480.0]) + [448.5, 463.9, 500.0, 1e6, 3e38,
                                                     2.0 ** -10, 2.0 ** -11, 1e-40]
    rng = np.random.default_rng(2)
    pts += [float(v) for v in np.exp(rng.uniform(np.log(1e-4), np.log(500), 3000)).astype(np.float32)]
    return [p for p in pts if p >= 0.0]


def test_e4m3_encode_vs_bruteforce(oracle_mod):
    for t in _e4m3_lattice():
        assert oracle_mod.f32_to_e4m3(t) == bf.brute_e4m3(t), t


def test_e4m3_encode_vs_torch(oracle_mod):
    rng = np.random.default_rng(3)
    t = np.concatenate([
        np.exp(rng.uniform(np.log(1e-6), np.log(463.9), 200000)).astype(np.float32),
        np.array(_e4m3_lattice(), np.float32)])
    t = t[t < 464.0]                  # torch gives NaN beyond the saturation tie
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    lib = oracle_mod._load()
    got = np.array([lib.oracle_f32_to_e4m3(float(v)) for v in t], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates(oracle_mod):
    for t in (448.0, 455.9, 464.0, 464.1, 1e9, 3.4e38):
        assert oracle_mod.f32_to_e4m3(t) == 0x7E


# --------------------------------------------------------------------------
# E2M1 round-to-nearest, bracket and guided choice (brute force)
# --------------------------------------------------------------------------

def test_e2m1_rtn_vs_bruteforce(oracle_mod):
    for a in _z_lattice():
        ac = min(a, 6.0)
        v, c = bf.brute_rtn(Fraction(ac))
        assert oracle_mod.e2m1_rtn(ac) == c, a
        assert Fraction(E2M1[c]) == v


def test_e2m1_ties_go_to_even_code(oracle_mod):
    # every midpoint goes to the neighbour whose mantissa bit is 0
    for m in MIDS:
        c = oracle_mod.e2m1_rtn(m)
        assert c % 2 == 0
        assert abs(E2M1[c] - m) == min(abs(v - m) for v in E2M1)


def test_bracket_vs_bruteforce(oracle_mod):
    for a in _z_lattice():
        ac = min(a, 6.0)
        lo, hi = oracle_mod.e2m1_bracket(ac)
        (vl, cl), (vh, ch) = bf.brute_bracket(Fraction(ac))
        assert (lo, hi) == (cl, ch), a


@pytest.mark.parametrize("sign", [1, -1])
def test_guided_choice_vs_bruteforce(oracle_mod, sign):
    for a in _z_lattice():
        ac = min(a, 6.0)
        for bit in (0, 1):
            c = oracle_mod.guided_code(ac, bit)
            v, cb = bf.brute_guided(Fraction(sign * ac), bit)
            assert c == cb and Fraction(E2M1[c]) == abs(v), (a, bit)


def test_guided_enumerates_all_codewords(oracle_mod):
    """On a codeword the bracket collapses and the bit is ignored; strictly
    between two neighbours the bit decides, and it always picks a member
    whose mantissa bit equals it."""
    for k, v in enumerate(E2M1):
        for bit in (0, 1):
            assert oracle_mod.guided_code(v, bit) == k
    for k in range(7):
        inner = (E2M1[k] + E2M1[k + 1]) / 2
        for a in (float(_nextafter(E2M1[k], 1)), inner, float(_nextafter(E2M1[k + 1], -1))):
            for bit in (0, 1):
                c = oracle_mod.guided_code(a, bit)
                assert c in (k, k + 1) and (c & 1) == bit


# --------------------------------------------------------------------------
# Whole pipeline vs brute force on tiny inputs
# --------------------------------------------------------------------------

def _special_tiny(rows=2, cols=64, seed=11):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[0, :16] = 0.0                       # a zero block
    x[0, 16] = -0.0
    x[0, 17:20] = [1e-39, -3e-40, 2.0 ** -133]   # bf16 subnormals
    x[1, 5] = 40.0                         # an outlier
    x[1, 40:48] = [0.25, -0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -6.0]
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xt = (xb.float() * (1 + 0.02 * torch.from_numpy(rng.standard_normal((rows, cols)).astype(np.float32)))).to(torch.bfloat16)
    g = torch.from_numpy(rng.standard_normal((rows, cols)).astype(np.float32)).to(torch.bfloat16)
    return inputs.bits(xb), inputs.bits(xt), inputs.bits(g)


def _tiny_cases():
    cases = [_special_tiny()]
    for seed, (r, c) in enumerate([(1, 32), (3, 32), (2, 96), (4, 64)]):
        s = inputs.tiny_site(100 + seed, r, c, eps=0.02)
        cases.append((inputs.bits(s.x_roll), inputs.bits(s.x_train), inputs.bits(s.grad)))
    # x_train == x_roll
    s = inputs.tiny_site(7, 2, 64)
    cases.append((inputs.bits(s.x_roll), inputs.bits(s.x_roll), inputs.bits(s.grad)))
    # all zeros
    z = np.zeros((1, 32), np.uint16)
    z[0, 1::2] = 0x8000
    cases.append((z, z, np.full((1, 32), 0x3F80, np.uint16)))
    return cases


@pytest.mark.parametrize("case", range(7))
def test_pipeline_vs_bruteforce(oracle_mod, case):
    xr, xt, g = _tiny_cases()[case]
    ref = bf.brute_pipeline(xr, xt, g)
    codes, mbits, scales, gscale = oracle_mod.capture(xr)
    assert np.array_equal(gscale.view(np.uint32), ref["gscale"].view(np.uint32))
    assert np.array_equal(scales, ref["scales"])
    assert np.array_equal(codes, ref["codes"])
    assert np.array_equal(mbits, ref["mbits"])
    out, mask = oracle_mod.guided_fwd(xt, mbits, scales, gscale)
    assert np.array_equal(mask, ref["mask"])
    assert np.array_equal(out, ref["out_guided"])
    out_r, mask_r = oracle_mod.rtn_fwd(xt, scales, gscale)
    assert np.array_equal(out_r, ref["out_rtn"]) and np.array_equal(mask_r, mask)
    gin = oracle_mod.fq_bwd(g, mask)
    assert np.array_equal(gin, ref["grad_in"])


# --------------------------------------------------------------------------
# Worked example (golden fixture from the post's rounding-boundary paragraph)
# --------------------------------------------------------------------------

def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                vals[k] = float.fromhex(v) if v.startswith("0x") else float(v)
    return vals


def test_straddle_example(oracle_mod):
    g = _golden("straddle_example.txt")
    row = np.zeros(32, np.float32)
    row[0] = g["amax_element"]
    row[16] = g["block_max_element"]
    row[17] = g["x_roll"]
    x_roll = inputs.bits(torch.from_numpy(row[None]).to(torch.bfloat16))
    row_t = row.copy()
    row_t[17] = g["x_train"]
    x_train = inputs.bits(torch.from_numpy(row_t[None]).to(torch.bfloat16))
    assert bf.bf16_bits_to_float(int(x_roll[0, 17])) - bf.bf16_bits_to_float(int(x_train[0, 17])) == g["bf16_gap"]

    codes, mbits, scales, gscale = oracle_mod.capture(x_roll)
    assert gscale[0] == g["s_g"]
    assert scales[0, 1] == int(g["block_scale_byte"])
    out_roll, _ = oracle_mod.rtn_fwd(x_roll, scales, gscale)
    out_rtn, _ = oracle_mod.rtn_fwd(x_train, scales, gscale)
    out_gd, _ = oracle_mod.guided_fwd(x_train, mbits, scales, gscale)
    f = lambda a: bf.bf16_bits_to_float(int(a[0, 17]))
    assert f(out_roll) == g["rtn_roll"]
    assert f(out_rtn) == g["rtn_train"]
    assert f(out_roll) - f(out_rtn) == g["fp4_gap_rtn"]
    assert f(out_gd) == g["guided_train"]
    assert f(out_roll) - f(out_gd) == g["fp4_gap_guided"]
    # vanilla QAT: the training side's own capture gives the same scale here
    _, _, sc_t, gs_t = oracle_mod.capture(x_train)
    out_v, _ = oracle_mod.rtn_fwd(x_train, sc_t, gs_t)
    assert f(out_v) == g["rtn_train"]


# --------------------------------------------------------------------------
# Closed forms and invariants that the mathematics fixes
# --------------------------------------------------------------------------

def test_compact_cache_size_closed_form(oracle_mod):
    """1 mantissa bit + one E4M3 byte per 16 elements = 1.5 bits/element,
    against 4 + 0.5 = 4.5 for the full NVFP4 codes: 3x, and keeping only the
    later half of the layers doubles it to the post's ~6x."""
    s = inputs.tiny_site(0, 64, 256)
    codes, mbits, scales, gscale = oracle_mod.capture(inputs.bits(s.x_roll))
    n = 64 * 256
    compact = mbits.nbytes + scales.nbytes
    full = codes.nbytes + scales.nbytes
    assert mbits.nbytes * 8 == n and scales.nbytes * 16 == n and codes.nbytes * 2 == n
    assert compact * 8 / n == 1.5 and full * 8 / n == 4.5
    assert full / compact == 3.0
    assert 2 * full / compact == 6.0


def test_global_scale_closed_form(oracle_mod):
    """s_g is amax/2688 rounded once, and the block holding the amax element
    gets the top E4M3 scale 448 with that element at code 7 (|z| ~ 6)."""
    for seed in range(4):
        s = inputs.tiny_site(seed, 8, 128)
        x = inputs.bits(s.x_roll)
        codes, mbits, scales, gscale = oracle_mod.capture(x)
        xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float().numpy()
        amax = np.abs(xf).max()
        assert gscale[0] == np.float32(amax) / np.float32(2688.0)
        err = abs(Fraction(float(gscale[0])) - Fraction(float(amax)) / 2688)
        assert err <= Fraction(float(np.spacing(gscale[0]))) / 2
        i = int(np.abs(xf).reshape(-1).argmax())
        assert scales.reshape(-1)[i // 16] == 0x7E
        assert oracle_mod.unpack_codes(codes)[i] & 7 == 7
    z = np.zeros((2, 32), np.uint16)
    assert oracle_mod.capture(z)[3][0] == 1.0


def test_scale_and_sign_symmetry(oracle_mod):
    """Multiplying x by 2^k scales s_g by 2^k and leaves codes, bits and
    block scales unchanged; negating x flips only the code sign bits."""
    s = inputs.tiny_site(3, 16, 64)
    xf = s.x_roll.float()
    base = oracle_mod.capture(inputs.bits(s.x_roll))
    for k in (-20, -3, 5, 40):
        xk = inputs.bits((xf * 2.0 ** k).to(torch.bfloat16))
        c, m, sc, gs = oracle_mod.capture(xk)
        assert np.array_equal(c, base[0]) and np.array_equal(m, base[1])
        assert np.array_equal(sc, base[2]) and gs[0] == np.float32(base[3][0] * 2.0 ** k)
    c, m, sc, gs = oracle_mod.capture(inputs.bits(-s.x_roll))
    assert np.array_equal(oracle_mod.unpack_codes(c), oracle_mod.unpack_codes(base[0]) ^ 8)
    assert np.array_equal(m, base[1]) and np.array_equal(sc, base[2])


def test_rtn_error_bound(oracle_mod):
    """Round-to-nearest fake-quant is within half a codeword gap (in units of
    s = s_g * s_b) of x wherever |z| <= 6, up to the bf16 rounding of the
    output."""
    s = inputs.tiny_site(9, 32, 128)
    x = inputs.bits(s.x_roll)
    codes, mbits, scales, gscale = oracle_mod.capture(x)
    out, mask = oracle_mod.rtn_fwd(x, scales, gscale)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float().numpy().reshape(-1)
    of = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).float().numpy().reshape(-1)
    sb = np.array([oracle_mod.e4m3_to_f32(int(b)) for b in scales.reshape(-1)], np.float64)
    d = np.repeat(sb, 16) * float(gscale[0])
    inside = oracle_mod.unpack_bits(mask).astype(bool)
    z = np.abs(xf) / d
    half_gap = np.where(z < 2, 0.25, np.where(z < 4, 0.5, 1.0))
    err = np.abs(xf - of)
    assert np.all((err <= half_gap * d * (1 + 1e-5) + np.abs(of) * 2.0 ** -8)[inside])
    # E4M3 rounds the block scale down by up to 1/16 relative, so a block
    # maximum can land just past 6 s; it is clipped to the codeword 6
    clipped = ~inside
    assert np.all(z[clipped] > 6) and np.all(z[clipped] < 6 * (1 + 1 / 15))
    assert np.all(np.abs(np.abs(of[clipped]) - 6 * d[clipped]) <= 6 * d[clipped] * 2.0 ** -8)


def _codes_pair(oracle_mod, site, num_groups=1, offsets=None):
    xr, xt = inputs.bits(site.x_roll), inputs.bits(site.x_train)
    codes, mbits, scales, gscale = oracle_mod.capture(xr, num_groups, offsets)
    q_roll = oracle_mod.unpack_codes(codes)
    q_star = oracle_mod.fake_quant_codes(xt, scales, gscale, mbits, num_groups, offsets).reshape(-1)
    q_rtn = oracle_mod.fake_quant_codes(xt, scales, gscale, None, num_groups, offsets).reshape(-1)
    return q_roll, q_star, q_rtn


def _signed_value(c):
    v = np.array(E2M1)[c & 7]
    return np.where(c & 8, -v, v)


def test_guided_equals_rollout_when_inputs_equal(oracle_mod):
    """x_train == x_roll  =>  q* == q_roll bitwise at every site."""
    s = inputs.single_activation(0, rows=64, cols=512)
    s.x_train = s.x_roll.clone()
    q_roll, q_star, q_rtn = _codes_pair(oracle_mod, s)
    assert np.array_equal(q_star, q_roll)
    assert np.array_equal(q_rtn, q_roll)


def test_per_site_guarantee(oracle_mod):
    """Rollout-guided rounding: wherever q_roll lies in the bracket of the
    training value, q* == q_roll; there |q* - q_roll| <= |RTN(z) - q_roll|.
    At the post's noise levels no site has q_roll outside the bracket."""
    s = inputs.single_activation(0, rows=128, cols=1024)
    q_roll, q_star, q_rtn = _codes_pair(oracle_mod, s)
    vr, vs, vn = _signed_value(q_roll), _signed_value(q_star), _signed_value(q_rtn)
    # bracket membership of q_roll, decided from the guided code and its
    # neighbour: q_roll in bracket <=> q* == q_roll by value (same bit) or
    # the bracket collapsed onto a codeword adjacent to q_roll
    assert np.all(np.abs(vs - vr) <= np.abs(vn - vr))
    mism_rtn = np.count_nonzero(vn != vr)
    mism_guided = np.count_nonzero(vs != vr)
    assert mism_rtn > 0                 # the noise makes some sites straddle
    assert mism_guided < mism_rtn


def test_grouped_capture_matches_per_group(oracle_mod):
    """A grouped capture equals capturing every group on its own, including
    an empty group (scale 1.0) and ragged group sizes."""
    s = inputs.tiny_site(21, 40, 64)
    x = inputs.bits(s.x_roll)
    x[10:17] = inputs.bits((s.x_roll[10:17].float() * 1000).to(torch.bfloat16))
    offs = np.array([0, 3, 3, 17, 40], np.int64)
    codes, mbits, scales, gscale = oracle_mod.capture(x, 4, offs)
    assert gscale[1] == 1.0
    for g in range(4):
        r0, r1 = offs[g], offs[g + 1]
        if r0 == r1:
            continue
        c, m, sc, gs = oracle_mod.capture(x[r0:r1])
        assert gs[0] == gscale[g]
        assert np.array_equal(c, codes[r0 * 32:r1 * 32])
        assert np.array_equal(m, mbits[r0 * 2:r1 * 2])
        assert np.array_equal(sc, scales[r0:r1])
    xt = inputs.bits(s.x_train)
    out, mask = oracle_mod.guided_fwd(xt, mbits, scales, gscale, 4, offs)
    for g in (0, 2, 3):
        r0, r1 = offs[g], offs[g + 1]
        o, mk = oracle_mod.guided_fwd(xt[r0:r1], mbits[r0 * 2:r1 * 2], scales[r0:r1], gscale[g:g + 1])
        assert np.array_equal(o, out[r0:r1]) and np.array_equal(mk, mask[r0 * 2:r1 * 2])


def test_row_entry_points_match_whole_tensor(oracle_mod):
    s = inputs.tiny_site(4, 12, 96)
    x, xt = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    offs = np.array([0, 5, 12], np.int64)
    codes, mbits, scales, gscale = oracle_mod.capture(x, 2, offs)
    amax = oracle_mod.group_amax(x, 2, offs)
    assert np.array_equal(np.array([oracle_mod.global_scale(float(a)) for a in amax], np.float32), gscale)
    rg = np.repeat(gscale, np.diff(offs))
    rows = np.array([1, 6, 11])
    c, m, sc = oracle_mod.capture_rows(x[rows], rg[rows])
    c_all = codes.reshape(12, 48)
    assert np.array_equal(c.reshape(3, 48), c_all[rows])
    assert np.array_equal(m.reshape(3, 3), mbits.reshape(12, 3)[rows])
    out, mask = oracle_mod.guided_fwd(xt, mbits, scales, gscale, 2, offs)
    o, mk = oracle_mod.fake_quant_rows(xt[rows], rg[rows], scales[rows], mbits.reshape(12, 3)[rows])
    assert np.array_equal(o, out[rows]) and np.array_equal(mk.reshape(3, 3), mask.reshape(12, 3)[rows])


def test_ste_backward_definition(oracle_mod):
    rng = np.random.default_rng(0)
    g = rng.integers(0, 1 << 16, 256, dtype=np.uint32).astype(np.uint16)
    mask = rng.integers(0, 1 << 32, 8, dtype=np.uint64).astype(np.uint32)
    gin = oracle_mod.fq_bwd(g, mask)
    keep = oracle_mod.unpack_bits(mask).astype(bool)
    assert np.array_equal(gin[keep], g[keep]) and np.all(gin[~keep] == 0)


# --------------------------------------------------------------------------
# Full-information guidance (the cache keeps the whole rollout code)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("sign", [1, -1])
def test_full_guided_choice_vs_bruteforce(oracle_mod, sign):
    rolls = [c for c in range(16)]
    for a in _z_lattice():
        z = sign * a
        for rc in rolls:
            rv = Fraction(E2M1[rc & 7]) * (-1 if rc & 8 else 1)
            v, c = bf.brute_full_guided(Fraction(z), rv)
            got = oracle_mod.full_guided_code(z, rc)
            assert got == c and Fraction(E2M1[got]) == abs(v), (z, rc)


def test_full_guidance_guarantee_holds_everywhere(oracle_mod):
    """With the whole rollout code, |q* - q_roll| <= |RTN(z) - q_roll| at
    every site (the per-site guarantee of rollout-guided rounding), also
    where the training value has moved past the neighbouring codewords; it
    agrees with 1-bit guidance wherever q_roll lies in the bracket."""
    s = inputs.tiny_site(17, 96, 512, eps=0.25)     # large drift on purpose
    xr, xt = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    codes, mbits, scales, gscale = oracle_mod.capture(xr)
    q_roll = oracle_mod.unpack_codes(codes)
    q_full = oracle_mod.full_guided_codes(xt, codes, scales, gscale).reshape(-1)
    q_bit = oracle_mod.fake_quant_codes(xt, scales, gscale, mbits).reshape(-1)
    q_rtn = oracle_mod.fake_quant_codes(xt, scales, gscale, None).reshape(-1)
    vr, vf, vb, vn = (_signed_value(c) for c in (q_roll, q_full, q_bit, q_rtn))
    assert np.all(np.abs(vf - vr) <= np.abs(vn - vr))
    violated = np.abs(vb - vr) > np.abs(vn - vr)      # where 1 bit is not enough
    assert violated.sum() > 0                         # the drift produces some
    # q_roll lies in the bracket exactly where full guidance reproduces it;
    # there the 1-bit choice reproduces it too
    in_bracket = vf == vr
    assert np.all(vb[in_bracket] == vr[in_bracket])
    assert np.count_nonzero(vf != vr) <= np.count_nonzero(vb != vr)


def test_full_guidance_equals_rollout_when_inputs_equal(oracle_mod):
    s = inputs.single_activation(0, rows=32, cols=256)
    xr = inputs.bits(s.x_roll)
    codes, mbits, scales, gscale = oracle_mod.capture(xr)
    q = oracle_mod.full_guided_codes(xr, codes, scales, gscale).reshape(-1)
    assert np.array_equal(q, oracle_mod.unpack_codes(codes))
    out_f, mask_f = oracle_mod.full_guided_fwd(xr, codes, scales, gscale)
    out_r, mask_r = oracle_mod.rtn_fwd(xr, scales, gscale)
    assert np.array_equal(out_f, out_r) and np.array_equal(mask_f, mask_r)


def test_full_guided_pipeline_vs_bruteforce(oracle_mod):
    """Whole full-information forward on tiny inputs against brute force:
    exhaustive bracket and nearest-member search, numpy fp32, torch bf16."""
    for xr, xt, g in _tiny_cases()[:5]:
        ref = bf.brute_pipeline(xr, xt, g)
        codes, mbits, scales, gscale = oracle_mod.capture(xr)
        rows, cols = xr.shape
        q_roll = oracle_mod.unpack_codes(codes)
        out, mask = oracle_mod.full_guided_fwd(xt, codes, scales, gscale)
        assert np.array_equal(mask, ref["mask"])
        xtf = [bf.bf16_bits_to_float(int(h)) for h in xt.reshape(-1)]
        s_g = np.float32(gscale[0])
        expect = np.zeros(rows * cols, np.uint16)
        for b in range(rows * cols // 16):
            sbv = bf.e4m3_value(int(scales.reshape(-1)[b]))
            d = s_g * np.float32(float(sbv))
            for i in range(16 * b, 16 * b + 16):
                if d == 0:
                    z, neg = Fraction(0), bool(np.signbit(np.float32(xtf[i])))
                else:
                    zf = np.float32(xtf[i]) / d
                    z, neg = Fraction(float(zf)), bool(np.signbit(zf))
                rc = int(q_roll[i])
                rv = Fraction(E2M1[rc & 7]) * (-1 if rc & 8 else 1)
                v, _ = bf.brute_full_guided(z, rv)
                exact = abs(v) * sbv * Fraction(float(s_g))
                f = np.float32(float(exact))
                if v < 0 or (v == 0 and neg):
                    f = -f
                expect[i] = bf.float_to_bf16_bits(f)
        assert np.array_equal(out.reshape(-1), expect)


# --------------------------------------------------------------------------
# Mismatch diagnostic (compact-cache paragraph: mismatched sites are mostly
# one adjacent codeword apart)
# --------------------------------------------------------------------------

def _ladder(c):
    c = np.asarray(c, np.int64)
    return np.where(c & 8, -(c & 7), c & 7)


def test_mismatch_histogram_vs_codes(oracle_mod):
    """The histogram counts the ladder distances of the per-site codes the
    other oracle entry points pick (and brute force on a tiny input)."""
    s = inputs.tiny_site(23, 64, 256, eps=0.05)
    xr, xt = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    codes, mbits, scales, gscale = oracle_mod.capture(xr)
    hist = oracle_mod.mismatch_histogram(xt, codes, scales, gscale)
    q_roll = oracle_mod.unpack_codes(codes)
    q = [oracle_mod.fake_quant_codes(xt, scales, gscale, None).reshape(-1),
         oracle_mod.fake_quant_codes(xt, scales, gscale, mbits).reshape(-1),
         oracle_mod.full_guided_codes(xt, codes, scales, gscale).reshape(-1)]
    for k in range(3):
        d = np.abs(_ladder(q[k]) - _ladder(q_roll))
        assert np.array_equal(hist[k], np.bincount(d, minlength=15))
    assert np.all(hist.sum(axis=1) == xr.size)
    # brute force on the special tiny case
    xr2, xt2, g2 = _special_tiny()
    ref = bf.brute_pipeline(xr2, xt2, g2)
    c2, m2, sc2, gs2 = oracle_mod.capture(xr2)
    h2 = oracle_mod.mismatch_histogram(xt2, c2, sc2, gs2)
    out_g = torch.from_numpy(ref["out_guided"].view(np.int16)).view(torch.bfloat16).float().numpy().reshape(-1)
    out_r = torch.from_numpy(ref["out_rtn"].view(np.int16)).view(torch.bfloat16).float().numpy().reshape(-1)
    qr = oracle_mod.unpack_codes(c2)
    sbv = np.repeat([float(bf.e4m3_value(int(b))) for b in sc2.reshape(-1)], 16)
    d = sbv * float(gs2[0])
    lr = _ladder(qr)
    grid = np.array(E2M1)
    for k, o in ((0, out_r), (1, out_g)):
        mag = np.where(d > 0, np.abs(o) / np.where(d > 0, d, 1), 0)
        code = np.array([int(np.argmin(np.abs(grid - m))) for m in mag])
        lad = np.where(np.signbit(o), -code, code)
        assert np.array_equal(h2[k], np.bincount(np.abs(lad - lr), minlength=15))


def test_mismatch_dominance_and_identity(oracle_mod):
    """Full guidance is at least as close as RTN at every site, so its
    cumulative histogram dominates; identical inputs give all-zero
    distances."""
    s = inputs.tiny_site(29, 64, 512, eps=0.2)
    xr, xt = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    codes, mbits, scales, gscale = oracle_mod.capture(xr)
    h = oracle_mod.mismatch_histogram(xt, codes, scales, gscale).astype(np.int64)
    assert np.all(np.cumsum(h[2]) >= np.cumsum(h[0]))
    assert h[0, 1:].sum() > h[2, 1:].sum()
    h0 = oracle_mod.mismatch_histogram(xr, codes, scales, gscale)
    assert np.all(h0[:, 0] == xr.size) and np.all(h0[:, 1:] == 0)


# --------------------------------------------------------------------------
# MXFP4 variant (results list: the method carries over to MXFP4 W4A4; the
# scale step is the OCP Microscaling one, the E2M1 rounding is unchanged)
# --------------------------------------------------------------------------

def test_e8m0_decode_vs_exact_and_torch(oracle_mod):
    b = np.arange(255, dtype=np.uint8)
    got = np.array([oracle_mod.e8m0_to_f32(int(v)) for v in b], np.float32)
    exact = [bf.e8m0_value(int(v)) for v in b]
    assert all(Fraction(float(g)) == e for g, e in zip(got, exact))
    if hasattr(torch, "float8_e8m0fnu"):
        t = torch.from_numpy(b).view(torch.float8_e8m0fnu).float().numpy()
        assert np.array_equal(t.view(np.uint32), got.view(np.uint32))


def test_mx_scale_vs_bruteforce(oracle_mod):
    """Every bf16 magnitude pattern as a block maximum: the E8M0 byte puts
    amax / X in [4, 8) (E2M1's top binade), clamped at 2^-127."""
    pats = np.arange(0x7F80, dtype=np.uint32)
    vals = (pats << 16).view(np.float32)
    for a in vals[::7].tolist() + [0.0, 2.0 ** -133, 2.0 ** -125, 2.0 ** -124, 3.3e38, 8.0, 7.99, 4.0]:
        a = float(np.float32(a))
        assert oracle_mod.mx_scale(a) == bf.brute_mx_scale(Fraction(a)), a


@pytest.mark.parametrize("case", range(7))
def test_mx_pipeline_vs_bruteforce(oracle_mod, case):
    xr, xt, _ = _tiny_cases()[case]
    ref = bf.brute_mx_pipeline(xr, xt)
    codes, mbits, scales = oracle_mod.mx_capture(xr)
    assert np.array_equal(scales, ref["scales"])
    assert np.array_equal(codes, ref["codes"])
    assert np.array_equal(mbits, ref["mbits"])
    out, mask = oracle_mod.mx_guided_fwd(xt, mbits, scales)
    assert np.array_equal(mask, ref["mask"]) and np.array_equal(out, ref["out_guided"])
    out_r, mask_r = oracle_mod.mx_rtn_fwd(xt, scales)
    assert np.array_equal(mask_r, ref["mask"]) and np.array_equal(out_r, ref["out_rtn"])
    out_f, mask_f = oracle_mod.mx_full_guided_fwd(xt, codes, scales)
    assert np.array_equal(mask_f, ref["mask"]) and np.array_equal(out_f, ref["out_full"])


def test_mx_scale_invariance_and_identity(oracle_mod):
    """x * 2^k shifts every E8M0 byte by k and leaves the codes alone (no
    clamping and no underflow in range); guided on x_roll itself returns the
    rollout's codes; codes decode to the outputs."""
    s = inputs.tiny_site(41, 16, 256, eps=0.02, outliers=False)
    xr = inputs.bits(s.x_roll)
    codes, mbits, scales = oracle_mod.mx_capture(xr)
    for k in (-20, 7):
        xk = inputs.bits((s.x_roll.float() * 2.0 ** k).to(torch.bfloat16))
        ck, mk, sk = oracle_mod.mx_capture(xk)
        assert np.array_equal(sk.astype(int), scales.astype(int) + k)
        assert np.array_equal(ck, codes) and np.array_equal(mk, mbits)
    q = oracle_mod.mx_fake_quant_codes(xr, scales, mbits=mbits).reshape(-1)
    assert np.array_equal(q, oracle_mod.unpack_codes(codes))
    q_full = oracle_mod.mx_fake_quant_codes(xr, scales, rcodes=codes).reshape(-1)
    assert np.array_equal(q_full, q)
    out, _ = oracle_mod.mx_guided_fwd(xr, mbits, scales)
    mag = np.array(E2M1)[q & 7] * np.repeat([oracle_mod.e8m0_to_f32(int(b)) for b in scales.reshape(-1)], 32)
    val = np.where(q & 8, -mag, mag).astype(np.float32)
    exp = inputs.bits(torch.from_numpy(val).to(torch.bfloat16).reshape(xr.shape))
    assert np.array_equal(out, exp)


def test_mx_rtn_error_bound(oracle_mod):
    """Inside the block's range, RTN lands within half a grid gap of z; the
    top binade can clip (amax / X up to 8 > 6)."""
    s = inputs.tiny_site(43, 32, 256, eps=0.0)
    xr = inputs.bits(s.x_roll)
    _, _, scales = oracle_mod.mx_capture(xr)
    q = oracle_mod.mx_fake_quant_codes(xr, scales).reshape(-1)
    X = np.repeat([oracle_mod.e8m0_to_f32(int(b)) for b in scales.reshape(-1)], 32)
    z = np.abs(s.x_roll.float().numpy().reshape(-1)) / X
    v = np.array(E2M1)[q & 7]
    gap = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))
    inside = z <= 6
    assert np.all(np.abs(z[inside] - v[inside]) <= gap[inside] / 2 + 1e-7)
    assert np.all(v[~inside] == 6.0) and np.all(z[~inside] < 8)


# --------------------------------------------------------------------------
# Block-scale layout of a block-scaled FP4 GEMM (128 x 4 tiles)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("rows,scols", [(1, 1), (5, 6), (128, 4), (130, 5), (300, 64), (257, 129)])
def test_swizzle_scales_vs_library(oracle_mod, rows, scols):
    """Against vllm's row-major -> 128x4 scale swizzle (a torch routine that
    runs on the CPU; it is written for E8M0 scales of 32-element blocks and
    the layout depends only on the scale matrix's shape)."""
    mx = pytest.importorskip("vllm.model_executor.layers.quantization.utils.mxfp8_utils")
    rng = np.random.default_rng(rows * 1000 + scols)
    lin = rng.integers(1, 256, (rows, scols), dtype=np.uint8)
    ref = mx.swizzle_mxfp8_scale(torch.from_numpy(lin), rows, scols * 32).reshape(-1).numpy()
    got = oracle_mod.swizzle_scales(lin)
    assert got.shape == ref.shape and np.array_equal(got, ref)


def test_swizzle_scales_is_a_padded_permutation(oracle_mod):
    rows, scols = 300, 37
    lin = (np.arange(rows * scols) % 251 + 1).astype(np.uint8).reshape(rows, scols)
    got = oracle_mod.swizzle_scales(lin)
    assert got.size == 384 * 40
    assert np.count_nonzero(got) == rows * scols
    assert np.array_equal(np.sort(got[got != 0]), np.sort(lin.reshape(-1)))


def test_mismatch_distance_by_grid_index(oracle_mod):
    """The ladder distance equals the number of steps between the two values
    in the sorted list of the 15 signed E2M1 codewords (+0 and -0 one point),
    on independent rollout / training values, so that opposite signs and long
    distances occur."""
    rng = np.random.default_rng(77)
    xr = rng.standard_normal((16, 256)).astype(np.float32) * np.exp(rng.standard_normal((16, 256)))
    xt = rng.standard_normal((16, 256)).astype(np.float32) * np.exp(rng.standard_normal((16, 256)))
    xr_b = inputs.bits(torch.from_numpy(xr).to(torch.bfloat16))
    xt_b = inputs.bits(torch.from_numpy(xt).to(torch.bfloat16))
    codes, mbits, scales, gscale = oracle_mod.capture(xr_b)
    hist = oracle_mod.mismatch_histogram(xt_b, codes, scales, gscale)
    grid = [float(v) for v, _ in bf.SIGNED_GRID]          # ascending, 15 points
    assert len(grid) == 15

    def index(c):
        v = float(Fraction(bf._MAGS[c & 7])) * (-1.0 if c & 8 else 1.0)
        return grid.index(v + 0.0)                           # -0.0 -> +0.0

    q_roll = oracle_mod.unpack_codes(codes)
    rules = [oracle_mod.fake_quant_codes(xt_b, scales, gscale, None).reshape(-1),
             oracle_mod.fake_quant_codes(xt_b, scales, gscale, mbits).reshape(-1),
             oracle_mod.full_guided_codes(xt_b, codes, scales, gscale).reshape(-1)]
    for k in range(3):
        d = np.array([abs(index(int(a)) - index(int(b))) for a, b in zip(rules[k], q_roll)])
        assert np.array_equal(hist[k], np.bincount(d, minlength=15)), k
    assert hist[0, 2:].sum() > 0 and np.count_nonzero(hist[0]) > 5   # long distances occur


# --------------------------------------------------------------------------
# W4A8: E4M3 activations with MX scales (results list: the W4A8 setting)
# --------------------------------------------------------------------------

def test_mx8_scale_vs_bruteforce(oracle_mod):
    pats = np.arange(0x7F80, dtype=np.uint32)
    vals = (pats << 16).view(np.float32)
    for a in vals[::11].tolist() + [0.0, 2.0 ** -133, 2.0 ** -119, 2.0 ** -118, 3.3e38, 512.0, 511.0,
                                   256.0, 448.0]:
        a = float(np.float32(a))
        assert oracle_mod.mx8_scale(a) == bf.brute_mx8_scale(Fraction(a)), a


def test_e4m3_bracket_and_guided_vs_bruteforce(oracle_mod):
    """On every E4M3 value, every midpoint and +-1 ulp around them, both bits:
    the bracket and the guided choice against exhaustive search; neighbouring
    codes alternate their lowest bit, so one member qualifies."""
    vals = sorted(float(v) for v, _ in bf.E4M3_TABLE)
    pts = set(vals)
    for a, b in zip(vals[:-1], vals[1:]):
        m = np.float32((a + b) / 2)
        pts.update([float(m), float(np.nextafter(m, np.float32(0))), float(np.nextafter(m, np.float32(1e9)))])
    pts.update([460.0, 1e6])
    for a in sorted(pts):
        a32 = float(np.float32(a))
        lo, hi = bf.brute_e4m3_bracket(Fraction(a32))
        assert oracle_mod.e4m3_bracket(min(a32, 448.0)) == (lo, hi), a32
        for bit in (0, 1):
            want = lo if lo == hi or (lo & 1) == bit else hi
            assert oracle_mod.e4m3_guided_code(min(a32, 448.0), bit) == want
        assert oracle_mod.e4m3_full_guided_code(a32, lo) == lo
        assert oracle_mod.e4m3_full_guided_code(-a32, 0x80 | hi) == hi


@pytest.mark.parametrize("case", range(7))
def test_mx8_pipeline_vs_bruteforce(oracle_mod, case):
    xr, xt, _ = _tiny_cases()[case]
    ref = bf.brute_mx8_pipeline(xr, xt)
    codes, mbits, scales = oracle_mod.mx8_capture(xr)
    assert np.array_equal(scales, ref["scales"])
    assert np.array_equal(codes, ref["codes"])
    assert np.array_equal(mbits, ref["mbits"])
    out, mask = oracle_mod.mx8_guided_fwd(xt, mbits, scales)
    assert np.array_equal(mask, ref["mask"]) and np.array_equal(out, ref["out_guided"])
    out_r, _ = oracle_mod.mx8_rtn_fwd(xt, scales)
    assert np.array_equal(out_r, ref["out_rtn"])
    out_f, _ = oracle_mod.mx8_full_guided_fwd(xt, codes, scales)
    assert np.array_equal(out_f, ref["out_full"])


def test_mx8_identity_and_cache_size(oracle_mod):
    """Guided on x_roll itself reproduces the rollout codes (all three rules);
    the W4A8 compact cache is 1 bit + one E8M0 byte per 32 elements = 1.25
    bits per element against 8.25 for the full FP8 codes."""
    s = inputs.tiny_site(47, 16, 256, eps=0.02)
    xr = inputs.bits(s.x_roll)
    codes, mbits, scales = oracle_mod.mx8_capture(xr)
    for kw in ({}, {"mbits": mbits}, {"rcodes": codes}):
        q = oracle_mod.mx8_fake_quant_codes(xr, scales, **kw).reshape(-1)
        assert np.array_equal(q, codes)
    n = xr.size
    assert (mbits.nbytes + scales.nbytes) * 8 / n == 1.25
    assert (codes.nbytes + scales.nbytes) * 8 / n == 8.25


def test_e4m3_encode_vs_torch_dense(oracle_mod):
    """Every 97th fp32 bit pattern below the saturation tie 464 (11.7 M
    values, subnormals included) against torch's float8_e4m3fn conversion."""
    end = 0x43E80000                                  # 464.0
    idx = np.arange(0, end, 97, dtype=np.uint32)
    ref = torch.from_numpy(idx.view(np.float32).copy()).to(torch.float8_e4m3fn)
    ref = ref.view(torch.uint8).numpy()
    got = np.empty(idx.size, np.uint8)
    for k0 in range(0, idx.size, 65536):              # contiguous runs, every 97th kept
        k1 = min(idx.size, k0 + 65536)
        first = int(idx[k0])
        got[k0:k1] = oracle_mod.e4m3_sweep(first, int(idx[k1 - 1]) - first + 1)[::97]
    assert np.array_equal(got, ref)


def test_mx_mismatch_histogram_vs_codes(oracle_mod):
    """The MXFP4 histogram re-bins the per-site codes of the pinned MX entry
    points by grid index, on independent values (sign flips) and on a
    drifted pair."""
    rng = np.random.default_rng(78)
    grid = [float(v) for v, _ in bf.SIGNED_GRID]

    def index(c):
        return grid.index(float(Fraction(bf._MAGS[c & 7])) * (-1.0 if c & 8 else 1.0) + 0.0)

    xr = (rng.standard_normal((16, 256)) * np.exp(rng.standard_normal((16, 256)))).astype(np.float32)
    pairs = [(xr, (rng.standard_normal((16, 256)) * 3).astype(np.float32)),
             (xr, (xr * (1 + 0.05 * rng.standard_normal((16, 256)))).astype(np.float32))]
    for a, b in pairs:
        xr_b = inputs.bits(torch.from_numpy(a).to(torch.bfloat16))
        xt_b = inputs.bits(torch.from_numpy(b).to(torch.bfloat16))
        codes, mbits, scales = oracle_mod.mx_capture(xr_b)
        hist = oracle_mod.mx_mismatch_histogram(xt_b, codes, scales)
        q_roll = oracle_mod.unpack_codes(codes)
        rules = [oracle_mod.mx_fake_quant_codes(xt_b, scales).reshape(-1),
                 oracle_mod.mx_fake_quant_codes(xt_b, scales, mbits=mbits).reshape(-1),
                 oracle_mod.mx_fake_quant_codes(xt_b, scales, rcodes=codes).reshape(-1)]
        for k in range(3):
            d = np.array([abs(index(int(p)) - index(int(q))) for p, q in zip(rules[k], q_roll)])
            assert np.array_equal(hist[k], np.bincount(d, minlength=15)), k


def _boundary_lattice():
    """Every codeword and midpoint of [0, 6], +-1..3 ulps around each, and
    random magnitudes (float32)."""
    pts = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0]
    out = set()
    for p in pts:
        v = np.float32(p)
        for k in range(4):
            out.add(float(v))
            v = np.nextafter(v, np.float32(7.0))
        v = np.float32(p)
        for k in range(3):
            v = np.nextafter(v, np.float32(-1.0))
            if v >= 0:
                out.add(float(v))
    rng = np.random.default_rng(77)
    out.update(float(a) for a in rng.uniform(0, 6, 3000).astype(np.float32))
    out.update(float(a) for a in (rng.uniform(0, 1e-3, 200).astype(np.float32)))
    return sorted(a for a in out if 0.0 <= a <= 6.0)


def test_guided_rules_keep_round_to_nearest_where_it_agrees(oracle_mod):
    """The guided forwards start from round to nearest and recompute only the
    sites where a rule may differ.  Pinned here with the oracle's own rules:
    the 1-bit rule returns the round-to-nearest code wherever that code's
    mantissa bit equals the cached bit, and the full-information rule returns
    it wherever the rollout's signed code equals it (both signs, z beyond 6
    clipped)."""
    lat = _boundary_lattice()
    for a in lat:
        r = oracle_mod.e2m1_rtn(a)
        assert oracle_mod.guided_code(a, r & 1) == r, a
        for z in (a, -a, a * 1.5 + 6.0, -(a * 1.5 + 6.0)):
            zc = min(abs(z), 6.0)
            rs = (8 if np.signbit(np.float32(z)) else 0) | oracle_mod.e2m1_rtn(np.float32(zc))
            assert oracle_mod.full_guided_code(z, rs) == rs & 7, z
    # and the premise is not vacuous: where the bit disagrees, the 1-bit rule
    # moves off round to nearest at every site that is not a codeword
    moved = sum(oracle_mod.guided_code(a, 1 - (oracle_mod.e2m1_rtn(a) & 1)) !=
                oracle_mod.e2m1_rtn(a) for a in lat)
    assert moved > 0.9 * len(lat)

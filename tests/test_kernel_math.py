"""Exhaustive CPU proofs of the two arithmetic identities the CUDA kernels
use in place of a per-element division and a codeword table (restated in
plain C in kernel_math_check.c):

  * the FMA-corrected reciprocal quotient equals IEEE x/d for every bf16
    numerator and fp32 denominator significand (both result binades), and
    run negated it equals -(x/d) there and keeps the sign opposite to x's
    for every finite bf16 x (zeros included) across the denominators' range;
  * rounding a + M down / up (M a power-of-two magic addend per binade)
    gives the E2M1 floor / ceiling of every fp32 a in [0, 6] and the
    mantissa bit of the floor codeword.

A negative control (the uncorrected product; a wrong addend) must fail, so
the check itself is known to detect errors."""
from __future__ import annotations

import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kernel_math_check.c")


def _build(tmp_path, *defs):
    exe = str(tmp_path / ("kmc" + "".join(d.lower() for d in defs)))
    flags = ["-O2", "-ffp-contract=off", "-frounding-math"]
    probe = subprocess.run(["gcc", "-mfma", "-E", "-x", "c", "/dev/null"], capture_output=True)
    if probe.returncode == 0:
        flags.append("-mfma")
    subprocess.run(["gcc", *flags, *[f"-D{d}" for d in defs], "-o", exe, SRC, "-lm", "-lpthread"],
                   check=True)
    return exe


def test_quotient_and_grid_identities_hold_exhaustively(tmp_path):
    r = subprocess.run([_build(tmp_path)], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "quotient: 0 mismatches" in r.stdout and "grid rounding: 0 mismatches" in r.stdout
    assert "negated quotient: 0 mismatches of 2147483648 cases, 0 in the sign" in r.stdout


def test_negative_control_fails(tmp_path):
    r = subprocess.run([_build(tmp_path, "NO_CORRECTION")], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 1
    assert "quotient: 0 mismatches" not in r.stdout
    assert "grid rounding: 0 mismatches" not in r.stdout


def test_sign_control_fails(tmp_path):
    """Negating the unnegated step's result loses the sign of x = -0 (its
    z is +0): the sign sweep must see it."""
    r = subprocess.run([_build(tmp_path, "SIGN_CONTROL")], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 1
    assert ", 0 in the sign" not in r.stdout

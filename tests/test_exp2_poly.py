"""Pins for the FMA-pipe exp2 of the forward kernel's softmax (csrc/exp2_poly.h,
written by csrc/gen_exp2_poly.py): the cubic 1 + f (C1 + C2 f + C3 f^2) is
checked against 2^f from the mathematics, evaluated the way the kernel does it
(float32 Horner with fused multiply-adds, range reduction by adding 1.5 * 2^23,
exponent added to the bit pattern, the argument clamped at -125 by the caller)."""
import os
import re
import subprocess
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "video_block_sparse_b200", "csrc")


def _coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    c = {int(m.group(1)): float(m.group(2)) for m in re.finditer(r"#define VSA_EXP2_C(\d) ([0-9.eE+-]+)f", text)}
    return np.float32(c[1]), np.float32(c[2]), np.float32(c[3])


def _fma32(a, b, c):
    # a*b + c with one rounding to float32 (the float64 product of two float32 is exact)
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)


def _ex2_fma(x):
    """The kernel's arithmetic, in numpy: t = x + 1.5 * 2^23, n = t - 1.5 * 2^23,
    f = x - n, p = 1 + f (C1 + f (C2 + f C3)), result bits = bits(p) + (bits(t) << 23)."""
    c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = _fma32(n, np.float32(-1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.ones_like(f))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_polynomial_is_exact_at_zero_and_within_its_bound():
    c1, c2, c3 = _coeffs()
    f = np.linspace(-0.5, 0.5, 200001)
    p = 1.0 + f * (float(c1) + f * (float(c2) + f * float(c3)))
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() <= 1.02e-4
    assert 1.0 + 0.0 * float(c1) == 1.0  # p(0) = 1 by construction (no constant term to round)
    # equioscillation: a minimax fit touches its bound at several points of the interval
    assert np.sum(rel > 0.95 * rel.max()) >= 4


def test_kernel_arithmetic_matches_exp2_over_the_softmax_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125.0, 8.5, 400000), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9, dtype=np.float64) + 0.5]).astype(np.float32)
    y = _ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 1.1e-4, float(rel.max())
    # integers give exact powers of two (f = 0 and p(0) = 1)
    ints = np.arange(-120, 9, dtype=np.float32)
    assert np.array_equal(_ex2_fma(ints), np.exp2(ints.astype(np.float64)).astype(np.float32))


def test_clamp_keeps_masked_logits_finite_and_tiny():
    y = _ex2_fma(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y <= np.float32(2.0 ** -124))


def test_generator_reproduces_the_header(tmp_path):
    """The committed header is what the generator writes."""
    import shutil
    gen = os.path.join(CSRC, "gen_exp2_poly.py")
    work = tmp_path / "csrc"
    work.mkdir()
    shutil.copy(gen, work / "gen_exp2_poly.py")
    subprocess.run([sys.executable, str(work / "gen_exp2_poly.py")], check=True, capture_output=True)
    assert (work / "exp2_poly.h").read_text() == open(os.path.join(CSRC, "exp2_poly.h")).read()

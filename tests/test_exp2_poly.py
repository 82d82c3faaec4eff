"""The MXFP8 forward takes a quarter of its exponentials on the FMA pipe
(exp2_poly in csrc/ptx.cuh): x = n + f with n the nearest integer, 2^f from a
degree-3 minimax polynomial on [-1/2, 1/2], n added to the exponent field.
Pinned here against 2^x itself: the coefficients are read from the source and
the routine is replayed in fp32 (single-rounding FMAs, the 1.5 * 2^23 rounding
constant, the integer add into the exponent field) on a dense grid."""
import math
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "causal_flash_attention_packed_b200" / "csrc" / "ptx.cuh"
BOUND = 7.6e-5  # minimax relative error of the fit is 7.48e-5


def _coeffs():
    text = SRC.read_text()
    got = {}
    for k in range(4):
        m = re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f", text)
        assert m, f"coefficient kExp2C{k} not found"
        got[k] = np.float32(float(m.group(1)))
    return [got[k] for k in range(4)]


def _fma32(a, b, c):
    # one rounding to fp32 of the exact a*b+c (a, b, c are fp32, so fp64 holds a*b exactly)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    big = np.float32(12582912.0)
    t = (xc + big).astype(np.float32)
    n = (t - big).astype(np.float32)
    f = (xc - n).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    r = bits.astype(np.uint32).view(np.float32)
    return np.where(x < np.float32(-125.0), np.float32(0.0), r)


def test_relative_error_bound_on_the_forward_range():
    # the forward feeds s * scale * log2(e) - M <= 8 (the running reference
    # moves once the row maximum exceeds it by 8)
    xs = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.linspace(-1.0, 1.0, 400_001),
                         np.arange(-125, 9, dtype=np.float64) + 0.5]).astype(np.float32)
    y = exp2_poly(xs).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= BOUND, rel.max()


def test_integers_and_halves():
    for k in range(-125, 9):
        for f in (0.0, 0.25, -0.25, 0.5, -0.5):
            x = np.float32(k + f)
            if x < -125:
                continue
            got = float(exp2_poly(np.array([x]))[0])
            want = math.ldexp(2.0 ** f, k)
            assert abs(got - want) <= BOUND * want, (k, f, got, want)


def test_zero_below_range_and_at_minus_infinity():
    xs = np.array([-125.5, -126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    assert np.all(exp2_poly(xs) == 0.0)


def test_fit_equioscillates():
    # a minimax fit of degree 3 reaches its error level with alternating signs
    # at (at least) 3 + 2 points of the interval (exact arithmetic, fp32 coefficients)
    c0, c1, c2, c3 = (float(c) for c in _coeffs())
    f = np.linspace(-0.5, 0.5, 1_000_001)
    err = (c0 + f * (c1 + f * (c2 + f * c3))) / np.exp2(f) - 1.0
    level = abs(err).max()
    assert level < BOUND
    peaks = [0] + [i for i in range(1, len(f) - 1)
                   if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(f) - 1]
    signs = [np.sign(err[i]) for i in peaks if abs(err[i]) >= 0.99 * level]
    alternations = sum(1 for a, b in zip(signs, signs[1:]) if a != b)
    assert alternations >= 4, signs

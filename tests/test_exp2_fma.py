"""Error bound of the kernels' FMA-pipe exponential (exp2_fma2 in csrc/ptx.cuh).

The forward kernels evaluate a fixed share of their 2^x on the FMA pipe:
x is clamped at -120, split as x = n + f with n = round(x) (by adding and
subtracting 1.5 * 2^23), 2^f comes from a degree-3 polynomial on [-1/2, 1/2]
and 2^n is applied by an integer add into the exponent field.  This test
replays those fp32 steps in numpy, with the coefficients and constants read
from the committed source, and checks the relative error against np.exp2
over the range the kernels use, the clamp, and the exponent add near the
bottom of the range.  It runs on the CPU.
"""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_55_b200", "csrc", "ptx.cuh")


def _body():
    src = open(SRC).read()
    m = re.search(r"float2 exp2_fma2\(float2 x\) \{(.*?)\n\}", src, re.S)
    assert m, "exp2_fma2 not found in ptx.cuh"
    return m.group(1)


def _constants():
    body = _body()
    magic = float(re.search(r"kMagic = ([0-9.e+-]+)f", body).group(1))
    clamp = float(re.search(r"fmaxf\(x\.x, (-?[0-9.]+)f\)", body).group(1))
    # Horner coefficients, highest degree first, in the order of the ffma2 calls.
    pairs = re.findall(r"make_float2\(([0-9.e+-]+)f, \1f\)", body)
    coef = [float(c) for c in pairs if abs(float(c)) != 1.0 and abs(float(c)) != magic]
    assert len(coef) == 4, coef
    return np.float32(magic), np.float32(clamp), [np.float32(c) for c in coef]


def _fma32(a, b, c):
    # a*b is exact in float64 (24 + 24 bits); one rounding of the sum to fp32
    # matches a fused multiply-add except in rare double-rounding ties.
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def replay(x):
    magic, clamp, (c3, c2, c1, c0) = _constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), clamp)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = _fma32(j, np.float32(-1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) + p.view(np.uint32).astype(np.uint64)
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32), f


def test_constants_match_the_fit():
    _, clamp, coef = _constants()
    assert clamp == -120.0
    # the committed coefficients are the fit of gen_exp2_poly.py (lowest degree last here)
    import importlib.util
    spec = importlib.util.spec_from_file_location("gen", os.path.join(os.path.dirname(SRC), "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, err = gen.fit(3)
    np.testing.assert_allclose(np.array(coef[::-1], dtype=np.float64), c, rtol=1e-6)
    assert err < 1e-4


def test_reduction_is_exact():
    x = np.linspace(-120.0, 8.0, 1_000_003, dtype=np.float32)
    _, f = replay(x)
    assert np.all(np.abs(f) <= 0.5)
    n = np.round(x.astype(np.float64))
    np.testing.assert_array_equal(f.astype(np.float64), x.astype(np.float64) - n)


def test_relative_error_bound_over_the_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32),
        rng.uniform(-120.0, 8.0, 1_000_000).astype(np.float32),
        # integers and half-integers, where the reduction switches n
        (np.arange(-120, 9).astype(np.float32)[:, None] + np.array([-0.5, -1e-4, 0.0, 1e-4, 0.5], np.float32)).ravel(),
    ])
    x = x[(x >= -120.0) & (x <= 8.0)]
    y, _ = replay(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) / ref - 1.0)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert rel.max() <= 1e-4, rel.max()
    # the claimed 2^-13.5 bound with a margin for the fp32 rounding steps
    assert rel.max() <= 8.3e-5 * 1.05, rel.max()


def test_bottom_of_the_range_stays_normal():
    """n down to -120: the exponent field of p (126 or 127) plus n stays >= 6,
    so the integer add never leaves the normal range."""
    x = np.linspace(-120.0, -110.0, 100_001, dtype=np.float32)
    y, _ = replay(x)
    exp_field = (y.view(np.uint32) >> 23) & 0xFF
    assert exp_field.min() >= 6
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1e-4


@pytest.mark.parametrize("x", [-120.5, -121.0, -126.0, -150.0, -1e30, -np.inf])
def test_clamp_below_minus_120(x):
    y, _ = replay(np.array([x], dtype=np.float32))
    y120, _ = replay(np.array([-120.0], dtype=np.float32))
    assert y[0] == y120[0]
    assert abs(float(y[0]) / 2.0 ** -120 - 1.0) <= 1e-4
    assert float(y[0]) < 1e-36

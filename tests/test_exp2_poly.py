"""The FMA-pipe 2^x of the kernels (csrc/exp2_poly.cuh), checked on the CPU.

The kernels evaluate 2 of every 8 key pairs' exponentials with this polynomial,
so its constants and its stated accuracy are pinned here against the exact
2^x: the header's coefficients are read from the source (not retyped), the
evaluation is emulated step by step in FP32 (each FMA rounded once, as
fma.rn.f32 does), and the relative error must stay within the bound the header
states, 2.2e-7, over the argument range the softmax uses (x <= 8, clamped at
-125).  A wrong digit in a coefficient, a dropped term or a wrong range
reduction fails this.
"""
import os
import re

import numpy as np
import pytest

HEADER = os.path.join(os.path.dirname(__file__), "..", "online_softmax_tcgen05_b200", "csrc",
                      "exp2_poly.cuh")


def _constants():
    src = open(HEADER).read()
    c = {}
    for name, val in re.findall(r"constexpr float (EXP2_\w+) = ([0-9.eE+-]+)f;", src):
        c[name] = np.float32(float(val))
    return c


def _fma32(a, b, c):
    # fma.rn.f32: a*b is exact in float64 for float32 inputs; the sum is rounded to
    # float64 and then to float32 (the double rounding can matter only in ties far
    # below this test's tolerance)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _add32(a, b):
    return (a.astype(np.float64) + b.astype(np.float64)).astype(np.float32)


def exp2_poly_emulated(x):
    """The steps of exp2_poly2 for one lane, in FP32."""
    c = _constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    R = c["EXP2_ROUND"]
    y = _add32(x, np.full_like(x, R))
    n = _add32(y, np.full_like(x, -R))
    f = _fma32(n, np.full_like(x, -1.0), x)
    p = _fma32(np.full_like(x, c["EXP2_C5"]), f, np.full_like(x, c["EXP2_C4"]))
    for k in ("EXP2_C3", "EXP2_C2", "EXP2_C1", "EXP2_C0"):
        p = _fma32(p, f, np.full_like(x, c[k]))
    # exponent add: bits(p) + bits(y) * 2^23 (mod 2^32)
    bits = (p.view(np.uint32).astype(np.uint64) +
            (y.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_constants_present():
    c = _constants()
    assert set(c) == {"EXP2_C0", "EXP2_C1", "EXP2_C2", "EXP2_C3", "EXP2_C4", "EXP2_C5",
                      "EXP2_ROUND"}
    assert c["EXP2_ROUND"] == np.float32(1.5 * 2 ** 23)
    # 2^f = 1 + f ln 2 + ...: the leading coefficients within the fit's adjustment
    assert abs(float(c["EXP2_C0"]) - 1.0) < 1e-6
    assert abs(float(c["EXP2_C1"]) - np.log(2.0)) < 1e-5


def test_relative_error_within_stated_bound():
    rng = np.random.default_rng(20261202)
    # dense over the reduced interval around several exponents, plus random x
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float64)
    xs = [np.float32(n) + f.astype(np.float32) for n in (-120, -30, -10, -1, 0, 3, 7)]
    xs.append(rng.uniform(-124.0, 8.0, 400000).astype(np.float32))
    x = np.concatenate(xs).astype(np.float32)
    got = exp2_poly_emulated(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(got / exact - 1.0)
    assert np.isfinite(got).all()
    assert rel.max() <= 2.2e-7, rel.max()


def test_integer_arguments_and_clamp():
    x = np.arange(-125, 9, dtype=np.float32)
    got = exp2_poly_emulated(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0) <= 2.2e-7)
    # below the clamp every value is 2^-125 (times p(0)): far below any row sum's
    # last bit and zero after an E4M3 cast (the smallest E4M3 subnormal is 2^-9)
    low = exp2_poly_emulated(np.array([-126.0, -200.0, -1e30], dtype=np.float32))
    assert np.allclose(low.astype(np.float64), 2.0 ** -125, rtol=2.2e-7)


@pytest.mark.parametrize("x", [8.0, 0.0, -0.5, 0.5])
def test_reduction_boundaries(x):
    got = float(exp2_poly_emulated(np.array([x], dtype=np.float32))[0])
    assert abs(got / 2.0 ** x - 1.0) <= 2.2e-7

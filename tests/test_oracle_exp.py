"""Pins for the oracle's exp / sigmoid / SiLU (the router's and SwiGLU's
nonlinearity; sigmoid router per "Colibri：在笔记本上跑744B参数的AI模型",
"关键特性").  The oracle's exp is its own (Cody-Waite + Taylor); these tests
tie it to the mathematics: correctly rounded e^x from Python's double exp,
exact special values, limits and symmetry."""
import math
from fractions import Fraction

import numpy as np


def _ulps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    ai = a.view(np.int32).astype(np.int64)
    bi = b.view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


def _exp_rn(x: np.ndarray) -> np.ndarray:
    # double exp (error < 1 ulp of double) rounded once to binary32
    return np.array([math.exp(float(v)) for v in x], np.float64).astype(np.float32)


def test_exp_special_values(ora):
    assert ora.exp(0.0) == 1.0
    assert ora.exp(-0.0) == 1.0
    assert ora.exp(float("inf")) == float("inf")
    assert ora.exp(-float("inf")) == 0.0
    assert math.isnan(ora.exp(float("nan")))
    assert ora.exp(89.0) == float("inf")
    assert ora.exp(-104.0) == 0.0
    assert ora.sigmoid(0.0) == 0.5
    assert ora.silu(0.0) == 0.0
    assert ora.sigmoid(200.0) == 1.0
    assert ora.sigmoid(-200.0) == 0.0


def test_exp_dense_sweep_within_one_ulp(ora):
    x = np.linspace(-103.9, 88.72, 400_001).astype(np.float32)
    y = ora.exp_array(x)
    u = _ulps(y, _exp_rn(x))
    assert u.max() <= 1, (u.max(), x[u.argmax()])


def test_exp_every_float_in_unit_interval_sample(ora):
    # every 97th binary32 in [-1, 1): the reduction r = x here, k = 0 or +-1
    bits = np.arange(0x3F800000, 0, -97, dtype=np.int64).astype(np.int32)
    pos = bits.view(np.float32)
    x = np.concatenate([pos, -pos])
    u = _ulps(ora.exp_array(x), _exp_rn(x))
    assert u.max() <= 1


def test_exp_integer_arguments(ora):
    for k in range(-80, 80):
        want = np.float32(math.exp(k))
        got = np.float32(ora.exp(float(k)))
        assert _ulps(np.array([got]), np.array([want]))[0] <= 1, k


def test_sigmoid_against_double(ora):
    x = np.linspace(-30, 30, 200_001).astype(np.float32)
    y = ora.sigmoid_array(x).astype(np.float64)
    ref = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 4 * 2.0 ** -24


def test_sigmoid_symmetry_and_monotone(ora):
    x = np.linspace(-20, 20, 40_001).astype(np.float32)
    s = ora.sigmoid_array(x).astype(np.float64)
    sm = ora.sigmoid_array(-x).astype(np.float64)
    assert np.abs(s + sm - 1.0).max() < 3 * 2.0 ** -24
    assert np.all(np.diff(s) >= 0)


def test_silu_against_double(ora):
    x = np.linspace(-20, 20, 100_001).astype(np.float32)
    y = ora.silu_array(x).astype(np.float64)
    xd = x.astype(np.float64)
    ref = xd / (1.0 + np.exp(-xd))
    err = np.abs(y - ref)
    assert np.all(err <= 5 * 2.0 ** -24 * np.abs(ref) + 1e-45)


def test_taylor_coefficients_are_rounded_reciprocal_factorials():
    # The definition's constants C2..C7 = 1/n! rounded to binary32, and the
    # Cody-Waite split of ln 2; checked here from exact rationals.
    want = {n: float.fromhex(h) for n, h in
            {2: "0x1.0p-1", 3: "0x1.555556p-3", 4: "0x1.555556p-5", 5: "0x1.111112p-7",
             6: "0x1.6c16c2p-10", 7: "0x1.a01a02p-13"}.items()}
    for n, c in want.items():
        exact = Fraction(1, math.factorial(n))
        # nearest binary32 to the rational: compare neighbours
        c32 = np.float32(c)
        up = np.nextafter(c32, np.float32(1))
        dn = np.nextafter(c32, np.float32(0))
        d = abs(Fraction(float(c32)) - exact)
        assert d <= abs(Fraction(float(up)) - exact) and d <= abs(Fraction(float(dn)) - exact), n
    hi = np.float32(float.fromhex("0x1.62e4p-1"))
    # hi keeps 15 significant bits: k*hi exact for |k| < 256
    m = int(np.array([hi]).view(np.int32)[0]) & 0x7FFFFF
    assert m & 0x1FF == 0
    lo = np.float32(float.fromhex("0x1.7f7d1cp-20"))
    # lo is the binary32 nearest to ln 2 - hi (within half an ulp of lo)
    half_ulp = float(np.spacing(lo)) / 2
    assert abs(float(hi) + float(lo) - math.log(2)) <= half_ulp + 2.0 ** -60

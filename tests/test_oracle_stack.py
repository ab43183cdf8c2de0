"""Pins of the oracle's stack pieces (harness of the 8-layer workload):
the residual x_next = x + MoE(RMSNorm(x)) adds the layer output to the
UN-normalised x, one correctly rounded binary32 addition per element.

Checked against exact rational arithmetic (not against numpy's float32 add)
and by a construction: a layer whose experts are all zero outputs zeros, so
a stack of such layers must return x bit for bit (a residual that added to
RMSNorm(x), or dropped x, fails)."""
from fractions import Fraction

import numpy as np

from tests.helpers import oracle_stack_forward


def _round_f32(q: Fraction) -> np.float32:
    """Round an exact rational to binary32, ties to even (normal range)."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    n, r = divmod(a, ulp)
    n = int(n)
    if r * 2 > ulp or (r * 2 == ulp and n % 2 == 1):
        n += 1
    return np.float32(sign * float(n * ulp))


def test_residual_add_exact_sums(ora):
    x = np.array([[1.0, -2.5, 3.25, 0.0, -0.0, 1e-3]], np.float32)
    m = np.array([[2.0, 2.5, -1.25, -0.0, -0.0, 0.0]], np.float32)
    got = ora.residual_add(x, m)
    want = [_round_f32(Fraction(float(a)) + Fraction(float(b))) for a, b in zip(x.ravel(), m.ravel())]
    assert np.array_equal(got.ravel(), np.array(want, np.float32))
    assert np.signbit(got[0, 4])  # -0 + -0 = -0


def test_residual_add_rounds_half_to_even(ora):
    # 1 + 2^-24 is half an ulp above 1 (tie -> 1); 1 + 3*2^-24 ties up to 1 + 2^-22
    x = np.array([[1.0, 1.0, 1.0 + 2.0 ** -23, 3.0]], np.float32)
    m = np.array([[2.0 ** -24, 3 * 2.0 ** -24, 2.0 ** -24, 2.0 ** -23]], np.float32)
    got = ora.residual_add(x, m)
    for g, a, b in zip(got.ravel(), x.ravel(), m.ravel()):
        assert g == _round_f32(Fraction(float(a)) + Fraction(float(b)))
    assert got[0, 0] == np.float32(1.0)
    assert got[0, 1] == np.float32(1.0 + 2.0 ** -22)
    assert got[0, 2] == np.float32(1.0 + 2.0 ** -22)


def test_residual_add_random_against_rationals(ora):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((4, 128)) * 3).astype(np.float32)
    m = (rng.standard_normal((4, 128)) * 0.1).astype(np.float32)
    got = ora.residual_add(x, m)
    for g, a, b in zip(got.ravel(), x.ravel(), m.ravel()):
        assert g == _round_f32(Fraction(float(a)) + Fraction(float(b)))


def test_stack_of_zero_expert_layers_returns_x(ora, syn):
    cfg = syn.config("tiny")
    H, I = cfg["hidden"], cfg["inter"]
    zero = ora.QExpert(np.zeros((I, H // 2), np.uint8), np.zeros(I, np.float32),
                       np.zeros((I, H // 2), np.uint8), np.zeros(I, np.float32),
                       np.zeros((H, I // 2), np.uint8), np.zeros(H, np.float32))
    x = syn.tokens(cfg, 3)
    out = oracle_stack_forward(cfg, x, 3, expert_fn=lambda layer, e, shared: zero)
    assert np.array_equal(out.view(np.uint32), x.view(np.uint32))


def test_stack_residual_uses_the_unnormalised_input(ora, syn):
    """One layer: out = x + layer(RMSNorm(x)), element by element."""
    from tests.helpers import oracle_layer_forward
    cfg = syn.config("tiny")
    x = syn.tokens(cfg, 2) * np.float32(3.0)
    out = oracle_stack_forward(cfg, x, 1)
    m, _, _, _ = oracle_layer_forward(cfg, ora.rmsnorm(x, cfg.get("rms_eps", 1e-5)), 0)
    want = np.array([_round_f32(Fraction(float(a)) + Fraction(float(b))) for a, b in zip(x.ravel(), m.ravel())],
                    np.float32).reshape(x.shape)
    assert np.array_equal(out, want)

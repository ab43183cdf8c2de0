"""The seeded input generator: published SplitMix64 outputs, the
Irwin-Hall normal's moments, uniform range, reproducibility and row access."""
import numpy as np


def test_splitmix64_published_outputs(syn):
    # SplitMix64 started at state 0: its first three outputs
    assert syn.draw(0, 0) == 0xE220A8397B1DCDAF
    assert syn.draw(0, 1) == 0x6E789E6AA1B965F4
    assert syn.draw(0, 2) == 0x06C45D188009454F
    # started at state 1234567
    assert syn.draw(1234567, 0) == 6457827717110365317
    assert syn.draw(1234567, 1) == 3203168211198807973


def test_normal_moments(syn):
    n = syn.normal(2_000_000, 0, 0, 77, 0.5).astype(np.float64)
    assert abs(n.mean()) < 3 * 0.5 / np.sqrt(n.size) * 2
    assert abs(n.std() - 0.5) < 0.002
    # Irwin-Hall-12 is bounded by 6 sigma
    assert np.abs(n).max() <= 3.0


def test_uniform_range(syn):
    u = syn.uniform(1_000_000, 0, 0, 78, -0.05, 0.05)
    assert u.min() >= -0.05 and u.max() < 0.05
    assert abs(u.mean()) < 1e-3


def test_reproducible_and_offsets(syn):
    a = syn.normal(1000, 3, 2, 50, 1.0)
    b = syn.normal(1000, 3, 2, 50, 1.0)
    assert np.array_equal(a, b)
    c = syn.normal(500, 3, 2, 50, 1.0, i0=500)
    assert np.array_equal(a[500:], c)
    assert not np.array_equal(a, syn.normal(1000, 3, 3, 50, 1.0))
    assert not np.array_equal(a, syn.normal(1000, 4, 2, 50, 1.0))


def test_rows_match_full_matrix(syn):
    cfg = syn.config("tiny")
    full = syn.expert_matrix(cfg, 0, 3, syn.DOWN)
    rows = syn.expert_rows(cfg, 0, 3, syn.DOWN, [0, 7, 255])
    assert np.array_equal(rows, full[[0, 7, 255]])


def test_bias_boost(syn):
    cfg = syn.config("prefill2048")
    b = syn.bias(cfg)
    raw = syn.uniform(256, 0, 0, syn.TID_BIAS, -0.05, 0.05)
    assert np.array_equal(b[32:], raw[32:])
    assert np.array_equal(b[:32], (raw[:32] + np.float32(0.2)).astype(np.float32))


def test_shared_token_mix(syn):
    cfg = syn.config("decode4")
    x = syn.tokens(cfg)
    base = syn.normal(6144, 0, 0, syn.TID_X_BASE, 1.0)
    n = syn.normal(4 * 6144, 0, 0, syn.TID_X, 1.0).reshape(4, 6144)
    assert np.array_equal(x, (base + (np.float32(0.5) * n).astype(np.float32)).astype(np.float32))

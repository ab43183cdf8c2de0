"""Pins for the oracle's int4 weight quantiser / packer and its Q8_0
activation quantiser.

Sources: "GLM-5.2-colibri-int4架构解析…" (wmrh.cn), section
"GLM-5.2-colibri-int4的量化流程": int4 by np.rint (== lrintf), one F32 scale
per weight row, packed into U8.  "Colibri：在笔记本上跑744B参数的AI模型",
"关键特性": Q8_0-style int8 activations.  The scale rules (absmax/7, clamp
[-8,7], low nibble first; absmax/127 per 32-block) are the readings stated in
the design notes."""
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split("=", 1)
            rows[k.strip()] = v.split()
    return rows


# --------------------------------------------------------------------------
# packing

def test_unpack_pack_identity_all_256_bytes(ora):
    b = np.arange(256, dtype=np.uint8)
    q = ora.unpack_int4(b)
    assert q.min() == -8 and q.max() == 7
    assert np.array_equal(ora.pack_int4(q), b)


def test_pack_unpack_identity_all_pairs(ora):
    v = np.arange(-8, 8, dtype=np.int8)
    q0, q1 = np.meshgrid(v, v, indexing="ij")
    q = np.stack([q0.ravel(), q1.ravel()], axis=1).ravel()
    assert np.array_equal(ora.unpack_int4(ora.pack_int4(q)), q)


def test_pack_golden_fixture(ora):
    g = _read_golden("int4_pack.txt")
    q = np.array([int(t) for t in g["q"]], np.int8)
    want = np.array([int(t, 16) for t in g["bytes"]], np.uint8)
    assert np.array_equal(ora.pack_int4(q), want)
    assert np.array_equal(ora.unpack_int4(want), q)


def test_unpack_nibble_values(ora):
    # low nibble = element 0, high nibble = element 1, two's complement
    assert list(ora.unpack_int4(np.array([0x8F], np.uint8))) == [-1, -8]
    assert list(ora.unpack_int4(np.array([0x71], np.uint8))) == [1, 7]


# --------------------------------------------------------------------------
# int4 rows

def test_int4_closed_form_power_of_two_scale(ora):
    rng = np.random.default_rng(1)
    for c in [2.0 ** -6, 2.0 ** -3, 2.0 ** 4]:
        k = rng.integers(-7, 8, size=(5, 64))
        k[:, 0] = 7
        k[2, 0] = -7  # the absmax may be negative
        w = (k * c).astype(np.float32)
        q, s = ora.quantize_rows_int4(w)
        assert np.all(s == np.float32(c))
        assert np.array_equal(ora.unpack_int4(q.ravel()).reshape(5, 64), k)


def test_int4_closed_form_any_scale(ora):
    rng = np.random.default_rng(2)
    for c in rng.uniform(1e-4, 10.0, size=20):
        k = rng.integers(-7, 8, size=96)
        k[rng.integers(96)] = -7 if rng.random() < 0.5 else 7
        w = (k * np.float32(c)).astype(np.float32)
        q, s = ora.quantize_rows_int4(w[None, :])
        assert np.array_equal(ora.unpack_int4(q.ravel()), k)


def test_int4_half_way_rounds_to_even(ora):
    c = 2.0 ** -4
    m = np.arange(-7, 7)
    halves = m + 0.5  # exactly representable
    w = np.concatenate([[7.0], halves]) * c
    w = np.concatenate([w, np.zeros(2 - len(w) % 2)]).astype(np.float32)
    q, s = ora.quantize_rows_int4(w[None, :])
    assert s[0] == np.float32(c)
    got = ora.unpack_int4(q.ravel())[1:1 + len(halves)]
    want = [round(Fraction(h).limit_denominator()) for h in halves]  # round-half-even
    assert list(got) == want


def test_int4_zero_row(ora):
    q, s = ora.quantize_rows_int4(np.zeros((3, 32), np.float32))
    assert np.all(q == 0) and np.all(s == 0)


def test_int4_error_bound_random_rows(ora, syn):
    w = syn.normal(64 * 512, 0, 0, 999, 0.01).reshape(64, 512)
    q, s = ora.quantize_rows_int4(w)
    qi = ora.unpack_int4(q.ravel()).reshape(64, 512).astype(np.float64)
    err = np.abs(w.astype(np.float64) - qi * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 1e-6))
    assert np.all(np.abs(qi).max(axis=1) == 7)
    assert qi.min() >= -7  # -8 needs |w| > absmax, which cannot happen
    amax = np.abs(w).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(7)).astype(np.float32))


# --------------------------------------------------------------------------
# Q8_0 activations

def test_q8_closed_form(ora):
    rng = np.random.default_rng(3)
    for c in [2.0 ** -7, 0.0123, 3.5]:
        k = rng.integers(-127, 128, size=(4, 64))
        k[:, 0] = 127
        k[:, 32] = -127
        x = (k * np.float32(c)).astype(np.float32)
        q, d = ora.quantize_act_q8(x)
        assert np.array_equal(q.astype(np.int64), k)
        if c == 2.0 ** -7:
            assert np.all(d == np.float32(c))


def test_q8_half_way_rounds_to_even(ora):
    c = 2.0 ** -5
    halves = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 125.5, -125.5, 100.5, -3.5])
    x = np.zeros(32)
    x[0] = 127
    x[1:1 + len(halves)] = halves
    q, d = ora.quantize_act_q8((x * c).astype(np.float32))
    assert d[0, 0] == np.float32(c)
    want = [round(Fraction(h)) for h in halves]
    assert list(q[0, 1:1 + len(halves)]) == want


def test_q8_constant_and_zero_blocks(ora):
    x = np.concatenate([np.full(32, -0.37), np.zeros(32), np.full(32, 5.0)]).astype(np.float32)
    q, d = ora.quantize_act_q8(x)
    assert np.all(q[0, :32] == -127) and np.all(q[0, 64:] == 127)
    assert np.all(q[0, 32:64] == 0) and d[0, 1] == 0


def test_q8_error_bound(ora, syn):
    x = syn.normal(16 * 6144, 0, 0, 998, 1.0).reshape(16, 6144)
    q, d = ora.quantize_act_q8(x)
    deq = q.reshape(16, 192, 32).astype(np.float64) * d[:, :, None]
    err = np.abs(x.reshape(16, 192, 32) - deq)
    assert np.all(err <= d[:, :, None] * (0.5 + 1e-6))
    assert np.all(np.abs(q.reshape(16, 192, 32)).max(axis=2) == 127)


@pytest.mark.parametrize("dim", [32, 64, 6144])
def test_q8_blocks_are_independent(ora, syn, dim):
    x = syn.normal(3 * dim, 0, 0, 997, 2.0).reshape(3, dim)
    q, d = ora.quantize_act_q8(x)
    for b in range(dim // 32):
        qb, db = ora.quantize_act_q8(x[:, 32 * b:32 * b + 32])
        assert np.array_equal(qb, q[:, 32 * b:32 * b + 32])
        assert np.array_equal(db[:, 0], d[:, b])

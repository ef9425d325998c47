"""Pins of the E4M3 quantisation oracle (CPU only): hand values, a brute-force
nearest search over all 256 bit patterns, the scale rule, and attention on
exactly representable inputs; plus planted mistakes."""
import math

import numpy as np
import pytest

from oracle import fp8_oracle as f8
from oracle import svg_oracle as so


HAND = [  # (x, E4M3(x)) derived by hand from the format: 3 mantissa bits, bias 7, max 448, subnormal quantum 2^-9
    (1.0, 1.0), (448.0, 448.0), (500.0, 448.0), (-1e6, -448.0), (464.0, 448.0),
    (1.0625, 1.0),            # 1 + 1/16: halfway between 1.0 and 1.125, ties to the even mantissa 000
    (1.1875, 1.25),           # halfway between 1.125 (001) and 1.25 (010): ties to 010
    (3.3, 3.25),              # binade [2, 4): quantum 0.25
    (0.0625, 0.0625),         # 2^-4, a normal power of two
    (2.0 ** -9, 2.0 ** -9),   # smallest subnormal
    (2.0 ** -10, 0.0),        # half the smallest subnormal: ties to even (zero)
    (3 * 2.0 ** -10, 2.0 ** -8),   # 1.5 subnormal quanta: ties to the even 2
    (0.0, 0.0),
]


def test_e4m3_hand_values():
    for x, want in HAND:
        assert f8.e4m3(x) == want, (x, f8.e4m3(x), want)


def test_e4m3_table_has_the_format_extremes():
    vals = f8.all_e4m3_values()
    pos = np.unique(vals[vals > 0])
    assert len(pos) == 126 and pos.max() == 448.0 and pos.min() == 2.0 ** -9
    assert 240.0 in pos and 256.0 in pos and 288.0 in pos


def test_e4m3_is_the_nearest_table_value():
    table = np.unique(f8.all_e4m3_values())
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.uniform(-4, 3, 4000),
                         rng.choice(table, 500) + rng.uniform(-1e-3, 1e-3, 500)])
    for x in xs:
        c = min(abs(x), 448.0) * np.sign(x)             # saturation first
        d = np.abs(table - c)
        best = table[d == d.min()]
        got = f8.e4m3(x)
        assert got in best, (x, got, best)
        if len(best) == 2:               # a tie: the candidate with the even mantissa, i.e. an even
            # multiple of its binade's quantum
            m = [(abs(b) / (2.0 ** (math.floor(math.log2(abs(b))) - 3)) if abs(b) >= 2 ** -6
                  else abs(b) / 2.0 ** -9) for b in best]
            assert got == best[int(np.argmin([v % 2 for v in m]))]


def test_scales_and_round_trip():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 32)) * rng.uniform(0.01, 50, (64, 1))).astype(np.float32)
    q8, s = f8.quantize_rows(x)
    assert s.dtype == np.float32
    assert np.array_equal(s, np.abs(x).max(1) / np.float32(448))
    assert np.all(np.abs(q8) <= 448) and np.max(np.abs(q8), axis=1).min() == 448.0   # the row maximum maps to 448
    rel = np.abs(q8 * s[:, None] - x) / np.maximum(np.abs(x), 1e-30)
    big = np.abs(x) >= s[:, None] * 2.0 ** -6                 # normal range: half a quantum, 2^-4 relative
    assert rel[big].max() <= 2.0 ** -4 + 1e-7
    k8, sk = f8.quantize_tensor(x)
    assert sk == np.abs(x).max() / np.float32(448) and np.abs(k8).max() == 448.0
    z8, zs = f8.quantize_rows(np.zeros((2, 4), np.float32))
    assert np.all(zs == 1.0) and np.all(z8 == 0.0)


def test_fp8_attention_on_representable_inputs_is_exact():
    """Rows whose values are E4M3 values with row maximum 448 quantise to themselves (scale 1)."""
    rng = np.random.default_rng(2)
    table = np.unique(f8.all_e4m3_values())
    table = table[np.abs(table) <= 8]
    N, D = 40, 16
    q = rng.choice(table, (N, D)); q[:, 0] = 448.0
    k = rng.choice(table, (N, D)); k[0, 0] = 448.0
    v = rng.standard_normal((N, D))
    q_off = np.array([0, 10, 25, 40]); k_off = np.array([0, 20, 40])
    sel = [[0], [0, 1], [1]]
    got, lse = f8.sparse_attention_fp8(q, k, v, q_off, k_off, sel, 0.001)
    want, wlse = so.sparse_attention(q, k, v, q_off, k_off, sel, 0.001)
    assert np.allclose(got, want, rtol=0, atol=1e-12) and np.allclose(lse, wlse, atol=1e-12)


def test_fp8_attention_with_power_of_two_scales_is_exact():
    """Rows that are E4M3 values times a power of two (row maximum 448 * 2^e) have scale 2^e
    exactly, so quantising and dequantising returns them unchanged: the 8-bit attention equals
    the float64 attention with every scale different from 1 (a dropped or inverted scale fails)."""
    rng = np.random.default_rng(3)
    table = np.unique(f8.all_e4m3_values())
    table = table[np.abs(table) <= 8]
    N, D = 48, 16
    eq = rng.integers(-6, 7, N).astype(np.float64)          # per query row
    q = rng.choice(table, (N, D)); q[:, 0] = 448.0
    q = q * 2.0 ** eq[:, None]
    k = rng.choice(table, (N, D)) * 2.0 ** -5; k[3, 2] = 448.0 * 2.0 ** -5   # head scale 2^-5
    v = rng.standard_normal((N, D))
    q8, sq = f8.quantize_rows(q)
    assert np.array_equal(sq, (2.0 ** eq).astype(np.float32)) and np.array_equal(q8 * sq[:, None], q)
    k8, sk = f8.quantize_tensor(k)
    assert sk == np.float32(2.0 ** -5) and np.array_equal(k8 * sk, k)
    q_off = np.array([0, 16, 30, 48]); k_off = np.array([0, 20, 48])
    sel = [[1], [0, 1], [0]]
    got, lse = f8.sparse_attention_fp8(q, k, v, q_off, k_off, sel, 0.05)
    want, wlse = so.sparse_attention(q, k, v, q_off, k_off, sel, 0.05)
    assert np.allclose(got, want, rtol=0, atol=1e-12) and np.allclose(lse, wlse, rtol=1e-12)


def _expect_failure(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_pins_catch_planted_mistakes(monkeypatch):
    # 1. ties away from zero instead of to even
    with monkeypatch.context() as m:
        def away(x):
            x = np.asarray(x, np.float64)
            a = np.abs(x)
            normal = a >= f8.E4M3_MIN_NORMAL
            _, e = np.frexp(np.where(normal, a, 1.0))
            qn = np.where(normal, np.ldexp(1.0, e - 4), f8.E4M3_SUBNORMAL_QUANTUM)
            return np.copysign(np.minimum(np.floor(a / qn + 0.5) * qn, 448.0), x)
        m.setattr(f8, "e4m3", away)
        _expect_failure(test_e4m3_hand_values)
    # 2. no saturation
    with monkeypatch.context() as m:
        orig = f8.e4m3
        m.setattr(f8, "e4m3", lambda x: np.where(np.abs(np.asarray(x, np.float64)) > 448, np.asarray(x, np.float64),
                                                 orig(x)))
        _expect_failure(test_e4m3_hand_values)
    # 3. a scale of amax / 256 (another format's maximum)
    with monkeypatch.context() as m:
        m.setattr(f8, "E4M3_MAX", 256.0)
        _expect_failure(test_scales_and_round_trip)
    # 4. the head's K scale left out of the logits
    with monkeypatch.context() as m:
        orig_qt = f8.quantize_tensor
        m.setattr(f8, "quantize_tensor", lambda x: (orig_qt(x)[0], np.float32(1.0)))
        _expect_failure(test_fp8_attention_with_power_of_two_scales_is_exact)

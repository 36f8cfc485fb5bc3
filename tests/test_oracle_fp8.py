"""Pins for the oracle's 8-bit formats and per-row power-of-two scaling.

Every finite e4m3 / e5m2 value is built from its bit fields (sign, biased
exponent, mantissa; subnormals at the lowest exponent) and must round to
itself; midpoints between neighbours go to the even code; values beyond the
largest finite value saturate. In range, the rounding agrees with torch's
float8 conversions (a library routine). The row scale is checked against a
brute-force search, and the narrow-E self-conditioning sum against the plain
one where every rounding is exact.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fp8 as F
from oracle import method as M


def _all_finite(fmt):
    """All finite non-negative values of the format, in code order, from the bit fields."""
    eb, mb, bias = (4, 3, 7) if fmt == "e4m3" else (5, 2, 15)
    vals = []
    for ex in range(2 ** eb):
        for m in range(2 ** mb):
            if fmt == "e4m3" and ex == 15 and m == 7:
                continue                          # the single NaN code of e4m3
            if fmt == "e5m2" and ex == 31:
                continue                          # infinities and NaNs
            if ex == 0:
                v = (m / 2 ** mb) * 2.0 ** (1 - bias)
            else:
                v = (1 + m / 2 ** mb) * 2.0 ** (ex - bias)
            vals.append(v)
    return np.array(vals)


@pytest.mark.parametrize("fmt,vmax,tiny", [("e4m3", 448.0, 2.0 ** -9), ("e5m2", 57344.0, 2.0 ** -16)])
def test_every_value_rounds_to_itself_and_midpoints_to_even(fmt, vmax, tiny):
    v = _all_finite(fmt)
    assert v.max() == vmax and v[1] == tiny
    np.testing.assert_array_equal(F.fp8_round(v, fmt), v)
    np.testing.assert_array_equal(F.fp8_round(-v, fmt), -v)
    mid = 0.5 * (v[:-1] + v[1:])
    got = F.fp8_round(mid, fmt)
    idx = np.arange(len(v) - 1)
    want = np.where(idx % 2 == 0, v[:-1], v[1:])   # the neighbour with the even code
    np.testing.assert_array_equal(got, want)
    # just off the midpoint: nearest
    np.testing.assert_array_equal(F.fp8_round(mid * (1 - 1e-9), fmt), v[:-1])
    np.testing.assert_array_equal(F.fp8_round(mid * (1 + 1e-9), fmt), v[1:])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_saturation(fmt):
    vmax = F.FORMATS[fmt][2]
    np.testing.assert_array_equal(F.fp8_round([vmax * 1.1, -vmax * 4, 1e30], fmt),
                                  [vmax, -vmax, vmax])


@pytest.mark.parametrize("fmt,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_agrees_with_library_conversion_in_range(fmt, tdt):
    g = np.random.default_rng(0)
    vmax = F.FORMATS[fmt][2]
    x = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-6, 4, 20000),
                        g.uniform(-vmax, vmax, 2000)]).astype(np.float32)
    x = x[np.abs(x) <= vmax]                  # beyond it the library gives NaN, the device saturates
    want = torch.from_numpy(x).to(tdt).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(F.fp8_round(x.astype(np.float64), fmt), want)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_row_scale_exponent_is_the_smallest_that_fits(fmt):
    vmax = F.FORMATS[fmt][2]
    g = np.random.default_rng(1)
    amax = np.concatenate([g.uniform(0, 1, 500) * 10.0 ** g.integers(-8, 8, 500),
                           [vmax, vmax * (1 + 2 ** -20), vmax / 2, 1.0, 0.0]])
    e = F.row_scale_exponent(amax, fmt)
    for a, ei in zip(amax, e):
        if a == 0:
            assert ei == 0
            continue
        assert a * 2.0 ** -ei <= vmax
        assert a * 2.0 ** -(ei - 1) > vmax


def test_quantize_rows_round_trip():
    g = np.random.default_rng(2)
    X = g.standard_normal((64, 256)) * np.exp(g.uniform(-8, 8, (64, 1)))
    q, e = F.quantize_rows(X, "e4m3")
    assert np.abs(q).max() <= 448.0
    assert np.all(np.abs(q).max(axis=1) >= 224.0)   # the scale uses the top binade
    Xd = F.dequantize_rows(q, e)
    # within half a spacing (3 mantissa bits: 2^-4 relative) or the subnormal step
    tol = np.maximum(np.abs(X) * 2.0 ** -4, np.ldexp(1.0, e[:, None] - 10))
    assert np.all(np.abs(Xd - X) <= tol)


def test_narrow_sc_equals_plain_sc_when_rounding_is_exact():
    """E codes that are small integers with exponent 0 and logits whose
    probabilities against the reference are powers of two: every rounding is
    exact, so the narrow-E sum is the plain p.E."""
    g = np.random.default_rng(3)
    V, d = 64, 16
    codes = g.integers(-8, 9, (V, d)).astype(np.float64)
    exps = np.zeros(V, dtype=np.int64)
    z = np.log(2.0) * -g.integers(0, 12, (2, V)).astype(np.float64)
    m_ref = np.zeros(2)
    sc = F.sc_from_quantized_p(z, m_ref, codes, exps, 0)
    p = np.exp(z) / np.exp(z).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(sc, p @ codes, rtol=1e-14, atol=1e-14)
    # the step exponent u only moves the scaling: the same result for u = -3
    np.testing.assert_allclose(F.sc_from_quantized_p(z, m_ref, codes, exps, -3), sc, rtol=1e-14)


def test_step_exponent_keeps_the_largest_probability_in_range():
    """u = max row exponent - 10: a probability of e^REDO_GAP times 2^(e - u) fits e5m2."""
    e = np.array([-14, -12, -13, -12])
    u = F.step_exponent(e)
    assert u == -22
    assert math.exp(F.REDO_GAP) * 2.0 ** (e.max() - u) <= F.FORMATS["e5m2"][2]


def test_narrow_attention_with_exact_roundings_is_the_plain_attention():
    """E rows exactly representable (codes, exponent 0), h rows exactly
    representable after their power-of-two scaling, and logits whose
    probabilities against the reference are powers of two: entropy, argmax and
    sc equal the plain attention's."""
    g = np.random.default_rng(4)
    V, d = 128, 8
    E = g.integers(-6, 7, (V, d)).astype(np.float64)
    E[:, 0] = 8.0                                   # every row's largest magnitude: exponent 0 below
    nE = F.NarrowE(E / 64.0)
    assert np.array_equal(nE.E_deq, E / 64.0)
    h = np.zeros((3, d))
    h[:, 0] = [1.0, 0.5, 2.0]
    att, m_ref = F.narrow_attention(nE, h, np.log(2.0) * 64.0 / 8.0, canvas=[0, 1, 2], prev=[0, 1, 2])
    plain = M.vocab_attention(h, E / 64.0, np.log(2.0) * 64.0 / 8.0)
    np.testing.assert_allclose(att.H, plain.H, atol=1e-12)
    assert np.array_equal(att.argmax, plain.argmax)
    np.testing.assert_allclose(att.sc, plain.sc, rtol=1e-12, atol=1e-12)


def test_reference_is_raised_only_when_it_lags_too_far():
    g = np.random.default_rng(5)
    V, d = 256, 32
    nE = F.NarrowE(g.standard_normal((V, d)) / np.sqrt(d))
    h = 3.0 * nE.E_deq[[7, 9]].astype(np.float64)     # row 0 leans on token 7, row 1 on 9
    scale = 1.0
    # canvas token = the leaned-on token: the reference is the row maximum, kept
    _, m1 = F.narrow_attention(nE, h, scale, canvas=[7, 9], prev=[7, 9])
    att, _ = F.narrow_attention(nE, h, scale, canvas=[7, 9], prev=[7, 9], m_ref=m1)
    assert np.all(att.zmax - m1 <= F.REDO_GAP)
    # a far-off canvas token with a large scale: the lag exceeds the gap, so the
    # reference becomes the exact maximum
    _, m2 = F.narrow_attention(nE, h, 40.0, canvas=[3, 4], prev=[3, 4])
    att2, _ = F.narrow_attention(nE, h, 40.0, canvas=[3, 4], prev=[3, 4], m_ref=m2)
    np.testing.assert_allclose(m2, att2.zmax, rtol=0, atol=0)


def test_narrow_sc_is_close_to_the_plain_sc_of_the_dequantised_values():
    """The e5m2 rounding of the probabilities (2 mantissa bits, errors of both
    signs) leaves sc within a few percent of p.E_deq for a random problem."""
    g = np.random.default_rng(6)
    V, d = 4096, 64
    nE = F.NarrowE(g.standard_normal((V, d)) / np.sqrt(d))
    h = g.standard_normal((4, d))
    att, _ = F.narrow_attention(nE, h, 2.0, canvas=[0, 1, 2, 3], prev=[0, 1, 2, 3])
    hq, he = F.quantize_rows(h, "e4m3")
    plain = M.vocab_attention(F.dequantize_rows(hq, he), nE.E_deq, 2.0)
    rel = np.linalg.norm(att.sc - plain.sc, axis=1) / np.linalg.norm(plain.sc, axis=1)
    assert rel.max() < 0.05
    np.testing.assert_allclose(att.H, plain.H)


def test_block_scale_is_shared_by_the_block_and_fits_its_largest_row():
    """One exponent per block of GROUP vocabulary rows: the smallest that brings
    the block's largest magnitude within e4m3's range; a row a thousand times
    smaller than its block's largest keeps e4m3's relative precision as a
    vector (its entries lie within e4m3's normal range, 2^-6 .. 448)."""
    g = np.random.default_rng(7)
    V, d = 2 * F.GROUP, 16
    E = g.standard_normal((V, d)) * np.repeat([0.01, 3.0], F.GROUP)[:, None]
    E[5] *= 1e-3                                    # a much smaller row in block 0
    nE = F.NarrowE(E)
    for b in range(2):
        blk = slice(b * F.GROUP, (b + 1) * F.GROUP)
        assert len(set(nE.exps[blk].tolist())) == 1
        assert nE.exps[blk][0] == F.row_scale_exponent(np.abs(E[blk]).max(), "e4m3")
    rel = np.linalg.norm(nE.E_deq[5] - E[5]) / np.linalg.norm(E[5])
    assert rel <= 2.0 ** -4

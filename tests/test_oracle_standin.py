"""Pins for the oracle's temperature schedule, bf16 rounding and stand-in hidden state."""
import math

import numpy as np
import pytest
import torch

import synthetic
from oracle import method as M


@pytest.mark.parametrize("S,T0,T1", [(8, 1.0, 0.1), (16, 1.5, 0.05), (32, 1.0, 0.1), (2, 2.0, 1.0)])
def test_cosine_schedule_shape(S, T0, T1):
    T = [M.temperature(t, S, T0, T1) for t in range(S)]
    assert T[0] == pytest.approx(T0, abs=1e-15)
    assert T[-1] == pytest.approx(T1, abs=1e-15)
    assert all(a > b for a, b in zip(T, T[1:]))                     # lower at every later step
    for t in range(S):                                              # cosine symmetry
        assert T[t] + T[S - 1 - t] == pytest.approx(T0 + T1, abs=1e-14)
    if S % 2 == 1:
        assert T[S // 2] == pytest.approx((T0 + T1) / 2, abs=1e-15)
    # flat at both ends: the first and last differences are the smallest
    diffs = [a - b for a, b in zip(T, T[1:])]
    if S > 3:
        assert diffs[0] < diffs[len(diffs) // 2] and diffs[-1] < diffs[len(diffs) // 2]


def test_single_step_schedule():
    assert M.temperature(0, 1, 1.3, 0.1) == 1.3


def test_bf16_round_against_library_conversion():
    g = np.random.default_rng(0)
    x = np.concatenate([g.standard_normal(100000) * 0.05, g.standard_normal(1000) * 1e3,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, 2 ** -130])])
    x32 = x.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(M.bf16_round(x32.astype(np.float64)), want)


def test_bf16_ties_to_even():
    assert M.bf16_round(np.array([1.0 + 2 ** -8]))[0] == 1.0
    assert M.bf16_round(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6


def _w(**kw):
    return synthetic.TINY.replace(**kw)


def test_standin_without_noise_is_the_linear_combination():
    w = _w(noise_var_d=0.0, coef_target=6.0, coef_canvas=2.0)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    tgt, can = M.init_block(w, 0)
    h = M.standin_hidden(w, E, tgt, can, np.zeros((w.C, w.d)), 0, 0)
    np.testing.assert_allclose(h, 6.0 * E[tgt].astype(np.float64) + 2.0 * E[can].astype(np.float64),
                               rtol=0, atol=1e-15)


def test_standin_noise_statistics_and_sc_term():
    w = _w(C=64, d=256, V=512)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    tgt, can = M.init_block(w, 0)
    base = w.coef_target * E[tgt].astype(np.float64) + w.coef_canvas * E[can].astype(np.float64)
    h0 = M.standin_hidden(w, E, tgt, can, np.zeros((w.C, w.d)), 0, 3)
    eps = (h0 - base) * math.sqrt(w.d / w.noise_var_d)
    assert abs(eps.mean()) < 0.02 and abs(eps.var() - 1.0) < 0.03
    sc = np.random.default_rng(1).standard_normal((w.C, w.d))
    h1 = M.standin_hidden(w, E, tgt, can, sc, 0, 3)
    np.testing.assert_allclose(h1 - h0, sc, atol=1e-12)
    # the noise is keyed on the step: another step draws other noise
    h2 = M.standin_hidden(w, E, tgt, can, np.zeros((w.C, w.d)), 0, 4)
    assert not np.allclose(h2, h0)


def test_standin_bf16_rounds_hidden_state():
    w = _w(dtype="bf16")
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    tgt, can = M.init_block(w, 0)
    h = M.standin_hidden(w, E, tgt, can, np.zeros((w.C, w.d)), 0, 0)
    np.testing.assert_array_equal(M.bf16_round(h), h)


def test_init_tokens_in_range_and_distinct_streams():
    w = _w(C=256, V=1024)
    tgt, can = M.init_block(w, 0)
    assert tgt.min() >= 0 and tgt.max() < w.V and can.min() >= 0 and can.max() < w.V
    assert np.mean(tgt == can) < 0.05

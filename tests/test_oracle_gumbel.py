"""Pins of the oracle's multinomial token draw (Gumbel-max).

A Visual Guide to DiffusionGemma, 3.2 names drawing each position's token from
its predicted distribution. The oracle draws argmax_v (z_v + G_v) with keyed
standard Gumbel variates G_v. These tests pin it to facts that do not come from
its own code: the Gumbel distribution's closed-form CDF, mean (the
Euler-Mascheroni constant) and variance (pi^2/6); the Gumbel-max identity
(the draw follows softmax(z)), checked by chi-square against softmax computed
here; and the limits of a one-hot and a flat distribution.
"""
import math

import numpy as np
import pytest

from oracle import method as M
from oracle import rng

import synthetic

EULER_GAMMA = 0.5772156649015329

# Chi-square critical values at p = 0.001 (standard tables).
CHI2_999 = {3: 16.266, 7: 24.322}


def test_uniform_cut_is_open_and_exact_in_fp32():
    k = rng.key(11, 2, rng.TAG_GUMBEL + 3, np.arange(100000, dtype=np.uint64))
    W = rng.gumbel_uniform(k)
    assert np.all(W > 0.0) and np.all(W < 1.0)
    assert np.array_equal(W.astype(np.float32).astype(np.float64), W)
    ends = rng.gumbel_uniform(np.array([0, (1 << 64) - 1], dtype=np.uint64))
    assert ends[0] == 2.0 ** -24 and ends[1] == 1.0 - 2.0 ** -24


def test_gumbel_cdf_mean_variance():
    n = 200000
    g = rng.gumbel(5, 0, rng.TAG_GUMBEL, np.arange(n, dtype=np.uint64))
    assert abs(g.mean() - EULER_GAMMA) < 0.012
    assert abs(g.var() - math.pi ** 2 / 6) < 0.04
    # Kolmogorov-Smirnov distance to P(G <= x) = exp(-exp(-x)).
    xs = np.sort(g)
    F = np.exp(-np.exp(-xs))
    ecdf_hi = np.arange(1, n + 1) / n
    ecdf_lo = np.arange(0, n) / n
    ks = max(np.max(ecdf_hi - F), np.max(F - ecdf_lo))
    assert ks < 1.95 / math.sqrt(n)        # p = 0.001


def _softmax(z):
    e = np.exp(z - z.max())
    return e / e.sum()


@pytest.mark.parametrize("z", [[0.0, 1.0, 2.0, -1.0], [3.0, 2.9, -4.0, 0.5]])
def test_draw_follows_softmax(z):
    rows = 40000
    z = np.asarray(z)
    Z = np.tile(z, (rows, 1))
    tok, _ = M.gumbel_max(Z, seed=3, block=1, t=4)
    counts = np.bincount(tok, minlength=z.size)
    expect = rows * _softmax(z)
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < CHI2_999[z.size - 1]


def test_flat_distribution_is_uniform():
    rows, V = 40000, 8
    tok, _ = M.gumbel_max(np.zeros((rows, V)), seed=9, block=0, t=0)
    counts = np.bincount(tok, minlength=V)
    expect = rows / V
    assert float(((counts - expect) ** 2 / expect).sum()) < CHI2_999[V - 1]


def test_one_hot_limit_draws_the_argmax():
    rows, V = 500, 64
    Z = np.zeros((rows, V))
    hot = (np.arange(rows) * 7) % V
    Z[np.arange(rows), hot] = 1000.0
    tok, gap = M.gumbel_max(Z, seed=1, block=0, t=0)
    assert np.array_equal(tok, hot)
    assert np.all(gap > 900.0)


def test_draw_depends_on_every_key_field():
    z = np.zeros((64, 512))
    base, _ = M.gumbel_max(z, 1, 2, 3)
    again, _ = M.gumbel_max(z, 1, 2, 3)
    assert np.array_equal(base, again)
    for other in [(2, 2, 3), (1, 3, 3), (1, 2, 4)]:
        tok, _ = M.gumbel_max(z, *other)
        assert np.mean(tok == base) < 0.05
    shifted, _ = M.gumbel_max(z, 1, 2, 3, rows0=1)
    assert np.array_equal(shifted[:-1], base[1:])


def test_step_accepts_the_draw_and_keeps_the_distribution():
    w = synthetic.TINY.replace(token_rule=1, coef_target=1.0, coef_canvas=0.5, logit_scale=2.0,
                               fixed_steps=1)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    st = M.begin_block(w, 0)
    st_ref = M.begin_block(w.replace(token_rule=0), 0)
    differs = 0
    for _ in range(3):
        h = M.standin_hidden(w, E, st.target, st.canvas, st.sc, st.block, st.t)
        rec = M.step(w, E, st, h=h)
        ref = M.step(w.replace(token_rule=0), E, st_ref, h=h)
        # same distribution, entropy, argmax and sc; only the token choice differs
        assert np.array_equal(rec.att.argmax, ref.att.argmax)
        assert np.allclose(rec.att.H, ref.att.H) and np.allclose(rec.att.sc, ref.att.sc)
        acc = rec.acc.accepted
        assert np.array_equal(rec.canvas_out[acc], rec.att.sampled[acc])
        assert np.array_equal(rec.canvas_out[~acc], rec.noise[~acc])
        differs += int(np.sum(rec.att.sampled != rec.att.argmax))
        st_ref.canvas, st_ref.sc = st.canvas.copy(), st.sc.copy()
    assert differs > 0        # a soft distribution does not always draw its mode

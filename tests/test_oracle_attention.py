"""Pins for the oracle's vocabulary softmax, entropy, argmax and self-conditioning vector.

Brute force in long double with the log-partition form of the entropy (the
oracle uses -sum p log p), closed forms (uniform logits, exact two-way tie,
one-hot), a library softmax, and the monotonicity of entropy in the inverse
temperature.
"""
import math

import numpy as np
import pytest
import torch

from oracle import method as M


def _brute(h, E, scale):
    """Unshifted softmax, entropy log Z - E_p[z], p.E and argmax, all in long double loops."""
    h = np.asarray(h, dtype=np.longdouble)
    E = np.asarray(E, dtype=np.longdouble)
    rows, V = h.shape[0], E.shape[0]
    out = []
    for i in range(rows):
        z = [scale * sum(h[i, k] * E[v, k] for k in range(E.shape[1])) for v in range(V)]
        ez = [np.exp(np.longdouble(x)) for x in z]
        Z = sum(ez)
        p = [x / Z for x in ez]
        H = np.log(Z) - sum(pv * zv for pv, zv in zip(p, z))
        sc = [sum(p[v] * E[v, k] for v in range(V)) for k in range(E.shape[1])]
        best = 0
        for v in range(1, V):
            if np.float32(z[v]) > np.float32(z[best]):
                best = v
        out.append((float(H), np.array(sc, dtype=np.float64), best))
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_long_double_brute_force(seed):
    g = np.random.default_rng(seed)
    rows, V, d = 3, 11, 5
    h = g.standard_normal((rows, d))
    E = g.standard_normal((V, d)).astype(np.float32)
    scale = 1.7
    att = M.vocab_attention(h, E, scale)
    for i, (H, sc, best) in enumerate(_brute(h, E, scale)):
        assert abs(att.H[i] - H) < 1e-12
        np.testing.assert_allclose(att.sc[i], sc, rtol=1e-12, atol=1e-14)
        assert att.argmax[i] == best


def test_matches_library_softmax():
    g = np.random.default_rng(5)
    h = g.standard_normal((4, 16))
    E = g.standard_normal((64, 16)).astype(np.float32)
    att = M.vocab_attention(h, E, 0.8)
    z = torch.from_numpy(0.8 * (h @ E.astype(np.float64).T))
    p = torch.softmax(z, dim=1)
    H = -(p * torch.log_softmax(z, dim=1)).sum(1)
    np.testing.assert_allclose(att.H, H.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(att.sc, (p @ torch.from_numpy(E.astype(np.float64))).numpy(),
                               rtol=1e-12, atol=1e-14)


def test_uniform_logits():
    """h = 0: every token equally likely, H = ln V, sc = mean embedding, argmax = 0."""
    g = np.random.default_rng(1)
    V, d = 64, 8
    E = g.standard_normal((V, d)).astype(np.float32)
    att = M.vocab_attention(np.zeros((2, d)), E, 3.0)
    np.testing.assert_allclose(att.H, math.log(V), rtol=0, atol=1e-12)
    np.testing.assert_allclose(att.sc, np.tile(E.astype(np.float64).mean(0), (2, 1)), atol=1e-14)
    assert list(att.argmax) == [0, 0]


def test_exact_two_way_tie():
    """Two identical best rows: H -> ln 2, sc -> their embedding, argmax -> the lower index."""
    u = np.array([0.6, -0.8], dtype=np.float32)
    E = np.stack([-u, u, u, -u]).astype(np.float32)
    att = M.vocab_attention(np.array([[0.6, -0.8]]), E, 200.0)
    assert abs(att.H[0] - math.log(2.0)) < 1e-12
    np.testing.assert_allclose(att.sc[0], u.astype(np.float64), atol=1e-12)
    assert att.argmax[0] == 1
    assert att.margin[0] == 0.0


def test_one_hot_limit():
    g = np.random.default_rng(2)
    V, d = 32, 16
    E = g.standard_normal((V, d)).astype(np.float32)
    h = E[[7, 20]].astype(np.float64)
    att = M.vocab_attention(h, E, 400.0)
    assert list(att.argmax) == [7, 20]
    assert np.all(att.H < 1e-9)
    np.testing.assert_allclose(att.sc, E[[7, 20]].astype(np.float64), atol=1e-9)


def test_entropy_decreases_as_temperature_drops():
    g = np.random.default_rng(3)
    h = g.standard_normal((5, 8))
    E = g.standard_normal((40, 8)).astype(np.float32)
    prev = None
    for scale in [0.05, 0.2, 0.5, 1.0, 2.0, 5.0, 20.0]:
        H = M.vocab_attention(h, E, scale).H
        assert np.all(H >= 0) and np.all(H <= math.log(40) + 1e-12)
        if prev is not None:
            assert np.all(H <= prev + 1e-12)
        prev = H


def test_logits_orientation():
    """z[i, v] = <h_i, E_v>: rows index positions, columns index vocabulary."""
    h = np.array([[1.0, 0.0, 0.0], [0.0, 0.0, 2.0]])
    E = np.array([[1, 2, 3], [4, 5, 6], [7, 8, 9], [1, 1, 1]], dtype=np.float32)
    z = M.logits(h, E, 0.5)
    assert z.shape == (2, 4)
    np.testing.assert_array_equal(z, [[0.5, 2.0, 3.5, 0.5], [3.0, 6.0, 9.0, 1.0]])

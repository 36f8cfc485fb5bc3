"""Pins for the oracle's self-conditioning feed-forward network.

A Visual Guide to DiffusionGemma, 5.1: the probability-weighted embeddings are
passed through a small feed-forward network and added to the next step's token
embeddings. Pinned by: the GELU's defining values (zero, odd part, the large-|a|
limits, the known value at 1), identity weights (the network reduces to the
elementwise GELU), brute force in long double over explicit loops, linearity in
the second layer, and the bias terms.
"""
import math

import numpy as np
import pytest

from oracle import method as M


def test_gelu_tanh_against_the_exact_gelu():
    """The tanh form approximates GELU(a) = a Phi(a) (Phi from the library's erf)
    to a few 1e-4 everywhere; its odd part is a/2 exactly; it tends to a and 0."""
    a = np.linspace(-6.0, 6.0, 2401)
    exact = a * 0.5 * (1.0 + np.array([math.erf(x / math.sqrt(2.0)) for x in a]))
    g = M.gelu_tanh(a)
    assert np.abs(g - exact).max() < 5e-4
    assert np.abs(g - exact).max() > 1e-5          # it is the approximation, not erf itself
    np.testing.assert_allclose(g - M.gelu_tanh(-a), a, rtol=0, atol=1e-14)
    assert M.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert M.gelu_tanh(np.array([10.0]))[0] == pytest.approx(10.0, abs=1e-12)
    assert abs(M.gelu_tanh(np.array([-10.0]))[0]) < 1e-12


def _brute(sc, W1, b1, W2, b2):
    C, d = sc.shape
    dff = W1.shape[0]
    L = np.longdouble
    k = L(math.sqrt(2.0 / math.pi))
    out = np.zeros((C, d), dtype=np.float64)
    for i in range(C):
        x = [L(M.bf16_round(np.array([sc[i, j]]))[0]) for j in range(d)]
        g = []
        for u in range(dff):
            a = sum(L(W1[u, j]) * x[j] for j in range(d)) + L(b1[u])
            v = L(0.5) * a * (L(1) + np.tanh(k * (a + L(0.044715) * a * a * a)))
            g.append(L(M.bf16_round(np.array([float(v)]))[0]))
        for j in range(d):
            out[i, j] = float(sum(L(W2[j, u]) * g[u] for u in range(dff)) + L(b2[j]))
    return out


@pytest.mark.parametrize("seed", [0, 1])
def test_matches_long_double_brute_force(seed):
    g = np.random.default_rng(seed)
    C, d, dff = 3, 8, 12
    sc = g.standard_normal((C, d))
    W1 = g.standard_normal((dff, d)) / np.sqrt(d)
    b1 = g.standard_normal(dff) * 0.1
    W2 = g.standard_normal((d, dff)) / np.sqrt(dff)
    b2 = g.standard_normal(d) * 0.1
    np.testing.assert_allclose(M.self_condition_ffnn(sc, W1, b1, W2, b2),
                               _brute(sc, W1, b1, W2, b2), rtol=0, atol=1e-12)


def test_identity_weights_give_the_elementwise_gelu():
    d = 16
    sc = np.linspace(-3.0, 3.0, 2 * d).reshape(2, d)
    eye = np.eye(d)
    y = M.self_condition_ffnn(sc, eye, np.zeros(d), eye, np.zeros(d))
    want = M.bf16_round(M.gelu_tanh(M.bf16_round(sc)))
    np.testing.assert_array_equal(y, want)


def test_orientation_of_the_weights():
    """W1 maps d inputs to d_ff units (rows are units): a one-hot input picks a column."""
    d, dff = 4, 6
    W1 = np.arange(dff * d, dtype=np.float64).reshape(dff, d) / 64.0
    W2 = np.zeros((d, dff))
    W2[2, 5] = 1.0
    sc = np.zeros((1, d))
    sc[0, 1] = 1.0
    y = M.self_condition_ffnn(sc, W1, np.zeros(dff), W2, np.zeros(d))
    assert y[0, 2] == pytest.approx(float(M.bf16_round(M.gelu_tanh(np.array([W1[5, 1]])))[0]))
    assert y[0, 0] == y[0, 1] == y[0, 3] == 0.0


def test_second_layer_is_linear_and_biases_add():
    g = np.random.default_rng(3)
    C, d, dff = 2, 8, 16
    sc = g.standard_normal((C, d))
    W1 = g.standard_normal((dff, d))
    b1 = g.standard_normal(dff)
    W2 = g.standard_normal((d, dff))
    b2 = g.standard_normal(d)
    y = M.self_condition_ffnn(sc, W1, b1, W2, b2)
    y2 = M.self_condition_ffnn(sc, W1, b1, 2.0 * W2, 2.0 * b2)
    np.testing.assert_allclose(y2, 2.0 * y, rtol=1e-14, atol=1e-14)
    y0 = M.self_condition_ffnn(sc, W1, b1, W2, np.zeros(d))
    np.testing.assert_allclose(y - y0, np.broadcast_to(b2, y.shape), rtol=0, atol=1e-12)


def test_added_to_bf16_embeddings_rounds_the_sum():
    emb = np.array([[1.0, -2.0]])
    y = np.array([[2.0 ** -9, 0.25]])
    out = M.add_to_embeddings(emb, y, "bf16")
    assert out[0, 0] == 1.0                 # 1 + 2^-9 rounds back to 1 in bf16 (8 bits)
    assert out[0, 1] == -1.75
    np.testing.assert_array_equal(M.add_to_embeddings(emb, y, "f32"), emb + y)

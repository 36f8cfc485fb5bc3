"""Pins for the oracle's entropy-bounded sampler, re-noising and adaptive stop."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import synthetic
from oracle import method as M
from oracle import rng

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLDEN, "acceptance_example.json")) as f:
        return json.load(f)


def test_hand_worked_acceptance_cumsum():
    g = _golden()
    acc = M.entropy_bounded_accept(np.array(g["H"], np.float32), g["tau"], rule=0)
    assert list(acc.order) == g["order"]
    assert list(acc.prefix) == g["prefix"]
    assert sorted(np.flatnonzero(acc.accepted)) == sorted(g["cumsum_accepted"])
    assert acc.k == len(g["cumsum_accepted"])


def test_hand_worked_acceptance_minus_max():
    g = _golden()
    acc = M.entropy_bounded_accept(np.array(g["H"], np.float32), g["tau"], rule=1)
    assert sorted(np.flatnonzero(acc.accepted)) == sorted(g["minus_max_accepted"])
    assert acc.k == len(g["minus_max_accepted"])


@pytest.mark.parametrize("rule,k_expected", [(0, 0), (1, 1)])
def test_all_above_tau(rule, k_expected):
    acc = M.entropy_bounded_accept(np.full(8, 3.0, np.float32), 1.0, rule)
    assert acc.k == k_expected


@pytest.mark.parametrize("rule", [0, 1])
def test_all_zero_entropy_accepts_everything(rule):
    acc = M.entropy_bounded_accept(np.zeros(16, np.float32), 0.0, rule)
    assert acc.k == 16 and acc.accepted.all()


def test_sort_is_stable_on_ties():
    H = np.array([0.5, 0.25, 0.5, 0.25, 0.0], np.float32)
    acc = M.entropy_bounded_accept(H, 10.0, 0)
    assert list(acc.order) == [4, 1, 3, 0, 2]


@pytest.mark.parametrize("seed", range(6))
def test_acceptance_matches_exact_brute_force(seed):
    """Dyadic entropies (exact in fp32): the largest accepted prefix, found with exact fractions."""
    g = np.random.default_rng(seed)
    C = 12
    H = (g.integers(0, 64, C) / 16.0).astype(np.float32)
    tau = float(g.integers(0, 80) / 8.0)
    for rule in (0, 1):
        acc = M.entropy_bounded_accept(H, tau, rule)
        order = sorted(range(C), key=lambda i: (Fraction(float(H[i])), i))
        best = 0
        for k in range(1, C + 1):
            s = sum(Fraction(float(H[i])) for i in order[:k])
            if rule == 1:
                s -= max(Fraction(float(H[i])) for i in order[:k])
            if s <= Fraction(tau):
                best = k
            else:
                break
        assert acc.k == best
        assert set(np.flatnonzero(acc.accepted)) == set(order[:best])


def _tiny(**kw):
    return synthetic.TINY.replace(**kw)


def test_step_invariants_on_stress_data():
    """Accepted -> argmax; rejected -> hashed noise token; accepted entropy within tau; k maximal."""
    w = _tiny(coef_target=0.5, coef_canvas=0.5, logit_scale=1.0, tau=2.0, max_steps=5)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    st = M.begin_block(w, 0)
    saw_partial = False
    while not st.done:
        rec = M.step(w, E, st)
        acc = rec.acc
        H32 = rec.att.H.astype(np.float32)
        noise = rng.tokens(w.seed, 0, rec.t, np.arange(w.C, dtype=np.uint64), w.V)
        assert np.array_equal(rec.canvas_out[acc.accepted], rec.att.argmax[acc.accepted])
        assert np.array_equal(rec.canvas_out[~acc.accepted], noise[~acc.accepted])
        assert float(np.sum(H32[acc.accepted], dtype=np.float64)) <= w.tau + 1e-5
        assert set(np.flatnonzero(acc.accepted)) == set(acc.order[:acc.k])
        if acc.k < w.C:
            assert acc.prefix[acc.k] > np.float32(w.tau)
        saw_partial |= 0 < acc.k < w.C
    assert saw_partial


class _Scripted:
    """Replaces vocab_attention with scripted (argmax, H) per call."""

    def __init__(self, C, d, script):
        self.C, self.d, self.script, self.calls = C, d, script, 0

    def __call__(self, h, E, scale):
        amax, H = self.script(self.calls)
        self.calls += 1
        return M.Attention(argmax=np.asarray(amax, np.int64), H=np.asarray(H, np.float64),
                           sc=np.zeros((self.C, self.d)), zmax=np.zeros(self.C),
                           margin=np.full(self.C, 10.0))


def _run(monkeypatch, w, script):
    monkeypatch.setattr(M, "vocab_attention", _Scripted(w.C, w.d, script))
    E = np.zeros((w.V, w.d), np.float32)
    st = M.begin_block(w, 0)
    recs = []
    while not st.done:
        recs.append(M.step(w, E, st))
    return st, recs


def test_stop_after_n_unchanged_canvases(monkeypatch):
    w = _tiny(max_steps=20, tau=1e9)
    amax = np.arange(w.C)
    st, recs = _run(monkeypatch, w, lambda t: (amax, np.full(w.C, 1.0)))
    # step 0 changes the random canvas to amax; steps 1, 2, 3 leave it unchanged
    assert [r.unchanged for r in recs] == [0, 1, 2, 3]
    assert st.steps_done == 4


def test_stop_on_confidence_needs_every_position(monkeypatch):
    w = _tiny(max_steps=20, tau=0.0, stop_unchanged=100)

    def script(t):
        H = np.full(w.C, 0.001)
        if t < 2:
            H[5] = 0.005          # not strictly below the threshold
        return np.arange(w.C), H
    st, recs = _run(monkeypatch, w, script)
    assert [r.all_confident for r in recs] == [False, False, True]
    assert st.steps_done == 3


def test_stop_at_step_budget(monkeypatch):
    w = _tiny(max_steps=6, tau=0.0)
    st, _ = _run(monkeypatch, w, lambda t: (np.arange(w.C), np.full(w.C, 2.0)))
    assert st.steps_done == 6


def test_fixed_steps_ignores_adaptive_stop(monkeypatch):
    w = _tiny(max_steps=7, tau=1e9, fixed_steps=1)
    st, _ = _run(monkeypatch, w, lambda t: (np.arange(w.C), np.zeros(w.C)))
    assert st.steps_done == 7


def test_argmax_stability_rule(monkeypatch):
    """stop_rule 1 counts unchanged argmax predictions, even while the canvas keeps changing."""
    w = _tiny(max_steps=20, tau=0.0, stop_rule=1)     # tau 0 with H > 0: all rejected
    st, recs = _run(monkeypatch, w, lambda t: (np.arange(w.C), np.full(w.C, 1.0)))
    assert [r.unchanged for r in recs] == [0, 1, 2, 3]
    assert st.steps_done == 4


def test_blocks_are_independent_and_reset():
    w = _tiny(blocks=3)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    out, steps = M.generate(w, E)
    for b in range(3):
        tok, n, _ = M.denoise_block(w, E, b)
        assert np.array_equal(out[b * w.C:(b + 1) * w.C], tok)
        assert steps[b] == n
    t0, c0 = M.init_block(w, 0)
    t1, c1 = M.init_block(w, 1)
    assert not np.array_equal(t0, t1) and not np.array_equal(c0, c1)

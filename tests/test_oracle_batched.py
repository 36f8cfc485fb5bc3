"""Pins of the oracle's batched canvases (independent canvases sharing a step).

Batched canvases (B users x C positions; A Visual Guide to DiffusionGemma, 5.2
multi-canvas sampling): the rows of the vocabulary attention are independent,
so B canvases can share one step, while the sampler and the stop test act on
each canvas alone. Pinned here: a
hand-worked two-canvas acceptance example (exact in binary) that a sort across
canvases would get wrong, the reduction to the single-canvas sampler, the
independence of one canvas's decisions from another's hidden state, and the
freezing of stopped canvases.
"""
import numpy as np

from oracle import method as M

import synthetic


def test_two_canvas_example():
    # canvas 0: sorted (1, 3, 0, 2), running sums 0.0625, 0.125, 0.375, 1.25
    # canvas 1: sorted (7, 5, 6, 4), running sums 0.125, 0.5, 1.0, 3.0
    H = np.array([0.25, 0.0625, 0.875, 0.0625, 2.0, 0.375, 0.5, 0.125], dtype=np.float32)
    acc, order, prefix, k = M.accept_canvases(H, 1.0, 0, 2)
    assert list(order) == [1, 3, 0, 2, 7, 5, 6, 4]
    assert list(prefix) == [0.0625, 0.125, 0.375, 1.25, 0.125, 0.5, 1.0, 3.0]
    assert list(np.flatnonzero(acc)) == [0, 1, 3, 5, 6, 7]
    assert list(k) == [3, 3]
    # one canvas over all eight positions decides differently
    single = M.entropy_bounded_accept(H, 1.0, 0)
    assert not np.array_equal(single.accepted, acc)
    # the minus-max rule compares the sum of the entries before each one
    acc1, _, _, k1 = M.accept_canvases(H, 1.0, 1, 2)
    assert list(k1) == [4, 4] and acc1.all()   # sums before each entry stay <= 1.0


def test_frozen_canvas_accepts_nothing():
    H = np.array([0.25, 0.0625, 0.875, 0.0625, 2.0, 0.375, 0.5, 0.125], dtype=np.float32)
    acc, order, prefix, k = M.accept_canvases(H, 1.0, 0, 2, frozen=[True, False])
    assert not acc[:4].any() and list(order[:4]) == [0, 1, 2, 3] and k[0] == 0
    assert list(np.flatnonzero(acc)) == [5, 6, 7]


def test_one_canvas_is_the_single_canvas_sampler():
    rng = np.random.default_rng(3)
    H = rng.exponential(0.5, size=64).astype(np.float32)
    acc, order, prefix, k = M.accept_canvases(H, 9.0, 0, 1)
    ref = M.entropy_bounded_accept(H, 9.0, 0)
    assert np.array_equal(acc, ref.accepted) and np.array_equal(order, ref.order)
    assert np.array_equal(prefix, ref.prefix) and k[0] == ref.k


def _tiny_batched(B):
    return synthetic.TINY.replace(C=16, canvases=B, tau=0.5 * (16 // B) * np.log(2),
                                  coef_target=0.5, coef_canvas=0.5, logit_scale=1.5)


def test_canvas_decisions_ignore_other_canvases():
    w = _tiny_batched(2)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    st_a = M.begin_block(w, 0)
    st_b = M.begin_block(w, 0)
    h = M.standin_hidden(w, E, st_a.target, st_a.canvas, st_a.sc, 0, 0)
    h2 = h.copy()
    tok = (np.arange(8) * 37 + 5) % w.V
    h2[8:] = 30.0 * E[tok]                   # canvas 1 becomes confident about tok
    ra = M.step(w, E, st_a, h=h)
    rb = M.step(w, E, st_b, h=h2)
    assert np.array_equal(ra.canvas_out[:8], rb.canvas_out[:8])
    assert np.array_equal(ra.acc.accepted[:8], rb.acc.accepted[:8])
    assert st_a.unchanged_c[0] == st_b.unchanged_c[0] and st_a.done_c[0] == st_b.done_c[0]
    assert not np.array_equal(ra.canvas_out[8:], rb.canvas_out[8:])
    assert np.array_equal(rb.canvas_out[8:], tok)


def test_block_invariants_and_freezing():
    w = _tiny_batched(4).replace(max_steps=8)
    E = synthetic.embedding_as_f32(synthetic.make_embedding(w))
    st = M.begin_block(w, 0)
    Cc = w.C // 4
    frozen_canvas = {}
    frozen_emit = {}
    froze_early = False
    while not st.done:
        before_done = st.done_c.copy()
        froze_early |= bool(before_done.any())
        # canvas 0 is made confident, so it stops first while the others go on
        h = M.standin_hidden(w, E, st.target, st.canvas, st.sc, st.block, st.t)
        h[:Cc] = 30.0 * E[st.target[:Cc]]
        rec = M.step(w, E, st, h=h)
        for c in range(4):
            seg = slice(c * Cc, (c + 1) * Cc)
            if before_done[c]:
                # a stopped canvas keeps its tokens and its emitted prediction
                assert np.array_equal(rec.canvas_out[seg], frozen_canvas[c])
                assert np.array_equal(st.emit[seg], frozen_emit[c])
                assert not rec.acc.accepted[seg].any()
                continue
            acc = rec.acc.accepted[seg]
            H32 = rec.att.H.astype(np.float32)[seg]
            # accepted = a prefix of the canvas's own order, within tau, maximal
            order = rec.acc.order[seg] - c * Cc
            kk = int(acc.sum())
            assert set(order[:kk]) == set(np.flatnonzero(acc))
            run = np.float32(0.0)
            for j in range(kk):
                run = np.float32(run + H32[order[j]])
            assert run <= np.float32(w.tau)
            if kk < Cc:
                assert np.float32(run + H32[order[kk]]) > np.float32(w.tau)
            assert np.array_equal(rec.canvas_out[seg][acc], rec.att.argmax[seg][acc])
            assert np.array_equal(rec.canvas_out[seg][~acc], rec.noise[seg][~acc])
            if st.done_c[c]:
                frozen_canvas[c] = rec.canvas_out[seg].copy()
                frozen_emit[c] = rec.att.argmax[seg].copy()
                assert np.array_equal(st.emit[seg], rec.att.argmax[seg])
                assert st.steps_c[c] == rec.t + 1
    assert st.steps_done == int(st.steps_c.max())
    assert froze_early and st.steps_c[0] < st.steps_done

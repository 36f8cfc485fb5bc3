"""Comparison of the CUDA path's step outputs with the oracle (test helper).

Tolerances (from the method's stated bar): token ids, accept masks, noise
tokens and step counts bit-exact, except positions that sit on a near-tie --
top-2 logit margin < 1e-3, entropy within 1e-3 of a rank neighbour, or a
running entropy sum within 1e-3 of tau at the acceptance boundary -- which are
counted and must stay <= 0.1% of all compared positions; entropies within 1e-3
absolute; self-conditioning vectors within 2e-2 relative L2 per position.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from oracle import method as M
from oracle import rng

H_ATOL = 1e-3
SC_RTOL = 2e-2
TIE = 1e-3
TIE_BUDGET = 1e-3


@dataclasses.dataclass
class Tally:
    positions: int = 0
    tie_mismatch: int = 0
    worst_H: float = 0.0
    worst_sc: float = 0.0
    steps: int = 0
    draws_off_mode: int = 0     # multinomial draws that differ from the argmax

    def check_budget(self):
        assert self.tie_mismatch <= TIE_BUDGET * max(self.positions, 1), (
            f"{self.tie_mismatch} near-tie mismatches over {self.positions} positions")


def near_tie_flags(att, acc, tau: float, rule: int) -> np.ndarray:
    """Per position: argmax margin, entropy-rank gap or acceptance boundary within TIE."""
    C = att.H.shape[0]
    H = att.H.astype(np.float64)
    flags = att.margin < TIE
    order = acc.order
    Hs = H[order]
    gap = np.full(C, np.inf)
    if C > 1:
        dif = np.abs(np.diff(Hs))
        gap[order[:-1]] = np.minimum(gap[order[:-1]], dif)
        gap[order[1:]] = np.minimum(gap[order[1:]], dif)
    flags |= gap < TIE
    pref = np.cumsum(Hs)
    ref = pref if rule == 0 else np.concatenate([[0.0], pref[:-1]])
    boundary = np.abs(ref - tau) < TIE
    flags[order[boundary]] = True
    return flags


def sc_rel_err(sc_gpu: np.ndarray, sc_ref: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(sc_gpu - sc_ref, axis=1)
    den = np.maximum(np.linalg.norm(sc_ref, axis=1), 1e-30)
    return num / den


def compare_attention(tally: Tally, att, H_gpu, argmax_gpu, sc_gpu, flags, rows=None):
    """H, argmax and sc of the GPU against the oracle's attention for the same h."""
    H_gpu = np.asarray(H_gpu, np.float64)
    err = np.abs(H_gpu - att.H)
    tally.worst_H = max(tally.worst_H, float(err.max()))
    assert err.max() <= H_ATOL, f"entropy error {err.max()} at row {int(err.argmax())}"
    mism = np.flatnonzero(np.asarray(argmax_gpu) != att.argmax)
    bad = [int(i) for i in mism if not flags[i]]
    assert not bad, f"argmax mismatch off a near-tie at rows {bad[:8]} (margins {att.margin[bad[:8]]})"
    tally.tie_mismatch += len(mism)
    r = sc_rel_err(np.asarray(sc_gpu, np.float64), att.sc)
    tally.worst_sc = max(tally.worst_sc, float(r.max()))
    assert r.max() <= SC_RTOL, f"sc relative error {r.max()} at row {int(r.argmax())}"


def compare_draw(tally: Tally, att, sampled_gpu):
    """Multinomial draws of the GPU against the oracle's Gumbel-max for the same h.

    A mismatch is allowed only where the oracle's two best z + G are within TIE
    (the GPU's logits and fast-log Gumbel variates carry errors well below it);
    such positions count toward the near-tie budget.
    """
    mism = np.flatnonzero(np.asarray(sampled_gpu) != att.sampled)
    bad = [int(i) for i in mism if not att.smargin[i] < TIE]
    assert not bad, f"draw mismatch off a near-tie at rows {bad[:8]} (gaps {att.smargin[bad[:8]]})"
    tally.tie_mismatch += len(mism)


def check_sampler_exact(w, block, t, H_gpu, argmax_gpu, canvas_in, out, chosen_gpu=None,
                        frozen=None):
    """The sampler given the GPU's own entropies and tokens must agree bit for bit.

    chosen_gpu: the tokens accepted positions take (the GPU's draws under the
    multinomial rule); the argmax when None. frozen: per canvas, stopped
    before this step (batched canvases).
    """
    H32 = np.asarray(H_gpu, np.float32)
    B = M.canvases(w)
    accepted, order, prefix, k = M.accept_canvases(H32, w.tau, w.accept_rule, B, frozen)
    noise = rng.tokens(w.seed, block, t, np.arange(w.C, dtype=np.uint64), w.V)
    tok = np.asarray(argmax_gpu if chosen_gpu is None else chosen_gpu)
    want_canvas = np.where(accepted, tok, noise)
    if frozen is not None:
        Cc = w.C // B
        for c in range(B):
            if frozen[c]:
                want_canvas[c * Cc:(c + 1) * Cc] = canvas_in[c * Cc:(c + 1) * Cc]
    assert np.array_equal(out["order"], order), "sort order differs"
    assert np.array_equal(out["prefix"], prefix), "prefix sums differ"
    assert np.array_equal(out["accept"].astype(bool), accepted), "accept mask differs"
    assert np.array_equal(out["canvas"], want_canvas), "canvas update differs"
    assert out["state"]["k"] == int(k.sum())
    return accepted


U32 = 2.0 ** -24      # fp32 unit roundoff


def h_agreement(w, h_gpu, h_orc, terms) -> float:
    """Fraction of hidden-state elements that differ, each within its error bound.

    The device evaluates h = A E[target] + B E[canvas] + sc + sigma g in fp32
    (four roundings of partial sums, and g from fp32 log, sqrt and cospi with a
    few ulps of relative error); the oracle evaluates it in fp64. With
    terms = |A E[target]| + |B E[canvas]| + |sc| + |sigma g| per element, every
    partial sum and the noise term are bounded by terms, so the fp32 result is
    within 8 u terms of the exact value (u = 2^-24; 4 ulps for the additions,
    4 for g). A bf16 workload then rounds both values to bf16: they may land on
    neighbouring bf16 values, so the bound there adds one bf16 ulp of the
    result (2^(e-8) for |h| in [2^(e-1), 2^e)).
    """
    h_gpu = np.asarray(h_gpu, np.float64)
    fp32_err = 8.0 * U32 * np.asarray(terms, np.float64)
    if w.dtype == "bf16":
        diff = h_gpu != h_orc
        if diff.any():
            e = np.frexp(np.maximum(np.abs(h_orc), np.abs(h_gpu)))[1]
            tol = np.ldexp(1.0, e - 8) + fp32_err
            assert np.all(np.abs(h_gpu - h_orc)[diff] <= tol[diff])
        return float(diff.mean())
    err = np.abs(h_gpu - h_orc)
    assert np.all(err <= fp32_err + 1e-30), float((err - fp32_err).max())
    return 0.0


def standin_terms(w, E32, target, canvas, sc, h_orc):
    """|A E[target]| + |B E[canvas]| + |sc| + |noise| of the oracle's stand-in (see h_agreement)."""
    a = w.coef_target * E32[np.asarray(target)].astype(np.float64)
    b = w.coef_canvas * E32[np.asarray(canvas)].astype(np.float64)
    s = np.asarray(sc, np.float64)
    # the noise term is what the unrounded sum needs beyond the other three; for
    # bf16 workloads h_orc is already rounded, which only adds to |noise| here
    n = np.asarray(h_orc, np.float64) - a - b - s
    return np.abs(a) + np.abs(b) + np.abs(s) + np.abs(n)


def reduce_partials_local(bufs, C: int, d: int) -> None:
    """The cross-shard reduction of vocabulary-parallel partials over buffers of
    one process (every buffer gets the result): the same sums and maxima the
    multi-GPU exchange (uniform_state_text_b200.allreduce_partials, NCCL) takes,
    for tests that run several shard contexts on one GPU or on the CPU. Test
    plumbing: eager torch ops, not part of the library's path."""
    import torch

    import uniform_state_text_b200 as dg
    views = [dg.partials_views(b, C, d) for b in bufs]
    fs = views[0][0].clone()
    for f, _ in views[1:]:
        fs += f
    ks = torch.stack([k.bitwise_xor(-(1 << 63)) for _, k in views]).amax(dim=0)
    ks.bitwise_xor_(-(1 << 63))
    for f, k in views:
        f.copy_(fs)
        k.copy_(ks)

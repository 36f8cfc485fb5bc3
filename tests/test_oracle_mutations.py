"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each one.

Every mutation is applied with monkeypatch to the oracle only and undone after
the test; a pin that passes with a mutation applied would be too weak.
"""
import math

import numpy as np
import pytest

from oracle import method as M
from oracle import rng

import test_oracle_attention as T_att
import test_oracle_rng as T_rng
import test_oracle_sampler as T_smp
import test_oracle_standin as T_std


def _fails(fn, *a, **kw):
    try:
        fn(*a, **kw)
    except AssertionError:
        return True
    return False


def test_wrong_mixer_constant_is_caught(monkeypatch):
    monkeypatch.setattr(rng, "_MUL2", rng._MUL2 ^ 0x10)
    assert _fails(T_rng.test_splitmix64_published_vector)


def test_wrong_schedule_denominator_is_caught(monkeypatch):
    def bad(t, S, T0, T1):
        return T1 + (T0 - T1) * 0.5 * (1.0 + math.cos(math.pi * t / S))
    monkeypatch.setattr(M, "temperature", bad)
    assert _fails(T_std.test_cosine_schedule_shape, 8, 1.0, 0.1)


def test_missing_logit_scale_is_caught(monkeypatch):
    real = M.logits
    monkeypatch.setattr(M, "logits", lambda h, E, scale: real(h, E, 1.0))
    assert _fails(T_att.test_matches_long_double_brute_force, 0)


def test_transposed_embedding_is_caught(monkeypatch):
    real = M.logits

    def bad(h, E, scale):
        z = real(h, E, scale)
        return z[:, ::-1].copy()          # vocabulary index reversed
    monkeypatch.setattr(M, "logits", bad)
    assert _fails(T_att.test_logits_orientation)


def test_entropy_in_bits_is_caught(monkeypatch):
    real = M.vocab_attention

    def bad(h, E, scale):
        a = real(h, E, scale)
        a.H = a.H / math.log(2.0)
        return a
    monkeypatch.setattr(M, "vocab_attention", bad)
    assert _fails(T_att.test_matches_long_double_brute_force, 1)


def test_unnormalised_self_conditioning_is_caught(monkeypatch):
    real = M.vocab_attention

    def bad(h, E, scale):
        a = real(h, E, scale)
        a.sc = a.sc * 1.01
        return a
    monkeypatch.setattr(M, "vocab_attention", bad)
    assert _fails(T_att.test_matches_long_double_brute_force, 2)


def test_strict_acceptance_comparison_is_caught(monkeypatch):
    def bad(H32, tau, rule):
        acc = M.Acceptance(order=np.argsort(H32, kind="stable"), accepted=np.zeros(len(H32), bool),
                           k=0, prefix=np.cumsum(np.asarray(H32, np.float32)))
        run = np.float32(0)
        for j, i in enumerate(acc.order):
            run = np.float32(run + H32[i])
            if run < np.float32(tau):
                acc.accepted[i] = True
                acc.k += 1
            else:
                break
        return acc
    monkeypatch.setattr(M, "entropy_bounded_accept", bad)
    assert _fails(T_smp.test_all_zero_entropy_accepts_everything, 0)


def test_renoise_with_wrong_step_key_is_caught(monkeypatch):
    real = rng.tokens

    def bad(seed, block, step, index, V):
        if step < rng.TAG_NOISE:
            step = step + 1
        return real(seed, block, step, index, V)
    monkeypatch.setattr(rng, "tokens", bad)
    assert _fails(T_smp.test_step_invariants_on_stress_data)


def test_dropped_noise_term_is_caught(monkeypatch):
    real = rng.gaussian
    monkeypatch.setattr(rng, "gaussian", lambda *a: 0.0 * real(*a))
    assert _fails(T_std.test_standin_noise_statistics_and_sc_term)


# --- multinomial draw (Gumbel-max) -------------------------------------------
import test_oracle_gumbel as T_gum


def test_gumbel_sign_flip_is_caught(monkeypatch):
    def bad(seed, block, step, index):
        W = rng.gumbel_uniform(rng.key(seed, block, step, index))
        return np.log(-np.log1p(-W))
    monkeypatch.setattr(rng, "gumbel", bad)
    assert _fails(T_gum.test_gumbel_cdf_mean_variance)


def test_gumbel_draw_at_wrong_temperature_is_caught(monkeypatch):
    real = M.gumbel_max
    monkeypatch.setattr(M, "gumbel_max", lambda z, *a, **k: real(2.0 * z, *a, **k))
    assert _fails(T_gum.test_draw_follows_softmax, [0.0, 1.0, 2.0, -1.0])


def test_gumbel_key_without_row_is_caught(monkeypatch):
    real = rng.gumbel

    def bad(seed, block, step, index):
        return real(seed, block, step, np.asarray(index, dtype=np.uint64) % np.uint64(4))
    monkeypatch.setattr(rng, "gumbel", bad)
    assert _fails(T_gum.test_draw_follows_softmax, [0.0, 1.0, 2.0, -1.0])


def test_multinomial_step_taking_the_argmax_is_caught(monkeypatch):
    real = M.vocab_attention

    def bad(h, E, scale, gumbel_key=None):
        a = real(h, E, scale, gumbel_key=gumbel_key)
        if a.sampled is not None:
            a.sampled = a.argmax.copy()
        return a
    monkeypatch.setattr(M, "vocab_attention", bad)
    assert _fails(T_gum.test_step_accepts_the_draw_and_keeps_the_distribution)


# --- batched canvases ----------------------------------------------------------
import test_oracle_batched as T_bat


def test_sort_across_canvases_is_caught(monkeypatch):
    def bad(H32, tau, rule, B, frozen=None):
        a = M.entropy_bounded_accept(H32, tau, rule)
        return a.accepted, a.order, a.prefix, np.array([a.k] + [0] * (B - 1))
    monkeypatch.setattr(M, "accept_canvases", bad)
    assert _fails(T_bat.test_two_canvas_example)


def test_budget_shared_between_canvases_is_caught(monkeypatch):
    real = M.accept_canvases
    monkeypatch.setattr(M, "accept_canvases",
                        lambda H32, tau, rule, B, frozen=None: real(H32, tau / B, rule, B, frozen))
    assert _fails(T_bat.test_two_canvas_example)


def test_stopped_canvas_not_frozen_is_caught(monkeypatch):
    real = M.accept_canvases
    monkeypatch.setattr(M, "accept_canvases",
                        lambda H32, tau, rule, B, frozen=None: real(H32, tau, rule, B, None))
    assert _fails(T_bat.test_block_invariants_and_freezing)

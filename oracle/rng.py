"""Counter-based randomness of the denoise loop (oracle side).

TEST INFRASTRUCTURE (see the package docstring).

The pages draw three kinds of random values: the uniform random initial canvas
(A Visual Guide to DiffusionGemma, 5.4 "canvas initialisation": tokens drawn
uniformly from the vocabulary), the fresh uniform token given to every rejected
position (5.4 "token re-noising"), and, in the synthetic stand-in backbone, a
Gaussian perturbation of the hidden state. All are keyed, not sequential, so
that a position's draw depends only on (seed, block, step, index).

SplitMix64 is the generator of Steele, Lea and Flood, "Fast splittable
pseudorandom number generators" (OOPSLA 2014), in the form of S. Vigna's public
domain reference: the state advances by the golden gamma 0x9E3779B97F4A7C15 and
each output is the state passed through a two-multiply xor-shift finaliser.
sm(x) below is the output produced from state x (gamma added, then mixed).

key(s, b, t, i) = sm(sm(sm(sm(s) ^ b) ^ t) ^ i), all arithmetic mod 2**64.
Token draws take key & (V - 1) (V is a power of two, so this is exact and
unbiased). Gaussian draws use Box-Muller on two 24-bit uniforms cut from one
key: u1 = ((k >> 40) + 1) / 2**24 in (0, 1], u2 = ((k >> 16) & 0xFFFFFF) / 2**24
in [0, 1), g = sqrt(-2 ln u1) * cos(2 pi u2).

The multinomial token choice (A Visual Guide to DiffusionGemma, 3.2: tokens
are drawn from the predicted distribution) uses one Gumbel variate per
(position, vocabulary entry). Standard Gumbel draws come from one key each:
W = (2 (k >> 41) + 1) / 2**24, an odd multiple of 2**-24 in (0, 1) that fp32
holds exactly; X = -ln(1 - W) is then a unit exponential and G = -ln X a
standard Gumbel variate (P(G <= x) = exp(-exp(-x))).
"""
from __future__ import annotations

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_MUL1 = 0xBF58476D1CE4E5B9
_MUL2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1

# Domain tags carried in the step field of the key.
TAG_INIT_CANVAS = (1 << 63) + 1
TAG_TARGET = (1 << 63) + 2
TAG_NOISE = 1 << 62          # + step index
TAG_GUMBEL = 1 << 61         # + step index; index = position * V + vocabulary entry


def _u64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.uint64)


def sm(x) -> np.ndarray:
    """One SplitMix64 output from state x (vectorised, wrapping uint64)."""
    with np.errstate(over="ignore"):
        z = _u64(x) + np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MUL1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MUL2)
        return z ^ (z >> np.uint64(31))


def sm_int(x: int) -> int:
    """Scalar SplitMix64 output on Python ints (same definition, no numpy)."""
    z = (x + GAMMA) & _MASK
    z = ((z ^ (z >> 30)) * _MUL1) & _MASK
    z = ((z ^ (z >> 27)) * _MUL2) & _MASK
    return z ^ (z >> 31)


def key(seed: int, block: int, step: int, index) -> np.ndarray:
    """key(s, b, t, i) for a vector of indices i."""
    s = int(sm_int(seed & _MASK))
    sb = int(sm_int((s ^ (block & _MASK)) & _MASK))
    sbt = int(sm_int((sb ^ (step & _MASK)) & _MASK))
    return sm(np.uint64(sbt) ^ _u64(index))


def tokens(seed: int, block: int, step: int, index, V: int) -> np.ndarray:
    """Uniform vocabulary tokens key & (V-1) as int64 (V a power of two)."""
    if V <= 0 or (V & (V - 1)) != 0:
        raise ValueError("V must be a power of two")
    return (key(seed, block, step, index) & np.uint64(V - 1)).astype(np.int64)


def gaussian(seed: int, block: int, step: int, index) -> np.ndarray:
    """Standard normal draws (fp64) by Box-Muller from one key per index."""
    k = key(seed, block, step, index)
    u1 = ((k >> np.uint64(40)).astype(np.float64) + 1.0) * 2.0 ** -24
    u2 = ((k >> np.uint64(16)) & np.uint64(0xFFFFFF)).astype(np.float64) * 2.0 ** -24
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def gumbel_uniform(k) -> np.ndarray:
    """W = (2 (k >> 41) + 1) / 2**24 in (0, 1), fp64 (exact in fp32 as well)."""
    return ((k >> np.uint64(41)).astype(np.float64) * 2.0 + 1.0) * 2.0 ** -24


def gumbel(seed: int, block: int, step: int, index) -> np.ndarray:
    """Standard Gumbel draws (fp64): G = -ln(-ln(1 - W)) from one key per index."""
    W = gumbel_uniform(key(seed, block, step, index))
    return -np.log(-np.log1p(-W))

"""8-bit floating point for a narrow vocabulary embedding (oracle).

TEST INFRASTRUCTURE (see the package docstring).

The pages name a quantised model for the smaller GPUs ("DiffusionGemma: from
autoregressive to diffusion denoising", the throughput table: the 26B-A4B model
in NVFP4 fits an 18 GB GPU; "A Visual Guide to DiffusionGemma" on the roofline
of the step). They give no format details. The reading here, for the step's
own arithmetic:

  * E is stored as e4m3 codes with one power-of-two scale per block of
    GROUP = 256 consecutive vocabulary rows: E_deq[v] = q[v] * 2^e[v], e[v]
    the smallest exponent with max |E[block of v]| * 2^-e[v] <= 448 (the
    e4m3 maximum), the same for every row of the block. Blocks run along the
    vocabulary, not along d (as 32-element MX blocks would), because the
    second contraction, p.E, sums over the vocabulary: a scale that varies
    along d cannot be taken out of that sum, one per vocabulary block folds
    into p exactly. e4m3 is a floating-point format: entries down to
    2^-6 / 448 (about 2^-14.8) of their block's largest keep its relative
    precision of 2^-4, so rows smaller than their block's largest lose
    little.
  * h is quantised the same way per canvas row (e4m3, power-of-two scale).
  * The logits, entropy, argmax and the partition sum are those of h_deq and
    E_deq (fp32 accumulation on the device, fp64 here).
  * For sc = sum_v p_v E_deq[v] / Z the device multiplies each probability
    taken against the row's reference, exp(z_v - m_ref), by 2^(e[v] - u)
    (u one exponent for the whole step) and rounds it to e5m2, whose range
    (2^-16 .. 57344) keeps probabilities down to about e^-13 of the
    reference; sc = 2^u sum_v P'_v q[v] / Z, with Z from the unrounded
    probabilities.

Rounding is to nearest, ties to even, with saturation at the format's largest
finite value (the device's satfinite conversions); subnormals are kept.
"""
from __future__ import annotations

import math

import numpy as np

# (mantissa bits, smallest normal exponent, largest finite value)
FORMATS = {
    "e4m3": (3, -6, 448.0),
    "e5m2": (2, -14, 57344.0),
}


def fp8_round(x, fmt: str) -> np.ndarray:
    """x rounded to the nearest value of the 8-bit format (ties to even), saturated."""
    mb, emin, vmax = FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    e = np.frexp(np.where(ax > 0, ax, 1.0))[1] - 1     # |x| in [2^e, 2^(e+1))
    e = np.maximum(e, emin)
    q = np.ldexp(1.0, (e - mb).astype(np.int64))      # spacing of the values in x's binade
    r = np.rint(x / q) * q                             # rint: ties to even
    return np.clip(r, -vmax, vmax)


def row_scale_exponent(amax, fmt: str = "e4m3") -> np.ndarray:
    """Smallest integer e with amax * 2^-e <= the format's largest value (0 for amax = 0).

    amax = m 2^x with m in [0.5, 1); the largest value is 0.875 2^k (448 = 0.875 2^9,
    57344 = 0.875 2^16), so e = x - k, plus one when m > 0.875.
    """
    _, _, vmax = FORMATS[fmt]
    m_top, k = math.frexp(vmax)
    amax = np.asarray(amax, dtype=np.float64)
    m, x = np.frexp(amax)
    e = x - k + (m > m_top).astype(np.int64)
    return np.where(amax > 0, e, 0).astype(np.int64)


def quantize_rows(X, fmt: str = "e4m3", group: int = 1):
    """Power-of-two scaling per block of `group` consecutive rows, and rounding:
    returns (codes as values, one exponent per row, equal within a block).

    X[r] ~= codes[r] * 2^exps[r]; codes lie in the format's range.
    """
    X = np.asarray(X, dtype=np.float64)
    amax = np.abs(X).max(axis=1)
    if group > 1:
        n = X.shape[0]
        assert n % group == 0
        amax = np.repeat(amax.reshape(n // group, group).max(axis=1), group)
    e = row_scale_exponent(amax, fmt)
    return fp8_round(np.ldexp(X, -e[:, None]), fmt), e


def dequantize_rows(codes, exps) -> np.ndarray:
    return np.ldexp(np.asarray(codes, np.float64), np.asarray(exps)[:, None])


def sc_from_quantized_p(z, m_ref, E_codes, E_exps, u: int) -> np.ndarray:
    """sc of one step in the narrow-E form: probabilities against the row's
    reference, scaled by 2^(e[v] - u) and rounded to e5m2, then summed against
    the e4m3 codes and normalised by the unrounded partition sum.

    z [rows][V] tempered logits (of h_deq and E_deq), m_ref [rows].
    """
    z = np.asarray(z, np.float64)
    m_ref = np.asarray(m_ref, np.float64)
    P = np.exp(z - m_ref[:, None])
    Z = P.sum(axis=1)
    Pq = fp8_round(np.ldexp(P, (np.asarray(E_exps)[None, :] - u)), "e5m2")
    num = Pq @ np.asarray(E_codes, np.float64)
    return np.ldexp(num, u) / Z[:, None]


# ----------------------------------------------------------------------------
# The step's vocabulary attention with narrow E.
# ----------------------------------------------------------------------------
# The reference of each row may lag the row's largest logit by at most
# REDO_GAP before the row is redone against its exact maximum, and the step
# exponent is the largest row exponent of E minus U_OFFSET: together they keep
# e^REDO_GAP 2^(e[v] - u) <= 54.6 * 2^10 within e5m2's range.
REDO_GAP = 4.0
U_OFFSET = 10
GROUP = 256          # vocabulary rows per scale of E


def step_exponent(E_exps) -> int:
    return int(np.max(E_exps)) - U_OFFSET


class NarrowE:
    """E held as e4m3 codes with one power-of-two exponent per block of GROUP
    vocabulary rows (see the module docstring; exps holds it for every row);
    E_deq is the embedding every other part of the step uses."""

    def __init__(self, E):
        V, d = E.shape
        self.codes = np.empty((V, d), dtype=np.float32)   # exact: e4m3 values are fp32 values
        self.exps = np.empty(V, dtype=np.int64)
        for r0 in range(0, V, 8192):                     # row chunks bound the fp64 temporaries
            q, e = quantize_rows(E[r0:r0 + 8192], "e4m3", group=min(GROUP, V))
            self.codes[r0:r0 + 8192] = q
            self.exps[r0:r0 + 8192] = e
        self.E_deq = np.ldexp(self.codes, self.exps[:, None]).astype(np.float32)   # exact as well
        self.u = step_exponent(self.exps)


def narrow_attention(nE: NarrowE, h, scale, canvas, prev, gumbel_key=None, m_ref=None):
    """Entropy, argmax, draw and sc of a step with narrow E.

    h (the stand-in or the caller's, already bf16) is quantised per row (one
    exponent per canvas row); the
    logits are those of h_deq and E_deq. The reference of row i is the logit of
    its canvas token or previous prediction, whichever is larger (prev = canvas
    on the block's first step), raised to the row's largest logit when it lags
    that by more than REDO_GAP; m_ref, when given, is used as it stands.
    Returns (Attention with the narrow-E sc, the references used).
    """
    from . import method as M

    hq, he = quantize_rows(h, "e4m3")
    h_deq = dequantize_rows(hq, he)
    att = M.vocab_attention(h_deq, nE.E_deq, scale, gumbel_key=gumbel_key)
    rows = np.arange(h_deq.shape[0])
    if m_ref is None:
        Ec = nE.E_deq[np.asarray(canvas)].astype(np.float64)
        Ep = nE.E_deq[np.asarray(prev)].astype(np.float64)
        m_ref = scale * np.maximum((h_deq * Ec).sum(axis=1), (h_deq * Ep).sum(axis=1))
        m_ref = np.where(att.zmax - m_ref > REDO_GAP, att.zmax, m_ref)
    m_ref = np.asarray(m_ref, np.float64)
    num = np.zeros((len(rows), nE.codes.shape[1]))
    Z = np.zeros(len(rows))
    for v0 in range(0, nE.codes.shape[0], 8192):
        Ed = nE.E_deq[v0:v0 + 8192].astype(np.float64)
        z = scale * (h_deq @ Ed.T)
        P = np.exp(z - m_ref[:, None])
        Z += P.sum(axis=1)
        Pq = fp8_round(np.ldexp(P, nE.exps[None, v0:v0 + 8192] - nE.u), "e5m2")
        num += Pq @ nE.codes[v0:v0 + 8192].astype(np.float64)
    att.sc = np.ldexp(num, nE.u) / Z[:, None]
    return att, m_ref

"""The denoise step of uniform-state text diffusion, written out plainly (oracle).

TEST INFRASTRUCTURE (see the package docstring).

Sources (page title, section):
  [VG]  "A Visual Guide to DiffusionGemma" (zh-CN translation, hubwiz.com):
        3.2 uniform-state diffusion; 5.1 self-conditioning; 5.2 multi-canvas
        sampling; 5.3 scheduler (step budget, logits temperature schedule,
        adaptive stop); 5.4 entropy-bounded sampler (canvas initialisation,
        token acceptance, token re-noising).
  [DP]  "DiffusionGemma: from autoregressive to diffusion denoising" (blog,
        vatt-ghern.pages.dev): the diffusion decode loop pseudocode
        (canvas = random_tokens(256); for step: logits = model(canvas);
        conf = confidence(logits); canvas = update(...)).
  [WS]  local-deploy workshop (yomxxx.com): "scheduler" (temperature high early,
        low late; stop when either stability or confidence holds; entropy below
        0.005) and "entropy-constrained sampler" (sort by entropy ascending,
        accept while the cumulative entropy stays within the threshold,
        re-noise the rest); generate(..., temperature_schedule="cosine").
  [EX]  "DiffusionGemma explained" (ai.google.dev, ja; zh-TW translation on
        gemma.gh.miniasp.com): self-conditioning multiplies the probability
        matrix by the token embedding table; 256-token canvases, block by block.

Readings where the pages are silent or garbled:
  * The acceptance formula is lost in extraction ([VG] 5.4 ends "based on the
    following formula:"). Default rule (accept_rule 0): accept the sorted
    prefix whose inclusive running entropy sum is <= tau ([WS]). Rule 1 reads
    [VG]'s "sum so far minus the maximum entropy": in ascending order the
    maximum so far is the current entry, so a position is accepted when the sum
    of the entries before it is <= tau (always accepts at least one).
  * Tokens are chosen by argmax (the most likely token per position, [VG] 3.2);
    ties go to the lowest vocabulary index. token_rule 1 instead draws each
    position's token from its softmax distribution ([VG] 3.2 names the
    multinomial draw): the Gumbel-max form, argmax_v (z_v + G_v) with one
    keyed standard Gumbel variate G_v per (position, entry) (rng.gumbel, step
    field TAG_GUMBEL + t, index position * V + v). Entropy, sc, the stop test
    and the emitted prediction still use the distribution and its argmax.
  * Logits temperature: T_t = T_end + (T_start - T_end) * (1 + cos(pi t/(S-1)))/2,
    t = 0..S-1 (the cosine schedule of [WS]; lower temperature at later steps,
    [VG] 5.3); S = 1 gives T_start.
  * Entropy in nats, H = -sum p log p, clamped at 0.
  * Entropy sort ties: lower position first (stable).
  * Adaptive stop (stop_rule 0): the canvas unchanged for N consecutive steps,
    OR all entropies < stop_entropy, OR the step budget reached. stop_rule 1
    compares the argmax predictions of consecutive steps instead.
  * A finished block emits the final step's argmax at every position.
  * Batched canvases (canvases = B > 1): B independent canvases of C/B
    positions share each step's vocabulary attention (the rows are
    independent). Entropy sort, acceptance (tau per canvas), re-noise and the
    adaptive stop apply to each canvas on its own; a canvas that has stopped is
    frozen (its tokens and emitted prediction no longer change) while the
    others go on, and the block ends when every canvas has stopped. Keys stay
    those of the combined row index, so canvas c is rows [c C/B, (c+1) C/B)
    of a C-row canvas.
  * Self-conditioning feeds sc = softmax(z) E of the tempered logits straight
    into the next step's stand-in hidden state. The small feed-forward network
    that [VG] 5.1 puts between sc and the next step's token embeddings is
    self_condition_ffnn (for a caller's backbone and weights): the pages give
    no shape, so the reading is two linear layers with a GELU between them
    (the tanh form), y = W2 gelu(W1 sc + b1) + b2, weights [out][in].

Precision: fp64 throughout. Decisions that turn floats into integers are taken
in fp32, the precision the CUDA kernels take them in: argmax over fp32-rounded
logits, the sort over fp32-rounded entropies, sequential fp32 prefix sums of
the sorted entropies compared with fp32(tau), and H_fp32 < fp32(stop_entropy).
For bf16 workloads the stand-in hidden state is rounded to bf16
(round-to-nearest-even) before the dot products, as the kernels see it.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from . import rng

_VOCAB_CHUNK = 8192


# ----------------------------------------------------------------------------
# Scheduler: cosine logits temperature ([VG] 5.3, [WS] scheduler).
# ----------------------------------------------------------------------------
def temperature(t: int, S: int, T_start: float, T_end: float) -> float:
    if S <= 1:
        return float(T_start)
    return T_end + (T_start - T_end) * 0.5 * (1.0 + math.cos(math.pi * t / (S - 1)))


# ----------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even), done on fp64 values directly.
# ----------------------------------------------------------------------------
def bf16_round(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                     # x = m * 2**e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits; below 2**-126 the quantum is fixed.
    e = np.maximum(e, -125)
    q = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)
    return np.where(x == 0.0, x, q)


# ----------------------------------------------------------------------------
# Canvas initialisation ([VG] 5.4) and the stand-in backbone.
# ----------------------------------------------------------------------------
def init_block(w, block: int):
    """Targets and initial canvas of one block: uniform tokens keyed on seed+block."""
    pos = np.arange(w.C, dtype=np.uint64)
    s = (w.seed + block) & ((1 << 64) - 1)
    target = rng.tokens(s, 0, rng.TAG_TARGET, pos, w.V)
    canvas = rng.tokens(s, 0, rng.TAG_INIT_CANVAS, pos, w.V)
    return target, canvas


def standin_hidden(w, E: np.ndarray, target, canvas, sc_prev, block: int, t: int):
    """h_i = A E[target_i] + B E[canvas_i] + sc_prev_i + eps_i, eps ~ N(0, (noise_var_d/d) I).

    Replaces the bidirectional denoiser, which needs trained weights. The
    self-conditioning vector of the previous step enters additively ([VG] 5.1).
    """
    C, d = w.C, w.d
    idx = (np.arange(C, dtype=np.uint64)[:, None] * np.uint64(d)
           + np.arange(d, dtype=np.uint64)[None, :])
    eps = rng.gaussian(w.seed, block, rng.TAG_NOISE + t, idx) * math.sqrt(w.noise_var_d / d)
    Et = E[np.asarray(target)].astype(np.float64)
    Ec = E[np.asarray(canvas)].astype(np.float64)
    h = w.coef_target * Et + w.coef_canvas * Ec + np.asarray(sc_prev, np.float64) + eps
    if w.dtype == "bf16":
        h = bf16_round(h)
    return h


# ----------------------------------------------------------------------------
# Logits -> probabilities, entropy, argmax, self-conditioning vector.
# ----------------------------------------------------------------------------
def logits(h: np.ndarray, E: np.ndarray, scale: float) -> np.ndarray:
    """z[i, v] = scale * <h_i, E_v>, fp64, materialised as [rows, V]."""
    h = np.asarray(h, dtype=np.float64)
    V = E.shape[0]
    z = np.empty((h.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, _VOCAB_CHUNK):
        Ec = E[v0:v0 + _VOCAB_CHUNK].astype(np.float64)
        z[:, v0:v0 + Ec.shape[0]] = scale * (h @ Ec.T)
    return z


@dataclasses.dataclass
class Attention:
    argmax: np.ndarray      # int64 [rows]; decided on fp32-rounded logits
    H: np.ndarray           # fp64 [rows]; entropy in nats, >= 0
    sc: np.ndarray          # fp64 [rows, d]; sum_v p_v E_v
    zmax: np.ndarray        # fp64 [rows]; largest logit
    margin: np.ndarray      # fp64 [rows]; gap between the two largest logits
    sampled: np.ndarray | None = None   # int64 [rows]; Gumbel-max draw (token_rule 1)
    smargin: np.ndarray | None = None   # fp64 [rows]; gap between the two best z + G


def gumbel_max(z: np.ndarray, seed: int, block: int, t: int, rows0: int = 0):
    """Draw one token per row from softmax(z) as argmax_v (z_v + G_v).

    G_v are independent standard Gumbel variates keyed on (seed, block,
    TAG_GUMBEL + t, row * V + v); row numbers start at rows0. Returns the tokens
    (first index on exact ties) and the gap between the two best scores.
    """
    rows, V = z.shape
    tok = np.empty(rows, dtype=np.int64)
    gap = np.empty(rows)
    for i in range(rows):
        idx = np.uint64((rows0 + i) * V) + np.arange(V, dtype=np.uint64)
        score = z[i] + rng.gumbel(seed, block, rng.TAG_GUMBEL + t, idx)
        tok[i] = int(np.argmax(score))
        if V > 1:
            top2 = np.partition(score, -2)[-2:]
            gap[i] = abs(top2[1] - top2[0])
        else:
            gap[i] = np.inf
    return tok, gap


def vocab_attention(h: np.ndarray, E: np.ndarray, scale: float,
                    gumbel_key: tuple[int, int, int] | None = None) -> Attention:
    """Per position: softmax of the tempered logits, its entropy, argmax and p.E.

    The probability of each vocabulary token is the softmax of the logits
    divided by the temperature ([VG] 5.3 logits scheduler); confidence is the
    entropy of that distribution ([VG] 5.3 adaptive stop, 5.4 acceptance); the
    self-conditioning vector is the probability row times the embedding table
    ([VG] 5.1, [EX] self-conditioning). With gumbel_key = (seed, block, t) it
    also draws one token per position from that distribution (gumbel_max).
    """
    z = logits(h, E, scale)
    rows = z.shape[0]
    zmax = z.max(axis=1)
    z32 = z.astype(np.float32)
    argmax = np.argmax(z32, axis=1).astype(np.int64)        # first index of max
    top2 = np.partition(z, -2, axis=1)[:, -2:] if z.shape[1] > 1 else np.stack([zmax, zmax], 1)
    margin = np.abs(top2[:, 1] - top2[:, 0])
    logZ = np.empty(rows)
    H = np.empty(rows)
    p = np.empty_like(z)
    for i in range(rows):
        shifted = z[i] - zmax[i]
        e = np.exp(shifted)
        Z = e.sum()
        logZ[i] = math.log(Z)
        p[i] = e / Z
        logp = shifted - logZ[i]
        H[i] = max(0.0, float(-(p[i] * logp).sum()))
    d = E.shape[1]
    sc = np.zeros((rows, d), dtype=np.float64)
    for v0 in range(0, E.shape[0], _VOCAB_CHUNK):
        Ec = E[v0:v0 + _VOCAB_CHUNK].astype(np.float64)
        sc += p[:, v0:v0 + Ec.shape[0]] @ Ec
    sampled = smargin = None
    if gumbel_key is not None:
        sampled, smargin = gumbel_max(z, *gumbel_key)
    return Attention(argmax=argmax, H=H, sc=sc, zmax=zmax, margin=margin,
                     sampled=sampled, smargin=smargin)


# ----------------------------------------------------------------------------
# Self-conditioning feed-forward network ([VG] 5.1: the probability-weighted
# embeddings "are passed to a small FFNN and added to the next step's token
# embeddings"; [EX] self-conditioning).
# ----------------------------------------------------------------------------
def gelu_tanh(a: np.ndarray) -> np.ndarray:
    """GELU in its tanh form: a/2 (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3)))."""
    a = np.asarray(a, dtype=np.float64)
    return 0.5 * a * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (a + 0.044715 * a ** 3)))


def self_condition_ffnn(sc, W1, b1, W2, b2) -> np.ndarray:
    """y = W2 gelu(W1 sc + b1) + b2 for every canvas row of sc [C][d].

    W1 [d_ff][d] and W2 [d][d_ff] (each row: one output unit's weights), b1
    [d_ff], b2 [d]. The tensor-core kernels take sc and the hidden activations
    as bf16 operands, so both are rounded to bf16 (round to nearest even) before
    the products, as there; everything else is fp64.
    """
    x = bf16_round(np.asarray(sc, np.float64))
    a = x @ np.asarray(W1, np.float64).T + np.asarray(b1, np.float64)[None, :]
    g = bf16_round(gelu_tanh(a))
    return g @ np.asarray(W2, np.float64).T + np.asarray(b2, np.float64)[None, :]


def add_to_embeddings(emb, y, dtype: str) -> np.ndarray:
    """The next step's token embeddings plus the network's output, in emb's type
    (bf16 embeddings: the sum rounded to bf16)."""
    s = np.asarray(emb, np.float64) + np.asarray(y, np.float64)
    return bf16_round(s) if dtype == "bf16" else s


# ----------------------------------------------------------------------------
# Entropy-bounded sampler ([VG] 5.4, [WS] entropy-constrained sampler).
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Acceptance:
    order: np.ndarray       # positions sorted by (H_fp32, position)
    accepted: np.ndarray    # bool [C]
    k: int                  # number accepted
    prefix: np.ndarray      # fp32 inclusive prefix sums in sorted order


def entropy_bounded_accept(H32: np.ndarray, tau: float, rule: int) -> Acceptance:
    """Sort positions from lowest to highest entropy and walk the list.

    rule 0: accept while the running sum including this entry is <= tau.
    rule 1: accept while the running sum minus the largest entropy seen so far
            (the current entry, in ascending order) is <= tau.
    Sums are sequential fp32 additions in sorted order, compared with fp32(tau).
    """
    H32 = np.asarray(H32, dtype=np.float32)
    C = H32.shape[0]
    order = np.argsort(H32, kind="stable")
    tau32 = np.float32(tau)
    prefix = np.zeros(C, dtype=np.float32)
    run = np.float32(0.0)
    accepted = np.zeros(C, dtype=bool)
    k = 0
    stopped = False
    for j in range(C):
        before = run
        run = np.float32(run + H32[order[j]])
        prefix[j] = run
        ok = (run <= tau32) if rule == 0 else (before <= tau32)
        if ok and not stopped:
            accepted[order[j]] = True
            k += 1
        else:
            stopped = True
    return Acceptance(order=order, accepted=accepted, k=k, prefix=prefix)


def accept_canvases(H32: np.ndarray, tau: float, rule: int, B: int, frozen=None):
    """The entropy-bounded sampler on each of B canvases of len(H32)/B positions.

    Canvas c is positions [c C/B, (c+1) C/B); it is sorted and accepted on its
    own with its own budget tau. Frozen canvases (frozen[c] true) accept
    nothing and keep the identity order. Returns (accepted bool [C], order
    int64 [C] of global positions, per-canvas fp32 prefix sums [C], k per canvas).
    """
    H32 = np.asarray(H32, dtype=np.float32)
    C = H32.shape[0]
    Cc = C // B
    accepted = np.zeros(C, dtype=bool)
    order = np.arange(C, dtype=np.int64)
    prefix = np.zeros(C, dtype=np.float32)
    k = np.zeros(B, dtype=np.int64)
    for c in range(B):
        if frozen is not None and frozen[c]:
            continue
        seg = slice(c * Cc, (c + 1) * Cc)
        a = entropy_bounded_accept(H32[seg], tau, rule)
        accepted[seg] = a.accepted
        order[seg] = a.order + c * Cc
        prefix[seg] = a.prefix
        k[c] = a.k
    return accepted, order, prefix, k


def renoise(w, accepted, chosen, block: int, t: int):
    """Token re-noising ([VG] 5.4): accepted positions take the chosen token
    (argmax, or the draw under token_rule 1); every rejected one a fresh
    uniform token key(seed, block, t, position) & (V - 1) ([VG] 3.2: the noise
    of uniform-state diffusion is a uniformly random vocabulary token).
    Returns (proposed canvas, the noise tokens)."""
    noise = rng.tokens(w.seed, block, t, np.arange(w.C, dtype=np.uint64), w.V)
    return np.where(accepted, chosen, noise).astype(np.int64), noise


# ----------------------------------------------------------------------------
# One step and the block loop ([DP] decode loop; [VG] 5.2, 5.3).
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class State:
    block: int
    t: int
    target: np.ndarray
    canvas: np.ndarray
    sc: np.ndarray
    unchanged: int = 0
    argmax_prev: np.ndarray | None = None
    done: bool = False
    steps_done: int = 0
    # batched canvases: per-canvas stop state and the emitted predictions
    unchanged_c: np.ndarray | None = None
    done_c: np.ndarray | None = None
    steps_c: np.ndarray | None = None
    emit: np.ndarray | None = None


@dataclasses.dataclass
class StepRecord:
    t: int
    temperature: float
    h: np.ndarray
    att: Attention
    acc: Acceptance
    canvas_in: np.ndarray
    canvas_out: np.ndarray
    noise: np.ndarray
    unchanged: int
    all_confident: bool
    done: bool


def canvases(w) -> int:
    return int(getattr(w, "canvases", 1))


def begin_block(w, block: int) -> State:
    target, canvas = init_block(w, block)
    B = canvases(w)
    return State(block=block, t=0, target=target, canvas=canvas,
                 sc=np.zeros((w.C, w.d), dtype=np.float64),
                 unchanged_c=np.zeros(B, dtype=np.int64), done_c=np.zeros(B, dtype=bool),
                 steps_c=np.zeros(B, dtype=np.int64), emit=np.zeros(w.C, dtype=np.int64))


def step(w, E: np.ndarray, st: State, h: np.ndarray | None = None, narrow=None) -> StepRecord:
    """One denoise step from state st (mutated in place). h overrides the stand-in.

    narrow: an fp8.NarrowE for a workload with narrow E (E must then be its
    E_deq); the attention then follows fp8.narrow_attention.
    """
    t = st.t
    T = temperature(t, w.max_steps, w.T_start, w.T_end)
    if h is None:
        h = standin_hidden(w, E, st.target, st.canvas, st.sc, st.block, t)
    multinomial = getattr(w, "token_rule", 0) == 1
    gkey = (w.seed, st.block, t) if multinomial else None
    if narrow is not None:
        from . import fp8
        prev = st.argmax_prev if st.argmax_prev is not None else st.canvas
        att, _ = fp8.narrow_attention(narrow, h, w.logit_scale / T, st.canvas, prev,
                                      gumbel_key=gkey)
    elif multinomial:
        att = vocab_attention(h, E, w.logit_scale / T, gumbel_key=gkey)
    else:
        att = vocab_attention(h, E, w.logit_scale / T)
    H32 = att.H.astype(np.float32)
    chosen = att.sampled if multinomial else att.argmax
    B = canvases(w)
    Cc = w.C // B
    last = (t + 1 >= w.max_steps)
    canvas_out = st.canvas.copy()
    accepted, order, prefix, k_c = accept_canvases(H32, w.tau, w.accept_rule, B, st.done_c)
    proposed, noise = renoise(w, accepted, chosen, st.block, t)
    conf_c = np.zeros(B, dtype=bool)
    for c in range(B):
        seg = slice(c * Cc, (c + 1) * Cc)
        if st.done_c[c]:
            continue                      # a stopped canvas is frozen
        canvas_out[seg] = proposed[seg]
        conf_c[c] = bool(np.all(H32[seg] < np.float32(w.stop_entropy)))
        if w.stop_rule == 0:
            same = bool(np.array_equal(canvas_out[seg], st.canvas[seg]))
        else:
            same = st.argmax_prev is not None and bool(
                np.array_equal(att.argmax[seg], st.argmax_prev[seg]))
        st.unchanged_c[c] = st.unchanged_c[c] + 1 if same else 0
        if w.fixed_steps:
            stop = last
        else:
            stop = last or conf_c[c] or st.unchanged_c[c] >= w.stop_unchanged
        if stop:
            st.done_c[c] = True
            st.steps_c[c] = t + 1
            st.emit[seg] = att.argmax[seg]
    if B == 1:
        acc = entropy_bounded_accept(H32, w.tau, w.accept_rule)
    else:
        acc = Acceptance(order=order, accepted=accepted, k=int(k_c.sum()), prefix=prefix)
    done = bool(np.all(st.done_c))
    unchanged = int(st.unchanged_c[0])
    all_conf = bool(np.all(conf_c))
    rec = StepRecord(t=t, temperature=T, h=h, att=att, acc=acc, canvas_in=st.canvas.copy(),
                     canvas_out=canvas_out, noise=noise, unchanged=unchanged,
                     all_confident=all_conf, done=done)
    st.canvas = canvas_out
    st.sc = att.sc
    st.unchanged = unchanged
    st.argmax_prev = att.argmax
    st.t = t + 1
    st.done = done
    st.steps_done = t + 1
    return rec


def denoise_block(w, E: np.ndarray, block: int, narrow=None):
    """Run the block's canvases to their stops.

    Returns (emitted tokens -- each canvas's argmax at its own final step --,
    steps the block ran, per-step records).
    """
    st = begin_block(w, block)
    records = []
    while not st.done:
        records.append(step(w, E, st, narrow=narrow))
    return st.emit.copy(), st.steps_done, records


def generate(w, E: np.ndarray):
    """Blocks 0..blocks-1 in sequence; each block's final argmax is emitted."""
    out = np.zeros(w.blocks * w.C, dtype=np.int64)
    steps = []
    for b in range(w.blocks):
        tokens, n, _ = denoise_block(w, E, b)
        out[b * w.C:(b + 1) * w.C] = tokens
        steps.append(n)
    return out, steps

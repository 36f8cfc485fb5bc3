"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

Teacher-forced step parity: before each GPU step the canvas, sc and step index
are read back; the oracle recomputes the stand-in hidden state from them
(compared element by element), then the vocabulary attention from the GPU's
own hidden state (entropy, argmax, sc) and the sampler twice: from the GPU's
entropies (must agree bit for bit) and from its own (near-tie budget).
Trajectory parity runs whole blocks through the CUDA-graph loop.
"""
import numpy as np
import pytest
import torch

import synthetic
import uniform_state_text_b200 as dg
from oracle import fp8 as F8
from oracle import method as M
from parity import (Tally, check_sampler_exact, compare_attention, compare_draw, h_agreement,
                    near_tie_flags, reduce_partials_local, standin_terms)

pytestmark = pytest.mark.gpu

IMPLS = [dg.DG_IMPL_SIMT, dg.DG_IMPL_TC]
_E_CACHE = {}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from uniform_state_text_b200 import build
    build.build()
    dg.lib()


def embedding(w):
    key = (w.V, w.d, w.dtype, w.e_seed)
    if key not in _E_CACHE:
        _E_CACHE.clear()
        E = synthetic.make_embedding(w)
        _E_CACHE[key] = (E.cuda(), synthetic.embedding_as_f32(E))
    return _E_CACHE[key]


def supported(w, impl):
    return dg.dg_workspace_bytes(dg.make_config(w, impl)) > 0


def make(w, impl):
    if not supported(w, impl):
        pytest.skip(f"impl {impl} does not cover {w.name}")
    Eg, E32 = embedding(w)
    den = dg.Denoiser(w, Eg, impl=impl)
    assert den.impl == impl
    return den, E32


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float32) \
        else t.detach().cpu().numpy()


def step_and_compare(den, w, E32, tally: Tally, prev_amax=None, do_step=None, peers=(),
                     h_given=None, narrow=None):
    """One GPU step (den.step(), or do_step()) compared with the oracle.

    peers: other contexts stepped by do_step (vocabulary shards) that must end
    in exactly den's state. h_given: the step's hidden state was supplied by the
    caller (compared bit for bit) instead of the stand-in. narrow: the oracle's
    F8.NarrowE of a narrow-E context (E32 is then its E_deq); the attention is
    the oracle's narrow_attention with the GPU's own row references.
    """
    st0 = den.state()
    if st0["done"]:
        return False
    B = M.canvases(w)
    cst0 = _np(den.read(dg.DG_CANVAS_STATE)).astype(np.int64).reshape(3, B)
    frozen = cst0[1] != 0
    canvas_in = _np(den.read(dg.DG_CANVAS)).astype(np.int64)
    sc_in = _np(den.read(dg.DG_SC)).astype(np.float64)
    target = _np(den.read(dg.DG_TARGET)).astype(np.int64)
    if do_step is None:
        den.step()
    else:
        do_step()
    h = _np(den.read(dg.DG_HIDDEN)).astype(np.float64)
    H = _np(den.read(dg.DG_ENTROPY))
    amax = _np(den.read(dg.DG_ARGMAX)).astype(np.int64)
    sc = _np(den.read(dg.DG_SC)).astype(np.float64)
    out = dict(accept=_np(den.read(dg.DG_ACCEPT)), canvas=_np(den.read(dg.DG_CANVAS)),
               order=_np(den.read(dg.DG_ORDER)), prefix=_np(den.read(dg.DG_PREFIX)))
    multinomial = w.token_rule == dg.DG_TOKEN_MULTINOMIAL
    sampled = _np(den.read(dg.DG_SAMPLED)).astype(np.int64) if multinomial else None
    st1 = den.state()
    out["state"] = st1
    assert st1["status"] == 0
    for peer in peers:
        assert peer.state() == st1
        for k in (dg.DG_HIDDEN, dg.DG_ENTROPY, dg.DG_ARGMAX, dg.DG_SC, dg.DG_CANVAS, dg.DG_ACCEPT,
                  dg.DG_ORDER, dg.DG_PREFIX, dg.DG_CANVAS_STATE, dg.DG_EMIT):
            assert np.array_equal(_np(peer.read(k)), _np(den.read(k))), k
        if multinomial:
            assert np.array_equal(_np(peer.read(dg.DG_SAMPLED)), sampled)
    t, b = st0["t"], st0["block"]
    if h_given is None:
        h_orc = M.standin_hidden(w, E32, target, canvas_in, sc_in, b, t)
        assert h_agreement(w, h, h_orc, standin_terms(w, E32, target, canvas_in, sc_in, h_orc)) < 2e-3
    else:
        assert np.array_equal(h, np.asarray(h_given, np.float64))
    T = M.temperature(t, w.max_steps, w.T_start, w.T_end)
    gkey = (w.seed, b, t) if multinomial else None
    if narrow is not None:
        m_ref = _np(den.read(dg.DG_MREF)).astype(np.float64)
        att, _ = F8.narrow_attention(narrow, h, w.logit_scale / T, canvas_in, canvas_in,
                                     gumbel_key=gkey, m_ref=m_ref)
    elif multinomial:
        att = M.vocab_attention(h, E32, w.logit_scale / T, gumbel_key=gkey)
    else:
        att = M.vocab_attention(h, E32, w.logit_scale / T)
    Cc = w.C // B
    flags = att.margin < 1e-3          # argmax near-ties (frozen canvases included)
    acc_orc = np.zeros(w.C, dtype=bool)
    for c in range(B):
        seg = slice(c * Cc, (c + 1) * Cc)
        if frozen[c]:
            continue
        a_c = M.entropy_bounded_accept(att.H[seg].astype(np.float32), w.tau, w.accept_rule)
        acc_orc[seg] = a_c.accepted
        sub = M.Attention(argmax=att.argmax[seg], H=att.H[seg], sc=att.sc[seg],
                          zmax=att.zmax[seg], margin=att.margin[seg])
        flags[seg] |= near_tie_flags(sub, a_c, w.tau, w.accept_rule)
    compare_attention(tally, att, H, amax, sc, flags)
    if multinomial:
        compare_draw(tally, att, sampled)
        tally.draws_off_mode += int(np.sum(sampled != amax))
    check_sampler_exact(w, b, t, H, amax, canvas_in, out, chosen_gpu=sampled, frozen=frozen)
    mism = np.flatnonzero(acc_orc != out["accept"].astype(bool))
    bad = [int(i) for i in mism if not flags[i]]
    assert not bad, f"accept mismatch off a near-tie at {bad[:8]}"
    tally.tie_mismatch += len(mism)
    tally.positions += w.C
    tally.steps += 1
    # adaptive stop of each running canvas from the same outputs
    cst1 = _np(den.read(dg.DG_CANVAS_STATE)).astype(np.int64).reshape(3, B)
    last = t + 1 >= w.max_steps
    for c in range(B):
        seg = slice(c * Cc, (c + 1) * Cc)
        if frozen[c]:
            assert np.array_equal(cst1[:, c], cst0[:, c])
            continue
        same = np.array_equal(out["canvas"][seg], canvas_in[seg]) if w.stop_rule == 0 else \
            (st0["has_prev"] == 1 and np.array_equal(amax[seg], prev_amax[seg]))
        unchanged = cst0[0, c] + 1 if same else 0
        conf = bool(np.all(H[seg].astype(np.float32) < np.float32(w.stop_entropy)))
        stop = last if w.fixed_steps else (last or conf or unchanged >= w.stop_unchanged)
        assert cst1[0, c] == unchanged and cst1[1, c] == int(stop)
        if stop:
            assert cst1[2, c] == t + 1
    assert st1["unchanged"] == cst1[0, 0] and st1["t"] == t + 1
    assert st1["done"] == int(bool(np.all(cst1[1] != 0)))
    return True


def run_teacher_forced(den, w, E32, max_steps=None, do_step=None, peers=(), narrow=None):
    tally = Tally()
    n = 0
    while max_steps is None or n < max_steps:
        if den.state()["done"]:
            break
        pre = _np(den.read(dg.DG_ARGMAX)).astype(np.int64) if den.state()["has_prev"] else None
        if not step_and_compare(den, w, E32, tally, pre, do_step=do_step, peers=peers,
                                narrow=narrow):
            break
        n += 1
    tally.check_budget()
    return tally


def shard_stepper(shards, bufs, w):
    """One step of a vocabulary-parallel canvas: every shard's partial step, the
    exchange (reduced in-process here; a multi-GPU run does it with NCCL), then
    every shard's finish."""
    def do_step():
        for s, b in zip(shards, bufs):
            s.step_partial(b)
            s.stream.synchronize()
        reduce_partials_local(bufs, w.C, w.d)
        torch.cuda.synchronize()
        for s, b in zip(shards, bufs):
            s.step_finish(b)
            s.stream.synchronize()
    return do_step


# ----------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 512, 256), (128, 4096, 256),
                                   (256, 8192, 512), (128, 16384, 768)])
def test_tc_small_shapes(shape):
    """The tensor-core kernel on small shapes (one range group up to several), 3 steps."""
    C, V, d = shape
    w = synthetic.SMALL.replace(C=C, V=V, d=d, tau=0.5 * C * np.log(2), max_steps=3,
                                fixed_steps=1, coef_target=1.0, coef_canvas=0.5, logit_scale=2.0)
    den, E32 = make(w, dg.DG_IMPL_TC)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps == 3
    assert den.state()["redo"] == 0
    den.close()


def test_tc_reference_too_low_is_recomputed():
    """Hidden states whose best logit far exceeds the per-row reference take the exact fix-up path."""
    w = synthetic.SMALL.replace(C=128, V=8192, d=512, tau=40.0, max_steps=2, fixed_steps=1)
    den, E32 = make(w, dg.DG_IMPL_TC)
    Eg, _ = embedding(w)
    canvas = _np(den.read(dg.DG_CANVAS)).astype(np.int64)
    tok = (canvas * 7 + 3) % w.V
    h = (30.0 * Eg[torch.from_numpy(tok).cuda()].float()).to(torch.bfloat16).contiguous()
    den.step_h(h)
    st = den.state()
    assert st["status"] == 0 and st["redo"] > 0
    att = M.vocab_attention(_np(h).astype(np.float64), E32, w.logit_scale / w.T_start)
    acc = M.entropy_bounded_accept(att.H.astype(np.float32), w.tau, w.accept_rule)
    flags = near_tie_flags(att, acc, w.tau, w.accept_rule)
    tally = Tally()
    compare_attention(tally, att, _np(den.read(dg.DG_ENTROPY)), _np(den.read(dg.DG_ARGMAX)),
                      _np(den.read(dg.DG_SC)).astype(np.float64), flags)
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_tiny_block_trajectory(impl):
    w = synthetic.TINY
    den, E32 = make(w, impl)
    out, steps = den.block(0)
    want, want_steps, _ = M.denoise_block(w, E32, 0)
    assert steps == want_steps
    assert np.array_equal(_np(out), want)
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("variant", ["fixed", "stress", "minus_max", "argmax_stop", "tau0",
                                     "multinomial"])
def test_tiny_teacher_forced(impl, variant):
    base = synthetic.TINY.replace(coef_target=0.5, coef_canvas=0.5, logit_scale=1.5, tau=2.0)
    w = {"fixed": base.replace(fixed_steps=1),
         "stress": base,
         "minus_max": base.replace(accept_rule=1, fixed_steps=1),
         "argmax_stop": base.replace(stop_rule=1),
         "tau0": base.replace(tau=0.0, max_steps=4),
         "multinomial": base.replace(token_rule=1, fixed_steps=1)}[variant]
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps >= 1
    if variant == "multinomial":
        assert tally.draws_off_mode > 0      # a soft distribution does not always give its mode
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("canvases", [2, 4])
def test_batched_canvases_teacher_forced(impl, canvases):
    """Canvases sharing a step: per-canvas sort, acceptance, re-noise and stop."""
    if impl == dg.DG_IMPL_TC:
        base = synthetic.STRESS_PARTIAL.replace(C=256, max_steps=6)
    else:
        base = synthetic.TINY.replace(coef_target=0.5, coef_canvas=0.5, logit_scale=1.5)
    Cc = base.C // canvases
    w = base.replace(canvases=canvases, tau=0.5 * Cc * np.log(2))
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps >= 1
    den.close()


def test_batched_canvases_with_draw_and_shards():
    """Two canvases per step under the multinomial rule, stepped as two
    vocabulary shards: the options compose (per-canvas sampler after the
    cross-shard reduction). Every step is compared with the oracle like a
    whole-vocabulary step (hidden state, entropy, argmax, sc, draw, sort,
    prefix sums, accept mask, canvas, per-canvas stop), and both shards must end
    in the same state bit for bit."""
    w = synthetic.STRESS_PARTIAL.replace(canvases=2, tau=0.5 * 128 * np.log(2), token_rule=1,
                                         max_steps=4, fixed_steps=1)
    Eg, E32 = embedding(w)
    half = w.V // 2
    shards = [dg.Denoiser(w, Eg, impl=dg.DG_IMPL_TC, shard=(0, half)),
              dg.Denoiser(w, Eg, impl=dg.DG_IMPL_TC, shard=(half, half))]
    bufs = [s.partials() for s in shards]
    tally = run_teacher_forced(shards[0], w, E32, do_step=shard_stepper(shards, bufs, w),
                               peers=shards[1:])
    assert tally.steps == w.max_steps and tally.draws_off_mode > 0
    for s in shards:
        s.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_batched_canvases_block(impl):
    """Whole blocks of batched canvases through the graph loop: each canvas's
    prediction at its own stop, and the block's step count, match the oracle."""
    if impl == dg.DG_IMPL_TC:
        w = synthetic.SMALL.replace(canvases=2, tau=0.5 * 128 * np.log(2), max_steps=24)
    else:
        w = synthetic.TINY.replace(canvases=4, tau=0.5 * 4 * np.log(2))
    den, E32 = make(w, impl)
    for b in range(2):
        out, steps = den.block(b)
        want, want_steps, _ = M.denoise_block(w, E32, b)
        assert steps == want_steps
        assert np.array_equal(_np(out), want)
        cst = _np(den.read(dg.DG_CANVAS_STATE)).reshape(3, w.canvases)
        assert np.all(cst[1] == 1)
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_small_multinomial_teacher_forced(impl):
    """Multinomial draws (Gumbel-max) on the partial-acceptance stress set, 4 steps."""
    w = synthetic.STRESS_PARTIAL.replace(token_rule=1, max_steps=4, fixed_steps=1)
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps == 4 and tally.draws_off_mode > 0
    den.close()


def test_full_size_multinomial_step():
    """One headline-size step under the multinomial rule, every row's draw compared."""
    w = synthetic.HEADLINE.replace(token_rule=1, fixed_steps=1)
    den, E32 = make(w, dg.DG_IMPL_TC)
    tally = run_teacher_forced(den, w, E32, max_steps=1)
    assert tally.steps == 1
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("name", ["canvas_c256_v32768_d1024_bf16",
                                  "stress_partial_c256_v32768_d1024_bf16",
                                  "stress_ties_c256_v32768_d1024_bf16"])
def test_small_teacher_forced(impl, name):
    w = synthetic.WORKLOADS[name]
    if name.startswith("stress_ties"):
        w = w.replace(max_steps=4, fixed_steps=1)
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32)
    print(name, impl, tally)
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_small_fixed_steps_sampled(impl):
    """The timing mode (adaptive stop off) over all 16 steps, compared at every step."""
    w = synthetic.SMALL.replace(fixed_steps=1)
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps == w.max_steps
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("name", ["canvas_c256_v262144_d2048_bf16",
                                  "canvas_c128_v262144_d2816_bf16"])
def test_full_size_two_fixed_steps(impl, name):
    """Full-size shapes in the timed configuration: two steps, every row compared."""
    w = synthetic.WORKLOADS[name].replace(fixed_steps=1)
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32, max_steps=2)
    assert tally.steps == 2
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_graph_loop_equals_stepwise(impl):
    w = synthetic.STRESS_PARTIAL
    den, E32 = make(w, impl)
    out, steps = den.block(0)
    g_out = _np(out)
    den.begin_block(0)
    n = 0
    while not den.step(want_done=True):
        n += 1
    n += 1
    assert n == steps
    assert np.array_equal(_np(den.read(dg.DG_ARGMAX)), g_out)
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_block_diffusion_small(impl):
    """Four sequential canvases; each block is independent and emits its final argmax."""
    w = synthetic.SMALL.replace(blocks=4, max_steps=24)
    den, E32 = make(w, impl)
    want, want_steps = M.generate(w, E32)
    got = []
    for b in range(w.blocks):
        out, steps = den.block(b)
        assert steps == want_steps[b]
        got.append(_np(out))
    assert np.array_equal(np.concatenate(got), want)
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
def test_block_diffusion_full_size(impl):
    w = synthetic.BLOCKS
    den, E32 = make(w, impl)
    buf = torch.empty(w.blocks * w.C, dtype=torch.int32, device="cuda")
    steps = []
    for b in range(w.blocks):
        _, s = den.block(b, out=buf[b * w.C:(b + 1) * w.C])
        steps.append(s)
    want, want_steps = M.generate(w, E32)
    assert steps == want_steps
    assert np.array_equal(_np(buf), want)
    den.close()


def _external_h(w, Eg, canvas, seed):
    """A hidden state that is not the stand-in's: row i leans on a random token
    with a strength rising from 0 to 12 along the canvas, plus isotropic noise,
    so the rows range from nearly uniform softmaxes to nearly one-hot ones and
    the canvas token's logit (the tensor-core path's reference) is often far
    below the row's largest logit."""
    g = torch.Generator().manual_seed(seed)
    tok = torch.randint(0, w.V, (w.C,), generator=g)
    lean = torch.linspace(0.0, 12.0, w.C)[:, None]
    noise = torch.randn(w.C, w.d, generator=g) * (0.5 / np.sqrt(w.d))
    h = lean * Eg[tok.cuda()].float().cpu() + noise
    return h.to(torch.bfloat16).contiguous()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("name", ["canvas_c256_v32768_d1024_bf16",
                                  "canvas_c256_v262144_d2048_bf16"])
def test_external_hidden_state_from_host(impl, name):
    """dg_denoise_step_h with a caller's hidden state (not the stand-in) in
    pinned host memory, two steps, against the oracle: entropy, argmax and sc
    of that h, then the sampler (sort, prefix sums, acceptance, re-noise), the
    canvas copied back to pinned host memory, and the stop state."""
    w = synthetic.WORKLOADS[name].replace(fixed_steps=1)
    den, E32 = make(w, impl)
    Eg, _ = embedding(w)
    tally = Tally()
    canvas_host = torch.empty(w.C, dtype=torch.int32).pin_memory()
    for step in range(2):
        canvas = _np(den.read(dg.DG_CANVAS)).astype(np.int64)
        h = _external_h(w, Eg, canvas, 1234 + step).pin_memory()
        pre = _np(den.read(dg.DG_ARGMAX)).astype(np.int64) if den.state()["has_prev"] else None
        do_step = lambda: den.step_h(h, canvas_host=canvas_host)   # noqa: E731
        assert step_and_compare(den, w, E32, tally, pre, do_step=do_step,
                                h_given=h.float().numpy())
        assert np.array_equal(canvas_host.numpy(), _np(den.read(dg.DG_CANVAS)))
    tally.check_budget()
    den.close()


def test_canvas_to_host_buffers():
    """dg_denoise_step_h's canvas_host on the tensor-core path: a pinned buffer
    (written by the merge kernel itself), a pageable one (copied after the
    step), and a fresh pinned one after the block has stopped (the merge
    kernel's early return writes it too) all equal the context's canvas."""
    w = synthetic.SMALL.replace(max_steps=2, fixed_steps=1)
    den, _ = make(w, dg.DG_IMPL_TC)
    Eg, _ = embedding(w)
    for kind in ("pinned", "pageable", "pinned after stop"):
        canvas = _np(den.read(dg.DG_CANVAS)).astype(np.int64)
        h = _external_h(w, Eg, canvas, 99).cuda()
        buf = torch.full((w.C,), -1, dtype=torch.int32)
        if kind != "pageable":
            buf = buf.pin_memory()
        den.step_h(h, canvas_host=buf)
        den.stream.synchronize()
        assert np.array_equal(buf.numpy(), _np(den.read(dg.DG_CANVAS))), kind
    assert den.state()["done"] == 1
    den.close()


def test_full_size_redo_pass():
    """The redo pass at the headline size. Caller hidden states h = 30 E[token]
    put a row's largest logit far above its reference (the logit of its canvas
    token, or of its previous argmax) unless that token is the row's argmax
    already: step 0 overshoots on every row, step 1 (the same tokens except on
    1% of the rows) on those rows only. Both steps are redone by the second
    tensor-core pass and must equal the oracle's step."""
    w = synthetic.HEADLINE.replace(fixed_steps=1, max_steps=4)
    den, E32 = make(w, dg.DG_IMPL_TC)
    Eg, _ = embedding(w)
    g = torch.Generator().manual_seed(11)
    tok_a = torch.randint(0, w.V, (w.C,), generator=g)
    tok_b = tok_a.clone()
    k = max(1, w.C // 100)
    tok_b[:k] = torch.randint(0, w.V, (k,), generator=g)

    def hid(tok):
        return (30.0 * Eg[tok.cuda()].float()).to(torch.bfloat16).contiguous()

    tally = Tally()
    redone = []
    for h in (hid(tok_a), hid(tok_b)):
        r0 = den.state()["redo"]
        pre = _np(den.read(dg.DG_ARGMAX)).astype(np.int64) if den.state()["has_prev"] else None
        assert step_and_compare(den, w, E32, tally, pre, do_step=lambda: den.step_h(h),
                                h_given=_np(h))
        redone.append(den.state()["redo"] - r0)
    assert redone[0] >= w.C - 2, redone      # all rows (bar a canvas token equal to the row's)
    assert redone[1] == k, redone
    tally.check_budget()
    den.close()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("variant", ["minus_max", "argmax_stop", "tau0"])
def test_sampler_rules_teacher_forced(impl, variant):
    """The acceptance and stop options on the 256-position partial-acceptance
    stress set, on both kernel families (the tensor-core path runs the sampler
    at the end of its attention kernel): "sum so far minus the largest" acceptance,
    the argmax-stability stop, and a zero entropy budget (nothing accepted)."""
    base = synthetic.STRESS_PARTIAL
    w = {"minus_max": base.replace(accept_rule=dg.DG_ACCEPT_MINUS_MAX, fixed_steps=1, max_steps=4),
         "argmax_stop": base.replace(stop_rule=dg.DG_STOP_ARGMAX, max_steps=8),
         "tau0": base.replace(tau=0.0, max_steps=3)}[variant]
    den, E32 = make(w, impl)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps >= 2
    if variant == "argmax_stop":
        assert den.state()["done"] == 1
    den.close()


@pytest.mark.parametrize("shape", [(37, 128, 24), (1, 64, 8), (200, 1024, 72), (256, 512, 64)])
def test_ragged_shapes_simt(shape):
    C, V, d = shape
    w = synthetic.TINY.replace(C=C, V=V, d=d, tau=0.5 * C * 0.693, coef_target=1.0,
                               coef_canvas=0.5, logit_scale=2.0, max_steps=5, fixed_steps=1)
    den, E32 = make(w, dg.DG_IMPL_SIMT)
    run_teacher_forced(den, w, E32)
    den.close()


@pytest.mark.parametrize("C,canvases", [(1024, 1), (1024, 64), (64, 64)])
def test_largest_and_single_position_canvases_simt(C, canvases):
    """The most positions a context takes (C = 1024) as one canvas and as the most
    canvases per step (64 of 16 positions), and canvases of one position each:
    sort, acceptance, re-noise and stop over up to 1024 keys."""
    Cc = C // canvases
    w = synthetic.TINY.replace(C=C, V=2048, d=64, canvases=canvases, tau=0.5 * Cc * np.log(2),
                               coef_target=1.0, coef_canvas=0.5, logit_scale=2.0, max_steps=4,
                               fixed_steps=1)
    assert supported(w, dg.DG_IMPL_SIMT)
    den, E32 = make(w, dg.DG_IMPL_SIMT)
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps == w.max_steps
    den.close()


def test_workspace_too_small_is_rejected():
    w = synthetic.TINY
    Eg, _ = embedding(w)
    cfg = dg.make_config(w)
    n = dg.dg_workspace_bytes(cfg)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    with pytest.raises(dg.DgError) as e:
        dg.dg_init(cfg, Eg.data_ptr(), ws.data_ptr(), n - 256, torch.cuda.Stream().cuda_stream)
    assert e.value.code == dg.DG_ENOMEM


def test_device_status_word_is_reported():
    """A status raised on the device (injected from the host) fails the next synchronising call."""
    w = synthetic.TINY
    den, _ = make(w, dg.DG_IMPL_SIMT)
    st = den.read(dg.DG_STATE)
    st[dg.DG_ST_STATUS] = dg.DG_ETIMEOUT
    den.write(dg.DG_STATE, st)
    with pytest.raises(dg.DgError) as e:
        den.step(want_done=True)
    assert e.value.code == dg.DG_ETIMEOUT
    den.close()


@pytest.mark.parametrize("emb_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(256, 32768, 1024, 1024), (200, 4096, 512, 256),
                                   (128, 8192, 2048, 1536)])
def test_self_condition_network(shape, emb_dtype):
    """dg_self_condition: the context's sc after a step goes through the
    two-layer network (tensor cores) and is added to the caller's next-step
    token embeddings; compared with the oracle's network on the same sc,
    weights and embeddings (ragged canvas included: 200 rows)."""
    C, V, d, dff = shape
    w = synthetic.SMALL.replace(C=C, V=V, d=d, tau=0.5 * C * np.log(2), max_steps=2,
                                fixed_steps=1, coef_target=1.0, coef_canvas=0.5, logit_scale=2.0)
    impl = dg.DG_IMPL_TC if C in (128, 256) else dg.DG_IMPL_SIMT
    den, E32 = make(w, impl)
    Eg, _ = embedding(w)
    den.step()
    sc = _np(den.read(dg.DG_SC)).astype(np.float64)
    canvas = _np(den.read(dg.DG_CANVAS)).astype(np.int64)
    g = torch.Generator().manual_seed(11)
    W1 = torch.randn(dff, d, generator=g).to(torch.bfloat16)
    b1 = torch.randn(dff, generator=g) * 0.1
    W2 = (torch.randn(d, dff, generator=g) / np.sqrt(dff)).to(torch.bfloat16)
    b2 = torch.randn(d, generator=g) * 0.1
    tdt = torch.bfloat16 if emb_dtype == "bf16" else torch.float32
    emb0 = Eg[torch.from_numpy(canvas).cuda()].to(tdt).contiguous()
    emb = emb0.clone()
    den.self_condition(W1.cuda(), b1.cuda(), W2.cuda(), b2.cuda(), emb)
    assert den.state()["status"] == 0
    y = M.self_condition_ffnn(sc, W1.float().numpy(), b1.numpy(), W2.float().numpy(), b2.numpy())
    want = M.add_to_embeddings(_np(emb0).astype(np.float64), y, emb_dtype)
    got = _np(emb).astype(np.float64)
    if emb_dtype == "bf16":
        # the sum is rounded to bf16 on both sides; one bf16 ulp of the result,
        # plus the fp32-vs-fp64 accumulation (far below it)
        e = np.frexp(np.maximum(np.abs(want), np.abs(got)))[1]
        tol = np.ldexp(1.0, e - 8) + 1e-4 * np.abs(y).max()
        assert np.all(np.abs(got - want) <= tol), float(np.abs(got - want).max())
    else:
        rel = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
        assert rel.max() < 1e-3, rel.max()
    den.close()


_NARROW = {}


def narrow_embedding(w):
    """The oracle's narrow E (e4m3 codes, per-row exponents) of the workload's E."""
    key = (w.V, w.d, w.e_seed)
    if key not in _NARROW:
        _NARROW.clear()
        _NARROW[key] = F8.NarrowE(embedding(w)[1])
    return _NARROW[key]


SMALL128 = synthetic.SMALL.replace(name="c128_v16384_d768", C=128, V=16384, d=768,
                                   tau=0.5 * 128 * np.log(2), coef_target=1.0, coef_canvas=0.5,
                                   logit_scale=2.0)


@pytest.mark.parametrize("name,steps,token_rule", [
    ("stress_partial_c256_v32768_d1024_bf16", 4, 0),
    ("stress_partial_c256_v32768_d1024_bf16", 2, 1),
    ("c128_v16384_d768", 3, 0),
    ("canvas_c256_v262144_d2048_bf16", 2, 0),
    ("canvas_c128_v262144_d2816_bf16", 2, 0)])
def test_fp8_embedding_teacher_forced(name, steps, token_rule):
    """Narrow E (e4m3 codes with a power-of-two scale per row, h quantised per
    row, probabilities rounded to e5m2 for p.E): every step against the
    oracle's narrow-E attention of the GPU's own hidden state and references,
    on CTA pairs (256 rows) and single CTAs (128 rows), with both token rules."""
    base = SMALL128 if name == "c128_v16384_d768" else synthetic.WORKLOADS[name]
    w = base.replace(e_format=dg.DG_E_FP8, fixed_steps=1, token_rule=token_rule)
    den, _ = make(w, dg.DG_IMPL_TC)
    nE = narrow_embedding(w)
    tally = run_teacher_forced(den, w, nE.E_deq, max_steps=steps, narrow=nE)
    assert tally.steps == steps
    den.close()


def test_fp8_external_hidden_state_from_host():
    """Narrow E with a caller's hidden state from pinned host memory, two
    steps: the narrow-E prologue quantises the caller's h, rows whose largest
    logit overshoots the reference (the redo gap is 4 nats here) take the redo
    pass, and the step equals the oracle's narrow-E step; the canvas reaches
    the caller's pinned buffer."""
    w = synthetic.SMALL.replace(e_format=dg.DG_E_FP8, fixed_steps=1)
    den, _ = make(w, dg.DG_IMPL_TC)
    Eg, _ = embedding(w)
    nE = narrow_embedding(w)
    tally = Tally()
    canvas_host = torch.empty(w.C, dtype=torch.int32).pin_memory()
    for step in range(2):
        canvas = _np(den.read(dg.DG_CANVAS)).astype(np.int64)
        h = _external_h(w, Eg, canvas, 4321 + step).pin_memory()
        pre = _np(den.read(dg.DG_ARGMAX)).astype(np.int64) if den.state()["has_prev"] else None
        do_step = lambda: den.step_h(h, canvas_host=canvas_host)   # noqa: E731
        assert step_and_compare(den, w, nE.E_deq, tally, pre, do_step=do_step,
                                h_given=h.float().numpy(), narrow=nE)
        assert np.array_equal(canvas_host.numpy(), _np(den.read(dg.DG_CANVAS)))
    assert den.state()["redo"] > 0
    tally.check_budget()
    den.close()


def test_fp8_embedding_block_through_the_graph_loop():
    """A whole adaptive block with narrow E through the captured loop: the
    emitted tokens and the step count equal the oracle's narrow-E run (its own
    reference and redo rule)."""
    w = synthetic.SMALL.replace(e_format=dg.DG_E_FP8, max_steps=8)
    den, _ = make(w, dg.DG_IMPL_TC)
    nE = narrow_embedding(w)
    out, steps = den.block(0)
    want, want_steps, recs = M.denoise_block(w, nE.E_deq, 0, narrow=nE)
    assert steps == want_steps
    ties = np.zeros(w.C, dtype=bool)
    for r in recs:
        ties |= r.att.margin < 1e-3
    bad = np.flatnonzero((_np(out) != want) & ~ties)
    assert bad.size == 0, bad[:8]
    den.close()


def test_device_wait_timeout_is_reported_and_recovered():
    """A bounded wait of the attention kernel runs out (a hand-off target that
    no step reaches, with a 20 ms limit): the kernel returns on its own, the
    next synchronising call reports DG_ETIMEOUT, and after dg_begin_block the
    context steps correctly again (checked against the oracle)."""
    import time
    w = synthetic.STRESS_PARTIAL.replace(V=8192, d=512, max_steps=3, fixed_steps=1)
    den, E32 = make(w, dg.DG_IMPL_TC)
    den.step()
    assert den.state()["status"] == 0
    with pytest.raises(dg.DgError):
        dg.dg_inject_stall(den.ctx, -1, 0)
    dg.dg_inject_stall(den.ctx, 20_000_000, 1)
    t0 = time.perf_counter()
    with pytest.raises(dg.DgError) as e:
        den.step(want_done=True)
    waited = time.perf_counter() - t0
    assert e.value.code == dg.DG_ETIMEOUT
    assert waited < 1.5, waited            # well under the default 2 s limit
    assert den.state()["status"] == dg.DG_ETIMEOUT
    dg.dg_inject_stall(den.ctx, 0, 0)
    den.begin_block(0)
    assert den.state()["status"] == 0
    tally = run_teacher_forced(den, w, E32)
    assert tally.steps == w.max_steps
    den.close()


def test_attention_kernel_clock_stamps():
    """Every tensor-core step stamps one CTA's %globaltimer and clock counter at
    its start and end (row 255 of DG_TC_TRACE_COUNTERS): the SM clock the kernel
    ran at comes out between 0.3 and 3 GHz, and the stamps move with each step.
    The timeline stamps of the redo pass and the merge kernel are in causal order."""
    w = synthetic.SMALL.replace(fixed_steps=1)
    den, _ = make(w, dg.DG_IMPL_TC)
    den.step()
    r1 = den.read(dg.DG_TC_TRACE_COUNTERS)[255].cpu().tolist()
    den.step()
    r2 = den.read(dg.DG_TC_TRACE_COUNTERS)[255].cpu().tolist()
    for r in (r1, r2):
        assert r[2] > r[0] and r[3] > r[1]
        ghz = (r[3] - r[1]) / (r[2] - r[0])
        assert 0.3 < ghz < 3.0, ghz
        # the step's timeline: each stamp follows the completion it waits for
        assert r[0] <= r[4] <= r[5] <= r[7] <= r[8] and r[6] <= r[7], r[:10]
    assert r2[0] > r1[2]
    assert r2[9] == r1[8] and r2[9] <= r2[4]        # the previous merge's end, kept
    den.close()


def test_block_loop_needs_a_stream():
    w = synthetic.TINY
    Eg, _ = embedding(w)
    den = dg.Denoiser(w, Eg, stream=torch.cuda.default_stream())
    with pytest.raises(dg.DgError) as e:
        den.block(0)
    assert e.value.code == dg.DG_EINVAL
    den.close()


@pytest.mark.parametrize("token_rule", [0, 1])
def test_vocab_parallel_shards(token_rule):
    """Two vocabulary shards, run one after the other on this GPU and reduced
    in-process (the exchange a multi-GPU run does with NCCL), give the step of
    the whole vocabulary: every shard ends in the same state, matching the
    oracle within the usual tolerances (only summation order differs)."""
    w = synthetic.STRESS_PARTIAL.replace(max_steps=4, fixed_steps=1, token_rule=token_rule)
    Eg, E32 = embedding(w)
    half = w.V // 2
    shards = [dg.Denoiser(w, Eg, impl=dg.DG_IMPL_TC, shard=(0, half)),
              dg.Denoiser(w, Eg, impl=dg.DG_IMPL_TC, shard=(half, half))]
    with pytest.raises(dg.DgError):
        shards[0].step()                          # a shard alone cannot run a whole step
    bufs = [s.partials() for s in shards]
    tally = run_teacher_forced(shards[0], w, E32, do_step=shard_stepper(shards, bufs, w),
                               peers=shards[1:])
    assert tally.steps == w.max_steps
    assert shards[0].state()["done"] == 1
    for s in shards:
        s.close()

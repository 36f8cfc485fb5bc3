"""Python binding of the denoise-step C ABI declared in include/dg.h.

Argument marshalling only: every step of the path runs in libdg.so's CUDA
kernels. The functions keep the C names (dg_init, dg_denoise_step, ...), take
raw pointers as Python ints, and raise DgError on a non-zero return code.
`Denoiser` is a convenience owner of the device buffers (allocated with torch,
which here only provides memory and streams).

The library must be built first (uniform_state_text_b200.build.build(), nvcc
for sm_100a); without it every call raises, there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# DG_LIBRARY selects another build of the same library (e.g. an instrumented one).
LIB_PATH = os.environ.get("DG_LIBRARY") or os.path.join(HERE, "libdg.so")

DG_OK, DG_EINVAL, DG_ENOMEM, DG_ECUDA, DG_ETIMEOUT, DG_EUNSUPPORTED, DG_ESTATE = 0, -1, -2, -3, -4, -5, -6
DG_F32, DG_BF16 = 0, 1
DG_STOP_CANVAS, DG_STOP_ARGMAX = 0, 1
DG_ACCEPT_CUMSUM, DG_ACCEPT_MINUS_MAX = 0, 1
DG_IMPL_AUTO, DG_IMPL_SIMT, DG_IMPL_TC = 0, 1, 2
DG_TOKEN_ARGMAX, DG_TOKEN_MULTINOMIAL = 0, 1
DG_E_NATIVE, DG_E_FP8 = 0, 1
(DG_CANVAS, DG_ARGMAX, DG_ENTROPY, DG_ACCEPT, DG_SC, DG_HIDDEN, DG_TARGET, DG_ORDER, DG_PREFIX,
 DG_STATE, DG_MREF, DG_SAMPLED, DG_EMIT, DG_CANVAS_STATE, DG_TC_TRACE_COUNTERS) = range(15)
DG_ST_T, DG_ST_BLOCK, DG_ST_UNCHANGED, DG_ST_DONE, DG_ST_STEPS, DG_ST_K, DG_ST_STATUS, \
    DG_ST_HASPREV, DG_ST_REDO = range(9)


class dg_config(ctypes.Structure):
    _fields_ = [
        ("C", ctypes.c_int32), ("V", ctypes.c_int32), ("d", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("max_steps", ctypes.c_int32),
        ("T_start", ctypes.c_float), ("T_end", ctypes.c_float), ("tau", ctypes.c_float),
        ("logit_scale", ctypes.c_float), ("coef_target", ctypes.c_float),
        ("coef_canvas", ctypes.c_float), ("noise_var_d", ctypes.c_float),
        ("stop_entropy", ctypes.c_float), ("stop_unchanged", ctypes.c_int32),
        ("stop_rule", ctypes.c_int32), ("accept_rule", ctypes.c_int32),
        ("fixed_steps", ctypes.c_int32), ("impl", ctypes.c_int32), ("token_rule", ctypes.c_int32),
        ("canvases", ctypes.c_int32),
        ("seed", ctypes.c_uint64),
        ("shard_v0", ctypes.c_int32), ("shard_nv", ctypes.c_int32),
        ("e_format", ctypes.c_int32),
    ]


class DgError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"dg error {code}: {msg}")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32


def lib():
    """Load libdg.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "uniform_state_text_b200.build.build() (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    cfgp = ctypes.POINTER(dg_config)
    L.dg_workspace_bytes.argtypes = [cfgp]
    L.dg_workspace_bytes.restype = ctypes.c_size_t
    L.dg_init.argtypes = [cfgp, _P, _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]
    L.dg_begin_block.argtypes = [_P, _I]
    L.dg_denoise_step.argtypes = [_P, ctypes.POINTER(_I)]
    L.dg_denoise_step_h.argtypes = [_P, _P, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]
    L.dg_denoise_block.argtypes = [_P, _I, _P, ctypes.POINTER(_I)]
    L.dg_read.argtypes = [_P, _I, _P]
    L.dg_write.argtypes = [_P, _I, _P]
    L.dg_profile.argtypes = [_P, _I]
    L.dg_profile_read.argtypes = [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I),
                                  ctypes.POINTER(ctypes.c_int64)]
    L.dg_impl.argtypes = [_P]
    L.dg_inject_stall.argtypes = [_P, ctypes.c_int64, _I]
    L.dg_self_condition_scratch_bytes.argtypes = [cfgp, _I]
    L.dg_self_condition_scratch_bytes.restype = ctypes.c_size_t
    L.dg_self_condition.argtypes = [_P, _I, _P, _P, _P, _P, _P, _I, _P]
    L.dg_vocab_attention_static.argtypes = [_I, _I, _I, _I, ctypes.c_float, _P, _P, _P, _P, _P, _P]
    L.dg_partials_bytes.argtypes = [cfgp]
    L.dg_partials_bytes.restype = ctypes.c_size_t
    L.dg_denoise_step_partial.argtypes = [_P, _P]
    L.dg_denoise_step_finish.argtypes = [_P, _P]
    L.dg_tc_schedule.argtypes = [_I, _I, _I, _I, _P, _I]
    L.dg_free.argtypes = [_P]
    L.dg_last_error.argtypes = [_P]
    L.dg_last_error.restype = ctypes.c_char_p
    for name in ("dg_init", "dg_begin_block", "dg_denoise_step", "dg_denoise_step_h",
                 "dg_denoise_block", "dg_read", "dg_write", "dg_profile", "dg_profile_read",
                 "dg_impl", "dg_free", "dg_vocab_attention_static", "dg_denoise_step_partial",
                 "dg_denoise_step_finish", "dg_tc_schedule", "dg_inject_stall",
                 "dg_self_condition"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(rc: int, ctx) -> int:
    if rc < 0:
        raise DgError(rc, dg_last_error(ctx))
    return rc


def make_config(w, impl: int = DG_IMPL_AUTO, shard=None) -> dg_config:
    """dg_config from a synthetic.Workload-like object (same field names).

    shard = (v0, nv): a context for vocabulary entries [v0, v0 + nv) of a
    vocabulary-parallel step.
    """
    v0, nv = shard if shard is not None else (0, 0)
    return dg_config(C=w.C, V=w.V, d=w.d, dtype=DG_BF16 if w.dtype == "bf16" else DG_F32,
                     max_steps=w.max_steps, T_start=w.T_start, T_end=w.T_end, tau=w.tau,
                     logit_scale=w.logit_scale, coef_target=w.coef_target,
                     coef_canvas=w.coef_canvas, noise_var_d=w.noise_var_d,
                     stop_entropy=w.stop_entropy, stop_unchanged=w.stop_unchanged,
                     stop_rule=w.stop_rule, accept_rule=w.accept_rule,
                     fixed_steps=w.fixed_steps, impl=impl,
                     token_rule=getattr(w, "token_rule", 0),
                     canvases=getattr(w, "canvases", 1), seed=w.seed,
                     shard_v0=v0, shard_nv=nv, e_format=getattr(w, "e_format", 0))


# ----------------------------------------------------------------------------
# The C ABI, same names.
# ----------------------------------------------------------------------------
def dg_workspace_bytes(cfg: dg_config) -> int:
    return int(lib().dg_workspace_bytes(ctypes.byref(cfg)))


def dg_init(cfg: dg_config, E_ptr: int, ws_ptr: int, ws_bytes: int, stream_ptr: int):
    out = _P()
    rc = lib().dg_init(ctypes.byref(cfg), _P(E_ptr), _P(ws_ptr), ws_bytes, _P(stream_ptr),
                       ctypes.byref(out))
    _check(rc, None)
    return out


def dg_begin_block(ctx, block: int) -> None:
    _check(lib().dg_begin_block(ctx, block), ctx)


def dg_denoise_step(ctx, want_done: bool = False):
    if not want_done:
        _check(lib().dg_denoise_step(ctx, None), ctx)
        return None
    done = _I()
    _check(lib().dg_denoise_step(ctx, ctypes.byref(done)), ctx)
    return int(done.value)


def dg_denoise_step_h(ctx, h_ptr: int, on_host: bool, canvas_host_ptr: int | None = None,
                      want_done: bool = False):
    done = _I()
    cptr = ctypes.cast(canvas_host_ptr, ctypes.POINTER(_I)) if canvas_host_ptr else None
    _check(lib().dg_denoise_step_h(ctx, _P(h_ptr), 1 if on_host else 0, cptr,
                                   ctypes.byref(done) if want_done else None), ctx)
    return int(done.value) if want_done else None


def dg_denoise_block(ctx, block: int, out_ptr: int, want_steps: bool = True):
    steps = _I()
    _check(lib().dg_denoise_block(ctx, block, _P(out_ptr),
                                  ctypes.byref(steps) if want_steps else None), ctx)
    return int(steps.value) if want_steps else None


def dg_read(ctx, what: int, dst_ptr: int) -> None:
    _check(lib().dg_read(ctx, what, _P(dst_ptr)), ctx)


def dg_write(ctx, what: int, src_ptr: int) -> None:
    _check(lib().dg_write(ctx, what, _P(src_ptr)), ctx)


def dg_profile(ctx, enable: bool) -> None:
    _check(lib().dg_profile(ctx, 1 if enable else 0), ctx)


def dg_profile_read(ctx):
    """(milliseconds in the vocabulary-attention kernels, steps timed, kernels launched)."""
    ms = ctypes.c_double()
    n = _I()
    nl = ctypes.c_int64()
    _check(lib().dg_profile_read(ctx, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(nl)), ctx)
    return float(ms.value), int(n.value), int(nl.value)


def dg_vocab_attention_static(C: int, V: int, d: int, dtype: int, scale: float, E_ptr: int,
                              h_ptr: int, H_ptr: int, argmax_ptr: int, sc_ptr: int,
                              stream_ptr: int) -> None:
    """Vocabulary attention with the library's static scratch (no allocation)."""
    _check(lib().dg_vocab_attention_static(C, V, d, dtype, scale, _P(E_ptr), _P(h_ptr), _P(H_ptr),
                                           _P(argmax_ptr), _P(sc_ptr), _P(stream_ptr)), None)


def dg_partials_bytes(cfg: dg_config) -> int:
    return int(lib().dg_partials_bytes(ctypes.byref(cfg)))


def dg_denoise_step_partial(ctx, partials_ptr: int) -> None:
    _check(lib().dg_denoise_step_partial(ctx, _P(partials_ptr)), ctx)


def dg_denoise_step_finish(ctx, partials_ptr: int) -> None:
    _check(lib().dg_denoise_step_finish(ctx, _P(partials_ptr)), ctx)


def dg_impl(ctx) -> int:
    return _check(lib().dg_impl(ctx), ctx)


def dg_self_condition_scratch_bytes(cfg: dg_config, d_ff: int) -> int:
    return int(lib().dg_self_condition_scratch_bytes(ctypes.byref(cfg), d_ff))


def dg_self_condition(ctx, d_ff: int, W1_ptr: int, b1_ptr: int, W2_ptr: int, b2_ptr: int,
                      emb_ptr: int, emb_dtype: int, scratch_ptr: int) -> None:
    """emb += W2 gelu(W1 sc + b1) + b2 on the context's stream (see include/dg.h)."""
    _check(lib().dg_self_condition(ctx, d_ff, _P(W1_ptr), _P(b1_ptr), _P(W2_ptr), _P(b2_ptr),
                                   _P(emb_ptr), emb_dtype, _P(scratch_ptr)), ctx)


def dg_inject_stall(ctx, wait_limit_ns: int, stall: int) -> None:
    """Failure-path testing: limit every bounded wait and make the hand-off unreachable."""
    _check(lib().dg_inject_stall(ctx, int(wait_limit_ns), int(stall)), ctx)


TC_SCHEDULE_FIELDS = ("CG", "W2", "RB", "n_vt", "n_ranges", "n_dt", "G", "n1", "n2", "ring",
                      "ctas")


def dg_tc_schedule(C: int, V: int, d: int, sms: int = 148) -> dict:
    """The tensor-core kernel's work split for a shape (host only; see include/dg.h)."""
    out = (ctypes.c_int32 * len(TC_SCHEDULE_FIELDS))()
    n = _check(lib().dg_tc_schedule(C, V, d, sms, ctypes.cast(out, ctypes.c_void_p),
                                    len(TC_SCHEDULE_FIELDS)), None)
    return dict(zip(TC_SCHEDULE_FIELDS, list(out)[:n]))


def dg_free(ctx) -> None:
    lib().dg_free(ctx)


def dg_last_error(ctx) -> str:
    msg = lib().dg_last_error(ctx)
    return msg.decode() if msg else ""


# ----------------------------------------------------------------------------
# Convenience owner of device buffers.
# ----------------------------------------------------------------------------
class Denoiser:
    """One context with its workspace; E must be a CUDA tensor [V, d] of the workload dtype."""

    def __init__(self, w, E, stream=None, impl: int = DG_IMPL_AUTO, shard=None):
        import torch

        self.w = w
        self.cfg = make_config(w, impl, shard)
        if not E.is_cuda or not E.is_contiguous():
            raise ValueError("E must be a contiguous CUDA tensor")
        self.E = E
        self.device = E.device
        self.stream = stream if stream is not None else torch.cuda.Stream(device=self.device)
        nbytes = dg_workspace_bytes(self.cfg)
        if nbytes == 0:
            raise DgError(DG_EINVAL, "invalid configuration: " + dg_last_error(None))
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.ctx = dg_init(self.cfg, E.data_ptr(), self.ws.data_ptr(), nbytes,
                           self.stream.cuda_stream)
        self.impl = dg_impl(self.ctx)
        self._dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    # state -----------------------------------------------------------------
    def _shape(self, what):
        import torch

        C, d = self.w.C, self.w.d
        return {DG_CANVAS: ((C,), torch.int32), DG_ARGMAX: ((C,), torch.int32),
                DG_ENTROPY: ((C,), torch.float32), DG_ACCEPT: ((C,), torch.int32),
                DG_SC: ((C, d), torch.float32), DG_HIDDEN: ((C, d), self._dtype),
                DG_TARGET: ((C,), torch.int32), DG_ORDER: ((C,), torch.int32),
                DG_PREFIX: ((C,), torch.float32), DG_STATE: ((16,), torch.int32),
                DG_MREF: ((C,), torch.float32), DG_SAMPLED: ((C,), torch.int32),
                DG_EMIT: ((C,), torch.int32),
                DG_CANVAS_STATE: ((3 * getattr(self.w, "canvases", 1),), torch.int32),
                DG_TC_TRACE_COUNTERS: ((256, 32), torch.int64)}[what]

    def read(self, what):
        import torch

        shape, dt = self._shape(what)
        out = torch.empty(shape, dtype=dt, device=self.device)
        dg_read(self.ctx, what, out.data_ptr())
        self.stream.synchronize()
        return out

    def write(self, what, tensor):
        shape, dt = self._shape(what)
        t = tensor.to(device=self.device, dtype=dt).contiguous()
        if tuple(t.shape) != shape:
            raise ValueError(f"expected shape {shape}")
        dg_write(self.ctx, what, t.data_ptr())
        self.stream.synchronize()

    def state(self) -> dict:
        s = self.read(DG_STATE).cpu().tolist()
        return dict(t=s[DG_ST_T], block=s[DG_ST_BLOCK], unchanged=s[DG_ST_UNCHANGED],
                    done=s[DG_ST_DONE], steps=s[DG_ST_STEPS], k=s[DG_ST_K],
                    status=s[DG_ST_STATUS], has_prev=s[DG_ST_HASPREV], redo=s[DG_ST_REDO])

    # loop ------------------------------------------------------------------
    def begin_block(self, block: int) -> None:
        dg_begin_block(self.ctx, block)

    def step(self, want_done: bool = False):
        return dg_denoise_step(self.ctx, want_done)

    def step_h(self, h, canvas_host=None, want_done: bool = False):
        on_host = not h.is_cuda
        return dg_denoise_step_h(self.ctx, h.data_ptr(), on_host,
                                 canvas_host.data_ptr() if canvas_host is not None else None,
                                 want_done)

    def block(self, block: int, out=None):
        import torch

        if out is None:
            out = torch.empty(self.w.C, dtype=torch.int32, device=self.device)
        steps = dg_denoise_block(self.ctx, block, out.data_ptr())
        return out, steps

    # vocabulary-parallel step --------------------------------------------------
    def partials(self):
        """A partials buffer for step_partial / step_finish (see dg_partials_bytes)."""
        import torch

        n = dg_partials_bytes(self.cfg)
        if n == 0:
            raise DgError(DG_EUNSUPPORTED, "no vocabulary-parallel step for this configuration")
        return torch.zeros(n // 8, dtype=torch.int64, device=self.device)

    def step_partial(self, buf) -> None:
        dg_denoise_step_partial(self.ctx, buf.data_ptr())

    def step_finish(self, buf) -> None:
        dg_denoise_step_finish(self.ctx, buf.data_ptr())

    # self-conditioning network ----------------------------------------------
    def self_condition(self, W1, b1, W2, b2, emb):
        """emb += W2 gelu(W1 sc + b1) + b2 with this context's sc (in place on emb).

        W1 [d_ff, d] and W2 [d, d_ff] bf16, b1 [d_ff] and b2 [d] fp32, emb [C, d]
        fp32 or bf16, all contiguous CUDA tensors; scratch is allocated here.
        """
        import torch

        d_ff = W1.shape[0]
        n = dg_self_condition_scratch_bytes(self.cfg, d_ff)
        if n == 0:
            raise DgError(DG_EUNSUPPORTED, "d and d_ff must be multiples of 128")
        scratch = torch.empty(n, dtype=torch.uint8, device=self.device)
        dg_self_condition(self.ctx, d_ff, W1.data_ptr(), b1.data_ptr(), W2.data_ptr(),
                          b2.data_ptr(), emb.data_ptr(),
                          DG_BF16 if emb.dtype == torch.bfloat16 else DG_F32, scratch.data_ptr())
        self.stream.synchronize()
        return emb

    def close(self) -> None:
        if getattr(self, "ctx", None) is not None:
            self.stream.synchronize()
            dg_free(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------------------
# Cross-shard reduction of the partials (torch only as plumbing: views and
# collectives on the caller's buffers).
# ----------------------------------------------------------------------------
def partials_views(buf, C: int, d: int):
    """(float view summed over shards, int64 view max-reduced over shards)."""
    import torch

    nf = 2 * C + C * d
    b = buf.view(torch.uint8)
    fsum = b[:4 * nf].view(torch.float32)
    keys = b[4 * nf:4 * nf + 16 * C].view(torch.int64)
    return fsum, keys


def allreduce_partials(buf, C: int, d: int, group=None) -> None:
    """Reduce one rank's partials with every other rank's (torch.distributed)."""
    import torch.distributed as dist

    fsum, keys = partials_views(buf, C, d)
    dist.all_reduce(fsum, op=dist.ReduceOp.SUM, group=group)
    # the keys are unsigned; flipping the top bit makes signed order agree
    keys.bitwise_xor_(-(1 << 63))
    dist.all_reduce(keys, op=dist.ReduceOp.MAX, group=group)
    keys.bitwise_xor_(-(1 << 63))

"""Seeded synthetic inputs shared by the CUDA path and the CPU oracle.

This module holds workload definitions (shapes, coefficients, schedules) and
the generator of the tied vocabulary embedding E. It holds none of the
method's arithmetic: the denoise step, the temperature schedule, the sampler
and the counter-based hash each live separately in the oracle and in the CUDA
library.

The pages (DiffusionGemma explained; A Visual Guide to DiffusionGemma) name no
dataset or benchmark for the step. The workloads below are synthetic stand-ins
with the canvas sizes the pages use: a 256-token canvas (A Visual Guide to
DiffusionGemma, section 5.2 "multi-canvas sampling") and a 128-token canvas for
the latency-sensitive row of the tuning table in the local-deploy workshop page
("tuning suggestions").

E ~ N(0, I/d) is drawn with numpy's PCG64 in independent row chunks (one
generator per chunk, seeded with (seed, chunk)), so the result does not depend
on the number of threads used to draw it. bf16 workloads round E to bf16 with
round-to-nearest-even (torch's conversion); both the CUDA path and the oracle
receive exactly those values.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

F32 = "f32"
BF16 = "bf16"

_CHUNK_ROWS = 4096


@dataclasses.dataclass(frozen=True)
class Workload:
    """One denoise workload. Field names follow the pages' notation.

    C: canvas positions, V: vocabulary size, d: hidden width.
    max_steps: S, the step budget (A Visual Guide to DiffusionGemma, 5.3).
    T_start/T_end: ends of the cosine logits-temperature schedule (5.3).
    tau: entropy bound of the entropy-bounded sampler, in nats (5.4).
    logit_scale: L in z = L * h.E^T / T (stand-in scale).
    coef_target/coef_canvas: A and B of the stand-in hidden state.
    noise_var_d: noise variance times d (variance = noise_var_d / d).
    stop_entropy / stop_unchanged: adaptive-stop thresholds (5.3).
    blocks: number of sequential canvases (multi-canvas sampling, 5.2).
    """

    name: str
    C: int
    V: int
    d: int
    dtype: str
    max_steps: int
    T_start: float
    T_end: float
    tau: float
    logit_scale: float = 8.0
    coef_target: float = 6.0
    coef_canvas: float = 2.0
    noise_var_d: float = 0.25
    stop_entropy: float = 0.005
    stop_unchanged: int = 3
    stop_rule: int = 0      # 0: canvas unchanged, 1: argmax unchanged
    accept_rule: int = 0    # 0: cumulative sum, 1: cumulative sum minus max
    token_rule: int = 0     # 0: argmax, 1: multinomial draw (Gumbel-max)
    canvases: int = 1       # independent canvases of C / canvases positions per step
    e_format: int = 0       # 0: E as dtype; 1: e4m3 codes, a power-of-two scale per 256 rows
    fixed_steps: int = 0    # 1: run exactly max_steps (timing mode)
    seed: int = 0
    blocks: int = 1
    e_seed: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def e_bytes(self) -> int:
        return self.V * self.d * (4 if self.dtype == F32 else 2)


def _tau(C: int, frac: float) -> float:
    return frac * C * math.log(2.0)


# The five workloads: a tiny fp32 check, a small bf16 canvas, the headline
# 256/262144/2048 canvas, a latency-sensitive 128-token canvas, and four
# sequential 256-token blocks.
TINY = Workload("tiny_c16_v512_d64_f32", 16, 512, 64, F32, 8, 1.0, 0.1, _tau(16, 0.5))
SMALL = Workload("canvas_c256_v32768_d1024_bf16", 256, 32768, 1024, BF16, 16, 1.0, 0.1,
                 _tau(256, 0.5))
HEADLINE = Workload("canvas_c256_v262144_d2048_bf16", 256, 262144, 2048, BF16, 32, 1.0, 0.1,
                    _tau(256, 0.5))
LATENCY = Workload("canvas_c128_v262144_d2816_bf16", 128, 262144, 2816, BF16, 16, 1.5, 0.05,
                   _tau(128, 0.25))
BLOCKS = Workload("blocks4_c256_v262144_d2048_bf16", 256, 262144, 2048, BF16, 64, 1.0, 0.1,
                  _tau(256, 0.5), blocks=4)

# Stress coefficient sets at the small canvas's shapes: weaker signal so that
# rejection, re-noising and near-ties actually occur.
STRESS_PARTIAL = SMALL.replace(name="stress_partial_c256_v32768_d1024_bf16",
                               coef_target=1.0, coef_canvas=0.5, logit_scale=2.0)
STRESS_TIES = SMALL.replace(name="stress_ties_c256_v32768_d1024_bf16",
                            coef_target=0.5, coef_canvas=0.5, logit_scale=1.0)

# Headline shapes with a quarter of the vocabulary (E = 268 MB, still larger than
# L2): small enough for a multi-pass profiler capture of one step.
PROFILE = HEADLINE.replace(name="profile_c256_v65536_d2048_bf16", V=65536)

# Batched canvases: two independent 128-token canvases per step at the headline
# vocabulary and width, and one 128-token canvas alone for comparison.
BATCHED = HEADLINE.replace(name="batched2x128_v262144_d2048_bf16", canvases=2,
                           tau=_tau(128, 0.5))
SINGLE128 = HEADLINE.replace(name="canvas_c128_v262144_d2048_bf16", C=128, tau=_tau(128, 0.5))

WORKLOADS = {w.name: w for w in (TINY, SMALL, HEADLINE, LATENCY, BLOCKS,
                                 STRESS_PARTIAL, STRESS_TIES, PROFILE, BATCHED, SINGLE128)}


def _chunk(args):
    seed, idx, rows, d = args
    g = np.random.default_rng([seed, idx])
    return g.standard_normal((rows, d), dtype=np.float32)


def make_embedding_f32(V: int, d: int, seed: int = 0, threads: int | None = None) -> np.ndarray:
    """E ~ N(0, I/d) as float32 [V, d], row-major (before any bf16 rounding)."""
    out = np.empty((V, d), dtype=np.float32)
    jobs = []
    for idx, r0 in enumerate(range(0, V, _CHUNK_ROWS)):
        jobs.append((seed, idx, min(_CHUNK_ROWS, V - r0), d))
    threads = threads or min(32, len(os.sched_getaffinity(0)))
    scale = np.float32(1.0 / math.sqrt(d))
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for idx, block in enumerate(ex.map(_chunk, jobs)):
            r0 = idx * _CHUNK_ROWS
            np.multiply(block, scale, out=out[r0:r0 + block.shape[0]])
    return out


def make_embedding(w: Workload, device: str = "cpu"):
    """E for workload w as a torch tensor in the workload's dtype.

    bf16 workloads are rounded with torch's round-to-nearest-even conversion.
    """
    import torch

    e = torch.from_numpy(make_embedding_f32(w.V, w.d, w.e_seed))
    if w.dtype == BF16:
        e = e.to(torch.bfloat16)
    return e.to(device) if device != "cpu" else e


def embedding_as_f32(e) -> np.ndarray:
    """Exact float32 view of E's values (bf16 widens exactly), for the oracle."""
    import torch

    return e.detach().to("cpu").to(torch.float32).numpy()

#!/usr/bin/env python
"""Benchmark of the denoise step: steps/s and canvas tokens/s, roofline fraction.

One bench "step" is one denoise step of the whole hot path (stand-in hidden
state, vocabulary attention, entropy sort, acceptance, re-noise, stop test) on
the headline canvas C=256, V=262144, d=2048 (bf16 E, fp32 accumulation), in
the fixed-step timing mode (adaptive stop off; each block runs its S=32 steps
and the next block starts). E (1.07 GB) is larger than L2 and is streamed from
HBM every step, so no L2 flush is needed between steps.

The JSON line (rank 0) carries:
  value     device-timed throughput with inputs resident (CUDA events around K
            steps on the context's stream, max over ranks; no event inside a
            step, where one would end the kernels' programmatic dependent
            launches).
  e2e       the same metric through dg_denoise_step_h with host buffers: every
            step copies its hidden state from pinned host memory (on the
            library's copy stream, overlapping the step before) and the updated
            canvas back to pinned host memory; host wall clock around K steps
            with a synchronisation on both sides.
  roofline  the vocabulary-attention kernel (the dominant kernel) against the
            tensor roofline: 4*C*d*V flops per step over its event-timed
            duration (events around its launches in a second run of the same
            K steps). The peak is the measured burst bf16 figure when the timed
            region is short (under 2 s), the sustained one otherwise; both
            fractions, the region's length and the sampled clock are given.
  step_timeline_us  the last timed step's kernel boundaries from in-kernel
            %globaltimer stamps, after the previous step's merge ended.
  cpu_baseline  the CPU oracle (fp64 numpy) on whole steps of the workload.
  workloads the other configurations: the tiny fp32 check (latency), the small
            and latency-sensitive canvases (throughput and roofline), and four
            sequential headline blocks to their adaptive stop (end-to-end
            tokens/s over all 1024 tokens, emitted tokens copied to the host).

--impl reference runs the CPU oracle as the reference arm (whole steps).
Multi-GPU (torchrun): by default independent canvases per rank (replicas, seed
= rank), no collective on the data path; value sums all ranks' steps over the
slowest rank's time. --parallel vocab instead splits one canvas's vocabulary
over the ranks (dg_denoise_step_partial, an NCCL exchange of the partial row
results, dg_denoise_step_finish): value is that canvas's steps/s.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "denoise steps/s & canvas tok/s at C=256,V=262k,d=2048; % of step roofline"
BURST_MAX_S = 2.0          # timed regions shorter than this are burst measurements


def measured_peaks():
    """Peaks from MEASURED_PEAKS.json (HBM GB/s, bf16 TFLOP/s burst and sustained).

    Also returns any clock figures the file records (keys naming MHz), which
    the roofline uses to state the clock its peaks were taken at.
    """
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        clocks = {}

        def walk(obj, pre=""):
            if isinstance(obj, dict):
                for k, v in obj.items():
                    walk(v, f"{pre}{k}.")
            elif isinstance(obj, (int, float)) and "mhz" in pre.lower():
                clocks[pre[:-1]] = float(obj)
        walk(p)
        return dict(hbm=float(p["hbm_gbs"]), tflops=float(p["bf16_tflops"]),
                    tflops_sustained=float(p["bf16_tflops_sustained"]), src="measured",
                    clocks=clocks)
    except Exception:
        return dict(hbm=6650.0, tflops=1590.0, tflops_sustained=1400.0, src="fallback",
                    clocks={})


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_threads() -> int:
    return int(os.environ.get("OPENBLAS_NUM_THREADS", len(os.sched_getaffinity(0))))


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(w, E32, steps: int = 1, budget_s: float | None = None):
    """The oracle, as it stands, on whole denoise steps of workload w.

    Runs one untimed step first (it pages E in and warms the BLAS threads),
    then `steps` timed steps (fewer if budget_s runs out after at least one).
    Returns the line's cpu_baseline object plus the seconds per step.
    """
    from oracle import method as M

    st = M.begin_block(w, 0)
    M.step(w, E32, st)
    times = []
    t_start = time.perf_counter()
    for _ in range(steps):
        if st.done:
            st = M.begin_block(w, st.block + 1)
        t0 = time.perf_counter()
        M.step(w, E32, st)
        times.append(time.perf_counter() - t0)
        if budget_s is not None and time.perf_counter() - t_start > budget_s:
            break
    step_s = float(np.mean(times))
    return {"value": 1.0 / step_s, "unit": "steps/s", "cores": cpu_threads(), "kind": "oracle",
            "cpu_model": cpu_model(), "steps_timed": len(times),
            "sample": f"{len(times)} whole step(s) of all {w.C} canvas rows (fp64 numpy oracle: "
                      f"stand-in h, vocabulary attention, sampler, stop test), "
                      f"{step_s:.2f} s per step, after one untimed step",
            "tok_per_s": w.C / step_s}, step_s


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(steps_per_rank: int, world: int, slowest_ms: float) -> float:
    """Weak scaling: every rank runs its own canvases; units of all ranks over the slowest rank's time."""
    return steps_per_rank * world / (slowest_ms / 1e3)


def shared_canvas_rate(steps: int, slowest_ms: float) -> float:
    """Strong scaling: all ranks step one canvas together; its steps over the slowest rank's time."""
    return steps / (slowest_ms / 1e3)


def step_roofline(w, pk):
    """Roofline time of one step as the workload's definition states it:
    max(4 C d V / P_bf16, 2 V d 2 / B_HBM), burst and sustained."""
    flops = 4.0 * w.C * w.d * w.V
    t_m = 2.0 * w.V * w.d * 2 / (pk["hbm"] * 1e9)
    return (max(flops / (pk["tflops"] * 1e12), t_m),
            max(flops / (pk["tflops_sustained"] * 1e12), t_m), flops)


def choose_peak(timed_s: float, clk) -> str:
    """'burst' for a timed region shorter than BURST_MAX_S, else 'sustained'.

    A region of a few milliseconds ends before the power cap acts on the clock
    (and nvidia-smi's 200 ms samples then mostly see the idle GPU around it),
    so its length decides; the sampled clock is reported beside the result.
    """
    return "burst" if timed_s < BURST_MAX_S else "sustained"


def kernel_roofline(w, pk, kernel_s: float, timed_s: float, clk, kernel: str, timeline=None):
    """Roofline object of the vocabulary-attention kernel at one launch per step.

    Algorithmic work per launch: 4 C d V flops (both contractions) and V d b_E
    bytes of E (read once). The bound is whichever takes longer at the peaks.
    With narrow E (e4m3 codes) the operands are 8-bit: E is V d bytes plus a
    4-byte exponent per row (one per 256-row block, stored per row), and the tensor peak is the measured bf16 peak
    times the nominal fp8/bf16 ratio (4.5 / 2.25 PFLOP/s dense).
    """
    fp8 = getattr(w, "e_format", 0) == 1
    esz = 1 if fp8 else (2 if w.dtype == "bf16" else 4)
    flops = 4.0 * w.C * w.d * w.V
    bytes_ = float(w.V) * w.d * esz + (4.0 * w.V if fp8 else 0.0) + w.C * w.d * (esz + 4)
    which = choose_peak(timed_s, clk)
    ratio = 2.0 if fp8 else 1.0
    P = ratio * (pk["tflops"] if which == "burst" else pk["tflops_sustained"])
    tensor_bound = flops / (P * 1e12) >= bytes_ / (pk["hbm"] * 1e9)
    if tensor_bound:
        achieved = flops / kernel_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": P, "unit": "TFLOP/s",
                "frac": achieved / P,
                "frac_burst": achieved / (ratio * pk["tflops"]),
                "frac_sustained": achieved / (ratio * pk["tflops_sustained"])}
    else:
        achieved = bytes_ / kernel_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"]}
    roof.update({
        "kernel": kernel, "kernel_us_per_launch": kernel_s * 1e6,
        "kernel_time_src": "CUDA events on the context's stream around each step's first "
                           "attention launch (the redo pass, which returns at once, is outside), "
                           "over a second run of the same steps; the step rate comes from the "
                           "run without them",
        "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": bytes_,
        "peak_choice": which,
        "peak_src": f"{pk['src']} ({'bf16 burst' if which == 'burst' else 'bf16 sustained'}"
                    f"{' x 2 (fp8/bf16 nominal ratio)' if fp8 else ''}"
                    f"{'' if tensor_bound else '; HBM copy'}); timed region {timed_s:.3f} s at "
                    f"median {clk['sm_mhz'] if clk else '?'} MHz (max "
                    f"{clk['sm_max_mhz'] if clk else '?'})",
        "timed_region_s": timed_s,
        "sm_mhz_median": clk["sm_mhz"] if clk else None,
    })
    kmhz = clk.get("kernel_sm_mhz") if clk else None
    if kmhz and tensor_bound:
        # the clock the kernel itself ran at (clock64 over %globaltimer of one
        # CTA), and the fraction of the nominal dense tensor peak at that clock
        # (148 SMs x 8192 bf16 flop per clock, x 2 for 8-bit operands)
        nominal = 148 * 8192 * ratio * kmhz * 1e6 / 1e12
        roof["kernel_sm_mhz"] = kmhz
        roof["frac_nominal_at_kernel_clock"] = achieved / nominal
    if timeline and tensor_bound:
        # the same kernel in the run without events, from its own stamps: from
        # its dependency wait to the redo pass finding it complete
        ks = (timeline["first_pass_done"] - timeline["attention_past_wait"]) * 1e-6
        if ks > 0:
            roof["kernel_us_timeline"] = ks * 1e6
            roof["frac_timeline"] = flops / ks / 1e12 / P
    if pk.get("clocks"):
        roof["peak_clocks"] = pk["clocks"]
    return roof


# DRAM bytes (read + write) per launch of the tensor-core kernel, from the ncu
# capture summarised under profiles/ (taken on the V=65536 profiling shape and
# scaled by the vocabulary, since E and the P ring both grow with V).
DRAM_TRAFFIC = {
    (synthetic.HEADLINE.name, 0): (4 * (291.782144e6 + 9.212928e6),
                                   "ncu dram__bytes_read.sum + dram__bytes_write.sum of one first-pass "
                                   "launch at C=256, V=65536, d=2048, scaled by 4 to V=262144"),
    (synthetic.HEADLINE.name, 1): (4 * (136.710912e6 + 6.254592e6),
                                   "ncu dram__bytes_read.sum + dram__bytes_write.sum of one first-pass "
                                   "launch (narrow E) at C=256, V=65536, d=2048, scaled by 4"),
}


def run_reference(args, w):
    """Reference arm: the CPU oracle on the host cores, same metric and config.

    Each timed step is one whole step of the workload. As many steps as
    --steps asks for are timed, but no more than fit in about two minutes (at
    least one); "steps" reports how many ran, "warmup" the one untimed step.
    """
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    E32 = synthetic.make_embedding_f32(w.V, w.d, w.e_seed)
    if w.dtype == "bf16":
        import torch
        E32 = torch.from_numpy(E32).to(torch.bfloat16).float().numpy()
    cb, step_s = cpu_baseline(w, E32, steps=max(1, args.steps), budget_s=120.0)
    n = cb["steps_timed"]
    val = 1.0 / step_s
    line = {"metric": METRIC, "value": val, "unit": "steps/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": n, "warmup": 1,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "tok_per_s": w.C * val,
            "steps_requested": args.steps, "warmup_requested": args.warmup,
            "config": {"workload": w.name, "C": w.C, "V": w.V, "d": w.d,
                       "canvases": w.canvases,
                       "token_rule": "multinomial" if w.token_rule == 1 else "argmax",
                       "mode": "fixed_steps"},
            "cpu_baseline": {"value": val, "unit": "steps/s", "cores": cb["cores"],
                             "kind": "oracle", "sample": cb["sample"], "cpu_model": cb["cpu_model"]},
            "e2e": {"value": val, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# GPU legs.
# ----------------------------------------------------------------------------
_E_CPU = {}


def embedding_cpu(w):
    """The workload's E on the host, made once per (V, d, dtype, seed) in a run."""
    key = (w.V, w.d, w.dtype, w.e_seed)
    if key not in _E_CPU:
        if len(_E_CPU) >= 3:
            _E_CPU.pop(next(iter(_E_CPU)))
        _E_CPU[key] = synthetic.make_embedding(w)
    return _E_CPU[key]


class FixedStepLoop:
    """Steps of one context in the fixed-step mode: a new block after every S steps."""

    def __init__(self, den, S):
        self.den, self.S, self.t, self.block = den, S, 0, 0

    def __call__(self):
        if self.t == self.S:
            self.block += 1
            self.den.begin_block(self.block)
            self.t = 0
        self.den.step()
        self.t += 1


def kernel_clock_mhz(den):
    """The SM clock the last attention launch ran at: clock64 over %globaltimer
    of one CTA across its lifetime (tensor-core contexts), or None."""
    import uniform_state_text_b200 as dg
    if den.impl != dg.DG_IMPL_TC:
        return None
    r = den.read(dg.DG_TC_TRACE_COUNTERS)[255].cpu().tolist()
    dt = r[2] - r[0]
    return 1e3 * (r[3] - r[1]) / dt if dt > 0 else None


def step_timeline(den):
    """The last step's timeline from the kernels' %globaltimer stamps (row 255
    of DG_TC_TRACE_COUNTERS, each by CTA 0 of its kernel), in us after the
    previous step's merge kernel ended; None for CUDA-core contexts."""
    import uniform_state_text_b200 as dg
    if den.impl != dg.DG_IMPL_TC:
        return None
    r = den.read(dg.DG_TC_TRACE_COUNTERS)[255].cpu().tolist()
    if not (r[9] > 0 and r[8] >= r[9]):
        return None
    keys = (("attention_started", 0), ("attention_past_wait", 4), ("first_pass_done", 5),
            ("merge_started", 6), ("merge_past_wait", 7), ("merge_done", 8))
    return {k: (r[j] - r[9]) / 1e3 for k, j in keys}


def timed_steps(den, step, steps: int, warmup: int, local: int, dist=None):
    """Device-timed region of `steps` calls of step() on den's stream.

    The region itself has no event inside a step: an event recorded between two
    kernels ends their programmatic dependent launch, and the two per step that
    timing the attention kernel needs added about 10 us of gaps per step
    (measured). So the same `steps` calls run twice: first bare, for the step
    time; then with dg_profile's events around each attention launch, for that
    kernel's duration and the launch count.

    Returns (ms of the bare region, max over ranks), (attention-kernel ms,
    steps timed, kernels launched) from the profiled pass, the clocks sampled
    during the bare region, its length in seconds and the timeline of its last
    step (step_timeline).
    """
    import torch

    import uniform_state_text_b200 as dg
    for _ in range(warmup):
        step()
    den.stream.synchronize()
    clocks = Clocks(local)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ev0.record(den.stream)
    for _ in range(steps):
        step()
    ev1.record(den.stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    kclk = kernel_clock_mhz(den)
    tl = step_timeline(den)
    dg.dg_profile(den.ctx, True)
    for _ in range(steps):
        step()
    prof = dg.dg_profile_read(den.ctx)
    dg.dg_profile(den.ctx, False)
    if dist:
        dist.barrier()
    st = den.state()
    if st["status"] != 0:
        raise RuntimeError(f"device status {st['status']}")
    if clk is not None:
        clk["kernel_sm_mhz"] = kclk
    return max_over_ranks(ms, dist, "cuda"), prof, clk, ms / 1e3, tl


def e2e_leg(den, w, steps: int, dist=None):
    """Wall clock of `steps` dg_denoise_step_h calls with host buffers.

    Every step copies a hidden state [C][d] in from pinned host memory (two
    alternating host buffers) and the updated canvas out to pinned host memory;
    the host is synchronised before the first call and after the last.
    """
    import torch

    import uniform_state_text_b200 as dg
    den.begin_block(0)
    den.step()
    h0 = den.read(dg.DG_HIDDEN).cpu()
    h_host = [h0.clone().pin_memory(), h0.clone().pin_memory()]
    canvas_host = torch.empty(w.C, dtype=torch.int32).pin_memory()
    S = w.max_steps

    def run(n):
        done_steps = 0
        for i in range(n):
            if done_steps == S:
                den.begin_block(0)
                done_steps = 0
            den.step_h(h_host[i % 2], canvas_host=canvas_host)
            done_steps += 1

    den.begin_block(0)
    run(3)
    torch.cuda.synchronize()
    den.begin_block(0)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    run(steps)
    torch.cuda.synchronize()
    el = time.perf_counter() - t0
    if den.state()["status"] != 0:
        raise RuntimeError("device status after the e2e leg")
    return max_over_ranks(el, dist, "cuda"), int(h0.numel() * h0.element_size()), int(w.C * 4)


def redo_leg(den, w, E, steps: int):
    """Cost of the redo pass: device time per step of dg_denoise_step_h with
    caller hidden states h = 30 E[token] whose largest logits overshoot the
    rows' references (the logits of the previous step's tokens) on no row, on
    1% of the rows, and on every row. Steps alternate between two hidden
    states; in the 'none' case both are the same, so after the untimed first
    step every reference is exact."""
    import torch

    import uniform_state_text_b200 as dg
    g = torch.Generator().manual_seed(7)
    tok_a = torch.randint(0, w.V, (w.C,), generator=g)
    tok_b = torch.randint(0, w.V, (w.C,), generator=g)
    few = tok_a.clone()
    k = max(1, w.C // 100)
    few[:k] = tok_b[:k]

    def hid(tok):
        return (30.0 * E[tok.to(E.device)].float()).to(E.dtype).contiguous()

    h_a = hid(tok_a)
    cases = {"none": h_a, "1pct": hid(few), "all": hid(tok_b)}
    n = max(2, min(steps, w.max_steps - 1))
    out = {"steps": n, "rows": w.C, "rounds": 3,
           "path": "dg_denoise_step_h with device hidden states, CUDA events on the stream; "
                   "the cases interleaved over 3 rounds, median per case"}
    times = {k: [] for k in cases}
    redone = {}
    for _ in range(3):
        for name, h_b in cases.items():
            den.begin_block(0)
            den.step_h(h_a)                               # step 0: every reference is low
            r0 = den.state()["redo"]
            ev0 = torch.cuda.Event(enable_timing=True)
            ev1 = torch.cuda.Event(enable_timing=True)
            ev0.record(den.stream)
            for i in range(n):
                den.step_h(h_b if i % 2 == 0 else h_a)
            ev1.record(den.stream)
            torch.cuda.synchronize()
            st = den.state()
            if st["status"] != 0:
                raise RuntimeError("device status after the redo leg")
            times[name].append(1e3 * ev0.elapsed_time(ev1) / n)
            redone[name] = (st["redo"] - r0) / n
    for name in cases:
        out[name] = {"us_per_step": float(np.median(times[name])),
                     "rows_redone_per_step": redone[name]}
    out["all_over_none"] = out["all"]["us_per_step"] / out["none"]["us_per_step"]
    return out


def headline_line(args, w, world, rank, local, dist):
    import torch

    import uniform_state_text_b200 as dg

    impl = {"auto": dg.DG_IMPL_AUTO, "simt": dg.DG_IMPL_SIMT, "tc": dg.DG_IMPL_TC}[args.kernels]
    E_cpu = embedding_cpu(w)
    E = E_cpu.to(f"cuda:{local}")
    den = dg.Denoiser(w, E, impl=impl)
    kern = "tcgen05" if den.impl == dg.DG_IMPL_TC else "CUDA-core"
    ms, (attn_ms, attn_steps, launches), clk, timed_s, timeline = timed_steps(
        den, FixedStepLoop(den, w.max_steps), args.steps, args.warmup, local, dist)
    value = whole_job_rate(args.steps, world, ms)
    ms_per_step = ms / args.steps

    e2e = None
    if not args.no_e2e:
        el, bi, bo = e2e_leg(den, w, args.steps, dist)
        e2e = {"value": args.steps * world / el, "unit": "steps/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
               "tok_per_s": w.C * args.steps * world / el, "steps": args.steps,
               "path": "dg_denoise_step_h: hidden state from pinned host memory (copy stream, "
                       "overlapping the step before), canvas to pinned host memory (written by "
                       "the step's merge kernel, no copy in the stream); host wall clock with a "
                       "synchronisation on both sides"}

    redo = None
    if den.impl == dg.DG_IMPL_TC and not args.no_workloads:
        redo = redo_leg(den, w, E, args.steps)

    pk = measured_peaks()
    t_b, t_s, _ = step_roofline(w, pk)
    roof = kernel_roofline(w, pk, (attn_ms / 1e3) / max(attn_steps, 1), timed_s, clk,
                           f"vocabulary attention ({kern})", timeline)
    traffic = DRAM_TRAFFIC.get((w.name, w.e_format)) if den.impl == dg.DG_IMPL_TC else None
    roof["traffic"] = traffic[0] if traffic else None
    roof["traffic_src"] = traffic[1] if traffic else None
    roof.update({"step_roofline_us": t_b * 1e6, "step_roofline_us_sustained": t_s * 1e6,
                 "step_roofline_pct": 100.0 * t_b / (ms_per_step / 1e3),
                 "step_roofline_pct_sustained": 100.0 * t_s / (ms_per_step / 1e3)})
    den.close()
    del E
    torch.cuda.empty_cache()
    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("e4m3/e5m2" if w.e_format == 1 else "bf16") if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded E ~ N(0, I/d), stand-in hidden state)",
            "tok_per_s": w.C * value,
            "roofline_pct": roof["step_roofline_pct"],
            "config": {"workload": w.name, "C": w.C, "V": w.V, "d": w.d,
                       "canvases": w.canvases,
                       "e_format": "e4m3 codes, power-of-two scale per 256-row block" if w.e_format == 1
                                   else "bf16",
                       "token_rule": "multinomial" if w.token_rule == 1 else "argmax",
                       "max_steps": w.max_steps, "mode": "fixed_steps (adaptive stop off)",
                       "kernels": "tc" if den.impl == dg.DG_IMPL_TC else "simt",
                       "l2": "no flush: E (%.2f GB) exceeds the 126 MB L2 and is streamed every step"
                             % (w.e_bytes / 1e9),
                       "parallelism": f"replicas x{world}"},
            "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
            "step_timeline_us": timeline, "redo_cost": redo}
    return line, E_cpu


def workload_throughput(w, steps, warmup, local, with_cpu: bool):
    """Device-timed fixed-step throughput of one more workload, with its roofline."""
    import torch

    import uniform_state_text_b200 as dg
    E_cpu = embedding_cpu(w)
    E = E_cpu.cuda()
    den = dg.Denoiser(w, E)
    kern = "tcgen05" if den.impl == dg.DG_IMPL_TC else "CUDA-core"
    ms, (attn_ms, attn_steps, launches), clk, timed_s, timeline = timed_steps(
        den, FixedStepLoop(den, w.max_steps), steps, warmup, local)
    pk = measured_peaks()
    t_b, t_s, _ = step_roofline(w, pk)
    ms_step = ms / steps
    out = {"workload": w.name, "C": w.C, "V": w.V, "d": w.d, "dtype": w.dtype,
           "e_format": "e4m3 codes, power-of-two scale per 256-row block" if w.e_format == 1 else "bf16",
           "mode": "fixed_steps", "steps": steps, "warmup": warmup,
           "value": 1e3 / ms_step, "unit": "steps/s", "ms_per_step": ms_step,
           "tok_per_s": w.C * 1e3 / ms_step, "gpu_launches": launches, "clocks": clk,
           "step_timeline_us": timeline, "step_roofline_us": t_b * 1e6,
           "step_roofline_pct": 100.0 * t_b / (ms_step / 1e3),
           "step_roofline_pct_sustained": 100.0 * t_s / (ms_step / 1e3),
           "roofline": kernel_roofline(w, pk, (attn_ms / 1e3) / max(attn_steps, 1), timed_s, clk,
                                       f"vocabulary attention ({kern})", timeline)}
    tr = DRAM_TRAFFIC.get((w.name, w.e_format)) if den.impl == dg.DG_IMPL_TC else None
    out["roofline"]["traffic"] = tr[0] if tr else None
    den.close()
    del E
    torch.cuda.empty_cache()
    if with_cpu:
        out["cpu_baseline"], _ = cpu_baseline(w, synthetic.embedding_as_f32(E_cpu), steps=1)
    return out


def tiny_latency(local, reps: int = 200):
    """The tiny fp32 check: latency of one step and of a whole adaptive block."""
    import torch

    import uniform_state_text_b200 as dg
    w = synthetic.TINY
    E = synthetic.make_embedding(w).cuda()
    wf = w.replace(fixed_steps=1)
    den = dg.Denoiser(wf, E)
    ms, (attn_ms, attn_steps, launches), clk, _, _ = timed_steps(
        den, FixedStepLoop(den, wf.max_steps), reps, 5, local)
    den.close()
    den = dg.Denoiser(w, E)
    out = torch.empty(w.C, dtype=torch.int32, device="cuda")
    host = torch.empty(w.C, dtype=torch.int32).pin_memory()
    for b in range(3):
        den.block(b, out=out)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    steps = 0
    for b in range(reps):
        steps += den.block(b, out=out)[1]
        host.copy_(out, non_blocking=True)
        den.stream.synchronize()
    el = time.perf_counter() - t0
    den.close()
    return {"workload": w.name, "C": w.C, "V": w.V, "d": w.d, "dtype": w.dtype,
            "step_latency_us": 1e3 * ms / reps, "value": reps / (ms / 1e3), "unit": "steps/s",
            "kernels": "CUDA-core (fp32)", "gpu_launches_per_step": launches / reps,
            "block_latency_us": 1e6 * el / reps, "block_steps_mean": steps / reps,
            "block_tok_per_s": w.C * reps / el,
            "block_path": "dg_denoise_block (graph loop to the adaptive stop) + emitted tokens to "
                          "pinned host memory, host wall clock per block",
            "roofline": None, "bound": "launch/latency (2.1 MFLOP per step)"}


def blocks_e2e(w, E_cpu, reps: int = 3):
    """Four sequential headline blocks to their adaptive stop, tokens to the host."""
    import torch

    import uniform_state_text_b200 as dg
    E = E_cpu.cuda()
    den = dg.Denoiser(w, E)
    buf = torch.empty(w.blocks * w.C, dtype=torch.int32, device="cuda")
    host = torch.empty(w.blocks * w.C, dtype=torch.int32).pin_memory()

    def run():
        steps = []
        for b in range(w.blocks):
            _, s = den.block(b, out=buf[b * w.C:(b + 1) * w.C])
            steps.append(s)
            host[b * w.C:(b + 1) * w.C].copy_(buf[b * w.C:(b + 1) * w.C], non_blocking=True)
        den.stream.synchronize()
        return steps

    run()
    torch.cuda.synchronize()
    times, steps = [], None
    for _ in range(reps):
        t0 = time.perf_counter()
        steps = run()
        times.append(time.perf_counter() - t0)
    den.close()
    del E
    torch.cuda.empty_cache()
    el = float(np.median(times))
    return {"workload": w.name, "blocks": w.blocks, "C": w.C, "V": w.V, "d": w.d,
            "dtype": w.dtype, "mode": "adaptive stop", "steps_per_block": steps,
            "value": w.blocks * w.C / el, "unit": "tok/s", "seconds": el,
            "path": "dg_denoise_block per block (graph loop to the adaptive stop), emitted tokens "
                    "copied to pinned host memory; host wall clock, median of %d runs" % reps,
            "d2h_bytes": w.blocks * w.C * 4}


def vocab_parallel_loop(den, buf, C, d, group=None):
    """One step of a canvas whose vocabulary is split over the ranks: the
    shard's partial step, the exchange of the partial row results (one sum and
    one max all-reduce), then the shard's finish (identical on every rank)."""
    import uniform_state_text_b200 as dg
    den.step_partial(buf)
    dg.allreduce_partials(buf, C, d, group=group)
    den.step_finish(buf)


def vocab_parallel_line(args, w, world, rank, local, dist):
    import torch

    import uniform_state_text_b200 as dg
    if w.V % (256 * world):
        raise SystemExit(f"V={w.V} does not split into {world} shards of 256-entry tiles")
    nv = w.V // world
    E = embedding_cpu(w).to(f"cuda:{local}")
    den = dg.Denoiser(w, E, impl=dg.DG_IMPL_TC, shard=(rank * nv, nv))
    buf = den.partials()
    state = {"t": 0, "block": 0}

    def step():
        if state["t"] == w.max_steps:
            state["block"] += 1
            den.begin_block(state["block"])
            state["t"] = 0
        with torch.cuda.stream(den.stream):
            vocab_parallel_loop(den, buf, w.C, w.d)
        state["t"] += 1

    ms, (attn_ms, attn_steps, launches), clk, timed_s, timeline = timed_steps(
        den, step, args.steps, args.warmup, local, dist)
    value = shared_canvas_rate(args.steps, ms)
    den.close()
    if rank == 0:
        return {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (seeded E ~ N(0, I/d), stand-in hidden state)",
                "tok_per_s": w.C * value,
                "config": {"workload": w.name, "C": w.C, "V": w.V, "d": w.d,
                           "mode": "fixed_steps (adaptive stop off)", "kernels": "tc",
                           "parallelism": f"vocabulary-parallel x{world} (NCCL sum+max exchange)",
                           "shard_entries": nv},
                "attention_ms_per_step_rank0": attn_ms / max(attn_steps, 1),
                "gpu_launches": launches, "clocks": clk, "e2e": None, "roofline": None,
                "cpu_baseline": None}
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=synthetic.HEADLINE.name, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--kernels", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "vocab"],
                    help="multi-GPU mode: independent canvases per rank, or one canvas's "
                         "vocabulary split over the ranks")
    ap.add_argument("--e-format", default="native", choices=["native", "fp8"],
                    help="E as given (bf16), or e4m3 codes with a power-of-two scale per 256-row block")
    ap.add_argument("--token-rule", default="argmax", choices=["argmax", "multinomial"],
                    help="token an accepted position takes")
    ap.add_argument("--canvases", type=int, default=0,
                    help="split the workload's C positions into this many independent "
                         "canvases (tau scaled per canvas); 0 keeps the workload's own")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads (tiny, small, latency, blocks)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    w = synthetic.WORKLOADS[args.workload].replace(fixed_steps=1)
    if args.token_rule == "multinomial":
        w = w.replace(token_rule=1)
    if args.e_format == "fp8":
        w = w.replace(e_format=1)
    if args.canvases > 0:
        w = w.replace(canvases=args.canvases, tau=w.tau * w.canvases / args.canvases)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import uniform_state_text_b200 as dg
    from uniform_state_text_b200 import build as dgbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        if world == 1 and args.gpus > 1:
            print(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes", file=sys.stderr)
            return 2
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        dgbuild.build()
    if dist:
        dist.barrier()
    dg.lib()

    if args.parallel == "vocab":
        line = vocab_parallel_line(args, w, world, rank, local, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if dist:
            dist.destroy_process_group()
        return 0

    w = w.replace(seed=rank)
    line, E_cpu = headline_line(args, w, world, rank, local, dist)
    if rank == 0 and world == 1:
        if not args.no_cpu_baseline:
            line["cpu_baseline"], _ = cpu_baseline(w, synthetic.embedding_as_f32(E_cpu), steps=1)
        else:
            line["cpu_baseline"] = None
        if not args.no_workloads and args.workload == synthetic.HEADLINE.name:
            wl = [tiny_latency(local)]
            for wk in (synthetic.SMALL, synthetic.LATENCY):
                wl.append(workload_throughput(wk.replace(fixed_steps=1), max(args.steps, 200),
                                              args.warmup, local, not args.no_cpu_baseline))
            # narrow E (e4m3 codes): the memory-bound latency canvas and the headline
            for wk in (synthetic.LATENCY, synthetic.HEADLINE):
                wl.append(workload_throughput(wk.replace(fixed_steps=1, e_format=1),
                                              max(args.steps, 200), args.warmup, local, False))
            wl.append(blocks_e2e(synthetic.BLOCKS, E_cpu))
            line["workloads"] = wl
    else:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

"""Host-side arithmetic of bench.py on CPU: the step and kernel rooflines, the
choice of peak, and the step timeline read from the kernels' stamps."""
import math

import pytest
import torch

import bench
import synthetic
import uniform_state_text_b200 as dg

PEAKS = dict(hbm=6542.4, tflops=1663.5, tflops_sustained=1410.5, src="test", clocks={})


def test_step_roofline_of_the_headline_canvas():
    w = synthetic.HEADLINE
    t_b, t_s, flops = bench.step_roofline(w, PEAKS)
    assert flops == 4.0 * 256 * 2048 * 262144
    # tensor-bound at both peaks: 5.50e11 flop at 1663.5 and 1410.5 TFLOP/s
    assert t_b == pytest.approx(flops / 1663.5e12)
    assert t_s == pytest.approx(flops / 1410.5e12)
    assert t_b * 1e6 == pytest.approx(330.5, abs=0.1)


def test_step_roofline_of_the_latency_canvas_is_hbm_bound():
    w = synthetic.WORKLOADS["canvas_c128_v262144_d2816_bf16"]
    t_b, _, _ = bench.step_roofline(w, PEAKS)
    assert t_b == pytest.approx(2.0 * w.V * w.d * 2 / 6542.4e9)     # E read twice, bf16


def test_peak_choice_follows_the_timed_region_length():
    assert bench.choose_peak(0.01, None) == "burst"
    assert bench.choose_peak(bench.BURST_MAX_S + 0.1, None) == "sustained"


def test_kernel_roofline_fractions():
    w = synthetic.HEADLINE
    flops = 4.0 * w.C * w.d * w.V
    kernel_s = 450e-6
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "kernel_sm_mhz": 1700.0}
    tl = {"attention_past_wait": 3.0, "first_pass_done": 423.0}
    r = bench.kernel_roofline(w, PEAKS, kernel_s, 0.01, clk, "k", tl)
    assert r["bound"] == "tensor" and r["peak"] == 1663.5 and r["peak_choice"] == "burst"
    assert r["achieved"] == pytest.approx(flops / kernel_s / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1663.5)
    assert r["frac_sustained"] == pytest.approx(r["achieved"] / 1410.5)
    assert r["kernel_us_timeline"] == pytest.approx(420.0)
    assert r["frac_timeline"] == pytest.approx(flops / 420e-6 / 1e12 / 1663.5)
    nominal = 148 * 8192 * 1700e6 / 1e12
    assert r["frac_nominal_at_kernel_clock"] == pytest.approx(r["achieved"] / nominal)
    # a long region takes the sustained peak
    r2 = bench.kernel_roofline(w, PEAKS, kernel_s, 5.0, clk, "k")
    assert r2["peak"] == 1410.5 and "frac_timeline" not in r2


def test_kernel_roofline_of_the_narrow_embedding_doubles_the_peak():
    w = synthetic.HEADLINE.replace(e_format=1)
    r = bench.kernel_roofline(w, PEAKS, 250e-6, 0.01, None, "k")
    assert r["peak"] == pytest.approx(2 * 1663.5)
    assert r["algorithmic_bytes_per_launch"] == pytest.approx(
        w.V * w.d * 1 + 4.0 * w.V + w.C * w.d * (1 + 4))


class _FakeDen:
    impl = dg.DG_IMPL_TC

    def __init__(self, row):
        self.row = row

    def read(self, what):
        assert what == dg.DG_TC_TRACE_COUNTERS
        t = torch.zeros(256, 32, dtype=torch.int64)
        t[255, :len(self.row)] = torch.tensor(self.row, dtype=torch.int64)
        return t


def test_step_timeline_from_the_stamps():
    base = 1_000_000_000
    row = [base + 2000, 7, base + 400000, 9, base + 3000, base + 421000, base + 422000,
           base + 422500, base + 431500, base]
    tl = bench.step_timeline(_FakeDen(row))
    assert tl == {"attention_started": 2.0, "attention_past_wait": 3.0, "first_pass_done": 421.0,
                  "merge_started": 422.0, "merge_past_wait": 422.5, "merge_done": 431.5}
    # no previous merge stamp yet: no timeline
    assert bench.step_timeline(_FakeDen(row[:9] + [0])) is None


def test_missing_peaks_file_falls_back(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk = bench.measured_peaks()
    assert pk["src"] == "fallback" and pk["tflops"] == 1590.0 and math.isclose(pk["hbm"], 6650.0)

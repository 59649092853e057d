"""The benchmark's work model and roofline arithmetic, against closed forms.

The step's ideal bytes (Q, K, V read and out written once) and its FLOP, split into
the dense contractions (Q K_l^T, P W, Q_l K^T, P V, Q_l K_l^T, Z k3V), the inverse
(8 m^3 per iteration) and the 65-tap conv, are checked against the figures derived
directly from the method's operation counts for the n = 16384 and n = 4096 bf16
workloads; the per-kernel roofline picks the bound whose ideal time is longer.
"""
import pytest

import bench
from workloads import WORKLOADS

PEAKS = {"hbm_gbs": 6557.8, "bf16_tflops": 1664.0, "sm_max_mhz": 1965.0}


def _split(w):
    BH, n, d, m = w.BH, w.n, w.d, w.m
    gemm = BH * (4 * 2 * n * m * d + 2 * 2 * m * m * d)
    pinv = BH * w.n_iter * 8 * m ** 3
    conv = BH * 2 * 65 * n * d if w.conv else 0
    return gemm, pinv, conv


def _printed(x):
    """Half a unit of the last printed digit of a figure given to three significant digits."""
    s = f"{x}"
    decimals = len(s.split(".")[1]) if "." in s else 0
    return 0.5 * 10 ** -decimals + 1e-9


@pytest.mark.parametrize("name,mbytes,gemm_g,pinv_g,conv_g", [
    ("n16384_bf16_corr", 268.4, 69.3, 25.8, 4.36),      # B4 H8 n16384 d64 m256, conv on
    ("longcls_bf16_masked", 67.1, 8.72, 6.44, 1.09),    # B32 H2 n4096 d32 m128, conv on
])
def test_step_work_matches_operation_counts(name, mbytes, gemm_g, pinv_g, conv_g):
    w = WORKLOADS[name]
    t_roof, nbytes, flops = bench.roofline_bound_time(w, PEAKS)
    gemm, pinv, conv = _split(w)
    assert nbytes == 4 * w.BH * w.n * w.d * 2
    assert nbytes / 1e6 == pytest.approx(mbytes, abs=_printed(mbytes))
    assert gemm / 1e9 == pytest.approx(gemm_g, abs=_printed(gemm_g))
    assert pinv / 1e9 == pytest.approx(pinv_g, abs=_printed(pinv_g))
    assert conv / 1e9 == pytest.approx(conv_g, abs=_printed(conv_g))
    assert flops == gemm + pinv + conv
    assert t_roof == max(nbytes / (PEAKS["hbm_gbs"] * 1e9), flops / (PEAKS["bf16_tflops"] * 1e12))


def test_headline_step_is_compute_bound_at_about_60_us():
    t_roof, _, _ = bench.roofline_bound_time(WORKLOADS["n16384_bf16_corr"], PEAKS)
    assert t_roof * 1e6 == pytest.approx(59.73, abs=0.05)


def test_kernel_rooflines_pick_the_longer_bound():
    w = WORKLOADS["n16384_bf16_corr"]
    # the inverse: tf32 on the tensor core, FLOP-bound (25.8 GFLOP against 12.6 MB)
    r = bench.roofline_for(w, "pinv", 0.130, PEAKS, bench.SIMT_KERNELS, None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["algorithmic_flops"] == w.BH * w.n_iter * 8 * w.m ** 3
    assert r["peak"] == pytest.approx(1664.0 * 1.1 / 2.25, abs=0.1)
    assert r["achieved"] == pytest.approx(r["algorithmic_flops"] / 0.130e-3 / 1e12, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3)
    # the landmark means: pure traffic, HBM-bound
    r = bench.roofline_for(w, "landmarks", 0.030, PEAKS, bench.SIMT_KERNELS, 139063040)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 139063040
    assert r["algorithmic_bytes"] == 2 * w.BH * w.n * w.d * 2 + 2 * w.BH * w.m * w.d * 4
    assert r["achieved"] == pytest.approx(r["algorithmic_bytes"] / 0.030e-3 / 1e9, rel=1e-3)


def test_pipe_aware_bound_charges_the_inverse_at_tf32():
    w = WORKLOADS["n16384_bf16_corr"]
    t = bench.roofline_bound_time_pipes(w, PEAKS)
    tf32 = PEAKS["bf16_tflops"] * 1.1 / 2.25
    m, n, d = w.m, w.n, w.d
    expect = (w.BH * (8 * n * m * d + 2 * m * m * d + 2 * 65 * n * d) / (PEAKS["bf16_tflops"] * 1e12)
              + w.BH * (6 * 8 * m ** 3 + 6 * m * m * d) / (tf32 * 1e12))
    assert t == pytest.approx(expect, rel=1e-12)
    assert 75e-6 < t < 77e-6                                   # about 76 us: compute-bound
    assert t > bench.roofline_bound_time(w, PEAKS)[0]          # never below the plain bound here
    wf = WORKLOADS["default_f32_masked"]                       # fp32: both bounds are the same
    assert bench.roofline_bound_time_pipes(wf, PEAKS) == bench.roofline_bound_time(wf, PEAKS)[0]


def test_exponential_bound_charges_two_softmaxes_to_the_mufu():
    """2 B H n m exponentials (kernel_1 and kernel_3) at 16 per clock per SM: about 58 us at
    the headline shape, just under the pipe-aware bound."""
    w = WORKLOADS["n16384_bf16_corr"]
    t, t_exp = bench.roofline_bound_time_exp(w, PEAKS)
    assert bench.step_exponentials(w) == 2 * 32 * 16384 * 256
    assert t_exp == pytest.approx(2 * 32 * 16384 * 256 / (148 * 16 * 1965e6), rel=1e-12)
    assert 57e-6 < t_exp < 58.5e-6
    assert t == max(t_exp, bench.roofline_bound_time_pipes(w, PEAKS))


def test_exact_branch_bound_counts_n_squared_work():
    """Path A: 4 n^2 d flops per head (Q K^T and P V) plus the conv, n^2 exponentials."""
    w = WORKLOADS["longcls_bf16_masked"]
    t, nbytes, flops = bench.roofline_bound_time_exact(w, PEAKS)
    assert flops == w.BH * (4 * w.n ** 2 * w.d + 2 * 65 * w.n * w.d)
    assert nbytes == 4 * w.BH * w.n * w.d * 2
    assert t == max(nbytes / (PEAKS["hbm_gbs"] * 1e9), flops / (PEAKS["bf16_tflops"] * 1e12))
    assert bench.step_exponentials(w, "exact") == w.BH * w.n * w.n
    nb, fl, unit = bench.kernel_work(w, "k3v_partial", "exact")
    assert fl == w.BH * 4 * w.n * w.n * w.d and unit == "tensor"


def test_clock_samples_are_taken_from_the_timed_window():
    """Only the nvidia-smi lines printed during the timed steps count (plus one polling
    interval); throttle reasons are read from the same lines; with none inside the window the
    sampler falls back to every line."""
    s = bench.ClockSampler(None)
    s.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    s.t = type("T", (), {"join": lambda self, timeout=None: None})()
    idle = "0, 1200, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = "0, 1965, 1965, 700.0, 0x4, Not Active, Not Active, Not Active, Active"
    s.lines = [idle, busy, busy, busy, idle]
    s.times = [10.0, 10.50, 10.52, 10.54, 11.0]
    c = s.stop((10.49, 10.55))
    assert c["sm_mhz"] == 1965 and c["samples"] == 3 and c["samples_from"] == "timed steps"
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 700.0
    c = s.stop((20.0, 20.1))
    assert c["samples"] == 5 and c["samples_from"] == "sampler lifetime" and c["sm_mhz"] == 1965

#!/usr/bin/env python3
"""Benchmark of the Nystromformer attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

One step = one whole forward (landmarks, kernel_2 + iterative inverse,
kernel_3 V, W = Z k3V, output with the depthwise conv) over one batch of
the workload, through the C ABI (nys_attn_forward). Default workload: the
n=16384 bf16 correlated-token shape (B=4, H=8, d=64, m=256, conv on).

Timing: W untimed warm-up steps; then K steps, each preceded by an L2 flush
(a 256 MiB device write followed by a 256 MiB read of another buffer, so that
no dirty lines are left to be written back during the step; outside the
timed interval) and bracketed by CUDA
events on the launching stream; a barrier and a device synchronisation on
both sides; the maximum over ranks is reported. The library brackets the
launches of the roofline kernel (the one with the largest device time) with
CUDA events on its own stream during the same timed steps; the per-kernel
breakdown comes from a separate untimed pass in which every launch is
bracketed (each event record delays the next launch by a few microseconds,
so the timed steps bracket only the one kernel they report). SM clocks and
throttle reasons are sampled with nvidia-smi during the timed steps.

Multi-GPU: the forward has no exchange step; each rank runs an independent
replica on its own seeded batch ("replicas only", weak scaling).

--impl reference times the fp64 CPU oracle on this machine's host cores instead
(rank 0 only), on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import HEADLINE, WORKLOADS, make_inputs  # noqa: E402

METRIC = "Nystrom attention tokens/s (B*H*n/s) at n=16384 bf16"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SMS = 148
FP32_LANES_PER_SM = 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources a kernel's launches depend on: its own headers and the host functions that plan
# and configure its launch (text taken from nys_attn.cu); a kernel launched inline in the
# forward's orchestration depends on that whole function
KERNEL_SOURCES = {
    "landmarks": (["landmarks.cuh"], ["launch_bf16", "launch_simt"]),
    "pinv": (["tc_pinv_pair.cuh", "tc_pinv_res.cuh", "sm100.cuh"], ["launch_pinv_pair", "launch_pinv_res"]),
    "k3v_partial": (["tc_k3v.cuh", "sm100.cuh"], ["launch_k3v_tc"]),
    "k3v_combine": (["simt.cuh"], ["launch_bf16", "launch_simt"]),
    "w_product": (["simt.cuh", "tc_w.cuh", "sm100.cuh"], ["launch_bf16", "launch_simt"]),
    "output": (["tc_output.cuh", "sm100.cuh"], ["launch_output_tc"]),
}


def _function_text(src, name):
    """The text of the top-level function `name` (from its signature to its closing brace)."""
    mt = re.search(r"\n[A-Za-z_][\w:<>]*\s+" + name + r"\(", src)
    if mt is None:
        raise KeyError(name)
    j = src.find("\n}\n", mt.start())
    return src[mt.start():j + 3]


def source_digest(kernel=None):
    """Digest of the CUDA sources of `kernel` (every source file when None): a traffic figure
    captured with ncu is only reported while the sources it was captured from are unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nystr_self_attention_scale_b200", "csrc")
    if kernel not in KERNEL_SOURCES:
        for name in sorted(os.listdir(csrc)):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
        return h.hexdigest()[:16]
    headers, funcs = KERNEL_SOURCES[kernel]
    for name in sorted(headers + ["common.cuh"]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(csrc, "nys_attn.cu")) as f:
        src = f.read()
    for fn in funcs + ["make_plan"]:
        h.update(fn.encode() + _function_text(src, fn).encode())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- algorithmic work per launch

def kernel_work(w, kernel, path="nystrom"):
    """(algorithmic bytes, algorithmic flops, compute unit) of one launch of `kernel`.

    Bytes count each input element read once and each output written once;
    flops count 2 per multiply-add of the dense contractions (softmax
    exponentials are not counted). On the exact branch (path A) kernel_3 V's
    machinery runs with all n query rows: 4 n^2 d flops per head, Q, K, V read;
    its epilogue (merge, conv, output) is the "output" kernel."""
    elt = 4 if w.dtype == "f32" else 2
    BH, n, d, m = w.BH, w.n, w.d, w.m
    tensor = BH * n * d * elt
    unit = "alu" if w.dtype == "f32" else "tensor"
    if path == "exact":
        if kernel == "k3v_partial":
            return 3 * tensor, BH * 4 * n * n * d, unit
        if kernel == "output":
            return 2 * tensor + BH * n * d * 4 * 3, BH * 2 * 65 * n * d if w.conv else 0, "alu"
        if kernel == "mask_bits":
            return w.B * n + w.B * n // 8, 0, "alu"
        raise KeyError(kernel)
    if kernel == "landmarks":
        return 2 * tensor + 2 * BH * m * d * 4, 0, "alu"
    if kernel == "pinv":
        return BH * 2 * m * d * 4 + BH * m * m * 4, BH * w.n_iter * 8 * m ** 3, \
            "alu" if w.dtype == "f32" else "tensor_tf32"
    if kernel == "k3v_partial":
        return 2 * tensor + BH * m * d * 4, BH * 4 * n * m * d, unit
    if kernel == "mask_bits":
        return w.B * n + w.B * n // 8, 0, "alu"
    if kernel == "k3v_combine":
        return BH * m * d * 8, 0, "alu"
    if kernel == "w_product":
        # tf32 tensor cores for bf16 inputs at m = 128 / 256, fp32 FMAs otherwise
        return BH * (m * m + 2 * m * d) * 4, BH * 2 * m * m * d, \
            "tensor_tf32" if (w.dtype == "bf16" and m % 128 == 0) else "alu"
    if kernel == "output":
        return 3 * tensor + BH * 2 * m * d * 4, BH * (4 * n * m * d + (2 * 65 * n * d if w.conv else 0)), unit
    raise KeyError(kernel)


def compute_peak_tflops(unit, peaks, kernel_impl_simt):
    """Peak of the unit a kernel runs on, in TFLOP/s."""
    if unit == "alu" or kernel_impl_simt:
        return N_SMS * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    if unit == "tensor_tf32":
        return peaks["bf16_tflops"] * 1.1 / 2.25   # nominal dense tf32 : bf16 = 1.1 : 2.25 PFLOP/s
    return peaks["bf16_tflops"]


SIMT_KERNELS = {"landmarks", "k3v_combine", "mask_bits"}


def roofline_for(w, kernel, avg_ms, peaks, simt_set, traffic, path="nystrom"):
    nbytes, flops, unit = kernel_work(w, kernel, path)
    simt = kernel in simt_set
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9)
    cpk = compute_peak_tflops(unit, peaks, simt)
    t_cmp = flops / (cpk * 1e12) if flops else 0.0
    sec = avg_ms * 1e-3
    if t_mem >= t_cmp:
        achieved = nbytes / sec / 1e9
        r = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = flops / sec / 1e12
        bound = "alu" if (simt or unit == "alu") else "tensor"
        r = {"bound": bound, "achieved": round(achieved, 3), "peak": round(cpk, 1), "unit": "TFLOP/s"}
    r["frac"] = round(achieved / r["peak"], 4)
    r["traffic"] = traffic
    r["kernel"] = kernel
    r["algorithmic_bytes"] = nbytes
    r["algorithmic_flops"] = flops
    r["avg_launch_us"] = round(avg_ms * 1e3, 2)
    return r


def roofline_bound_time(w, peaks):
    """t_roof = max(ideal bytes / HBM, total flops / bf16 peak) of the whole step."""
    elt = 4 if w.dtype == "f32" else 2
    nbytes = 4 * w.BH * w.n * w.d * elt
    m, n, d = w.m, w.n, w.d
    flops = w.BH * (4 * 2 * n * m * d + 2 * 2 * m * m * d + w.n_iter * 8 * m ** 3 +
                    (2 * 65 * n * d if w.conv else 0))
    peak = peaks["bf16_tflops"] if w.dtype == "bf16" else compute_peak_tflops("alu", peaks, True)
    return max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peak * 1e12)), nbytes, flops


def roofline_bound_time_pipes(w, peaks):
    """The same bound with every FLOP charged at the rate of the pipe that executes it: on the
    bf16 path the inverse's iteration runs in tf32 on the tensor core (kernel_2's three-term
    split product included), the contractions and the Toeplitz conv in bf16; fp32 runs all of
    it on the CUDA cores (then equal to roofline_bound_time)."""
    if w.dtype != "bf16":
        return roofline_bound_time(w, peaks)[0]
    m, n, d = w.m, w.n, w.d
    nbytes = 4 * w.BH * n * d * 2
    bf16 = w.BH * (4 * 2 * n * m * d + 2 * m * m * d + (2 * 65 * n * d if w.conv else 0))
    tf32 = w.BH * (w.n_iter * 8 * m ** 3 + 3 * 2 * m * m * d)
    t_flops = bf16 / (peaks["bf16_tflops"] * 1e12) + tf32 / (compute_peak_tflops("tensor_tf32", peaks, False) * 1e12)
    return max(nbytes / (peaks["hbm_gbs"] * 1e9), t_flops)


def roofline_bound_time_exact(w, peaks):
    """The exact branch (path A): t_roof = max(ideal bytes / HBM, flops / peak) with 4 n^2 d
    flops per head (Q K^T and P V) plus the conv; same ideal bytes as the Nystrom step."""
    elt = 4 if w.dtype == "f32" else 2
    nbytes = 4 * w.BH * w.n * w.d * elt
    flops = w.BH * (4 * w.n * w.n * w.d + (2 * 65 * w.n * w.d if w.conv else 0))
    peak = peaks["bf16_tflops"] if w.dtype == "bf16" else compute_peak_tflops("alu", peaks, True)
    return max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peak * 1e12)), nbytes, flops


MUFU_EX2_PER_CLK_SM = 16   # nominal special-function-unit rate of ex2.approx.f32 per SM


def step_exponentials(w, path="nystrom"):
    """Exponentials of one step: kernel_1 (n x m) and kernel_3 (m x n) per head; kernel_2's
    m x m is negligible and not counted. The exact branch: n x n per head."""
    if path == "exact":
        return w.BH * w.n * w.n
    return 2 * w.BH * w.n * w.m


def roofline_bound_time_exp(w, peaks, path="nystrom"):
    """The pipe-aware bound with the softmax exponentials added: every exponential charged to
    the MUFU unit at its nominal ex2.f32 rate (16 per clock per SM at the maximum SM clock),
    and the step bounded by the slowest of HBM traffic, tensor-pipe FLOP and MUFU time (the
    three pipes run concurrently). The kernels also evaluate part of the exponentials as
    FMA-pipe polynomials, so a kernel can beat the MUFU term; it is a reference, not a floor."""
    t_exp = step_exponentials(w, path) / (N_SMS * MUFU_EX2_PER_CLK_SM * peaks.get("sm_max_mhz", 1965.0) * 1e6)
    base = roofline_bound_time_exact(w, peaks)[0] if path == "exact" else roofline_bound_time_pipes(w, peaks)
    return max(base, t_exp), t_exp


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.times = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "20"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        # nvidia-smi can take a second or more to start on a fresh machine: the timed steps begin
        # only once it prints, so that its samples cover them
        t0 = time.time()
        while not self.lines and self.proc.poll() is None and time.time() - t0 < 5.0:
            time.sleep(0.02)
        time.sleep(0.05)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())
            self.times.append(time.time())

    def stop(self, window=None):
        """Summary of the samples; with window = (t0, t1) (host seconds) only those printed
        during it (plus one polling interval), unless there are none."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines, scope = self.lines, "sampler lifetime"
        if window is not None:
            inside = [ln for ln, t in zip(self.lines, self.times) if window[0] <= t <= window[1] + 0.025]
            if inside:
                lines, scope = inside, "timed steps"
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "samples_from": scope, "power_w_max": max(power), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU oracle timing

def oracle_sample(w, x, heads, rows=None, threads=0):
    import oracle
    b_idx = [b for b, _ in heads]
    h_idx = [h for _, h in heads]
    # gather the sampled heads into one [1, S, n, d] batch (head h keeps its conv weight)
    q = np.ascontiguousarray(x["q"][b_idx, h_idx][None])
    k = np.ascontiguousarray(x["k"][b_idx, h_idx][None])
    v = np.ascontiguousarray(x["v"][b_idx, h_idx][None])
    cw = None if x["conv_w"] is None else np.ascontiguousarray(x["conv_w"][h_idx])
    if x["mask"] is not None and len(set(b_idx)) > 1:
        raise ValueError("masked sample must come from one sequence")
    mask = None if x["mask"] is None else x["mask"][b_idx[0]:b_idx[0] + 1]
    t0 = time.perf_counter()
    oracle.forward(q, k, v, mask, cw, m=w.m, n_iter=w.n_iter, rows=rows, threads=threads)
    return time.perf_counter() - t0


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(w, x):
    import oracle
    oracle.build()
    cores = cpu_cores()
    nh = max(1, min(w.BH, cores))
    heads = [(i // w.H, i % w.H) for i in range(nh)]
    if x["mask"] is not None:
        heads = [(0, i % w.H) for i in range(min(nh, w.H))]
    sec = oracle_sample(w, x, heads, threads=min(cores, len(heads)))
    toks = len(heads) * w.n
    return {"value": round(toks / sec, 1), "unit": UNIT, "cores": min(cores, len(heads)),
            "kind": "oracle",
            "sample": f"{len(heads)} of {w.BH} heads, all {w.n} rows each, fp64 C oracle, "
                      f"{sec:.1f} s wall on {min(cores, len(heads))} threads"}


def rank_env():
    """(world size, rank, local rank) from the launcher's environment; (1, 0, 0) when run alone."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, world, device):
    """The largest value of a float over all ranks (the slowest rank's time).

    Identity at world size 1; otherwise one all-reduce(MAX) of a float64 on
    ``device`` ("cuda" under NCCL, "cpu" under gloo)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, steps, total_ms):
    """Whole-job tokens/s: the tokens every rank processed over the slowest rank's time."""
    return tokens_per_rank * world * steps / (total_ms * 1e-3)


def run_reference(args, w):
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    x = make_inputs(w, seed=0)
    cores = cpu_cores()
    nh = max(1, min(w.BH, cores))
    heads = [(i // w.H, i % w.H) for i in range(nh)]
    if x["mask"] is not None:
        heads = [(0, i % w.H) for i in range(min(nh, w.H))]
    threads = min(cores, len(heads))
    budget = float(os.environ.get("NYS_REFERENCE_BUDGET_S", "150"))
    # the requested warm-up steps (each a full sample), bounded to 60 s in all
    t_warm, warm_done, warm_total = 0.0, 0, 0.0
    while warm_done < args.warmup and (warm_done == 0 or warm_total + t_warm <= 60.0):
        t_warm = oracle_sample(w, x, heads, threads=threads)
        warm_total += t_warm
        warm_done += 1
    per = t_warm if t_warm > 0 else None
    steps_done, total = 0, 0.0
    while steps_done < args.steps:
        if per is not None and total + per > budget and steps_done > 0:
            break
        dt = oracle_sample(w, x, heads, threads=threads)
        total += dt
        per = dt
        steps_done += 1
    toks = len(heads) * w.n * steps_done
    value = toks / total
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
        "n_gpus": args.gpus, "steps": steps_done, "steps_requested": args.steps,
        "warmup": warm_done, "warmup_requested": args.warmup, "ms_per_step": round(1e3 * total / steps_done, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, see workloads/)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "d": w.d, "m": w.m,
                   "n_iter": w.n_iter, "conv": w.conv, "sample_heads": len(heads)},
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"per step {len(heads)} of {w.BH} heads x all {w.n} rows; "
                                   f"run capped at {budget:.0f} s"},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-flush", action="store_true")
    ap.add_argument("--path", default="nystrom", choices=["nystrom", "exact"],
                    help="exact: the layer's path A (exact softmax attention), through nys_attn_forward_ex")
    ap.add_argument("--inv-init", default="default", choices=["default", "exact"],
                    help="exact: the exact-coefficient Z_0 (inv_coeff_init_option), through nys_attn_forward_ex")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import nystr_self_attention_scale_b200 as nys

    x = make_inputs(w, seed=rank)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q = torch.from_numpy(x["q"]).to(dt).cuda()
    k = torch.from_numpy(x["k"]).to(dt).cuda()
    v = torch.from_numpy(x["v"]).to(dt).cuda()
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).cuda()
    conv_w = None if x["conv_w"] is None else torch.from_numpy(x["conv_w"]).cuda()
    out = torch.empty_like(q)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    flush_clean = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def flush_l2():
        # evict the step's inputs by writing a buffer larger than L2, then read another one so
        # that the written lines are written back here, untimed, and not during the next step
        flush.zero_()
        torch.sum(flush_clean, dim=0, keepdim=True, out=flush_sink)

    use_ex = args.path != "nystrom" or args.inv_init != "default"

    def step():
        if use_ex:
            nys.forward_ex(q, k, v, mask=mask, conv_w=conv_w, m=w.m, n_iter=w.n_iter, out=out,
                           inv_coeff_init_option=args.inv_init == "exact", exact=args.path == "exact")
        else:
            nys.forward(q, k, v, mask=mask, conv_w=conv_w, m=w.m, n_iter=w.n_iter, out=out)

    for _ in range(args.warmup):
        if not args.no_flush:
            flush_l2()
        step()
    torch.cuda.synchronize()
    assert nys.device_status() == 0

    # per-kernel breakdown: a separate, untimed pass in which every kernel launch is bracketed by
    # CUDA events (the event records delay each following launch, so the timed loop below
    # brackets only the dominant kernel, the one the roofline reports, and only in its last
    # tenth of steps: the brackets add a few microseconds to each step they are in)
    breakdown_steps = 10
    nys.profile_mask(None)
    nys.profile_enable(True)
    for _ in range(breakdown_steps):
        if not args.no_flush:
            flush_l2()
        step()
    torch.cuda.synchronize()
    prof_all = nys.profile_read()
    nys.profile_enable(False)
    dom = max(prof_all, key=lambda kname: prof_all[kname][1])
    per_step_launches = sum(n for n, _ in prof_all.values()) / breakdown_steps

    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id)
    sampler.start()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_timed0 = time.time()
    nys.profile_mask([dom])
    prof_steps = max(1, args.steps // 10)
    for i in range(args.steps):
        if i == args.steps - prof_steps:
            nys.profile_enable(True)
        if not args.no_flush:
            flush_l2()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t_timed1 = time.time()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop((t_timed0, t_timed1))
    prof = nys.profile_read()
    nys.profile_enable(False)
    nys.profile_mask(None)
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    status = nys.device_status()
    total_ms = max_over_ranks(total_ms, world, "cuda")
    ms_per_step = total_ms / args.steps
    value = job_throughput(w.tokens, world, args.steps, total_ms)

    peaks, peak_src = load_peaks()
    launches = int(round(per_step_launches * args.steps))
    kernels = {name: {"launches": n, "total_ms": round(ms, 4),
                      "avg_us": round(1e3 * ms / n, 2) if n else None}
               for name, (n, ms) in prof_all.items()}
    kernel_ms_total = sum(ms for _, ms in prof_all.values()) or 1.0
    for name in kernels:
        kernels[name]["share"] = round(prof_all[name][1] / kernel_ms_total, 4)
    traffic = None
    tf = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tf):
        with open(tf) as f:
            tr = json.load(f)
        ent = tr.get(dom)
        if ent and ent.get("source_digest") == source_digest(dom) and ent.get("workload") == w.name:
            traffic = ent.get("bytes_per_launch")
    simt = set(SIMT_KERNELS)
    if w.dtype == "f32":  # the float32 path runs every stage on CUDA cores
        simt |= {"pinv", "k3v_partial", "output", "w_product"}
    elif w.m % 128 != 0:
        simt.add("w_product")   # W on CUDA cores at m = 64
    if args.path == "exact":
        traffic = None   # the ncu traffic figures are for the Nystrom path's kernels
    roof = roofline_for(w, dom, prof[dom][1] / max(1, prof[dom][0]), peaks, simt, traffic, args.path)
    roof["launches_timed"] = int(prof[dom][0])   # the dominant kernel's launches in the timed steps
    roof["peak_source"] = f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})"
    if args.path == "exact":
        t_roof, ideal_bytes, total_flops = roofline_bound_time_exact(w, peaks)
        t_pipes = t_roof
    else:
        t_roof, ideal_bytes, total_flops = roofline_bound_time(w, peaks)
        t_pipes = roofline_bound_time_pipes(w, peaks)
    t_exp_roof, t_exp = roofline_bound_time_exp(w, peaks, args.path)

    e2e = None
    if not args.no_e2e and not use_ex:
        qh = torch.from_numpy(x["q"]).to(dt).pin_memory()
        kh = torch.from_numpy(x["k"]).to(dt).pin_memory()
        vh = torch.from_numpy(x["v"]).to(dt).pin_memory()
        mh = None if x["mask"] is None else torch.from_numpy(x["mask"]).pin_memory()
        wh = None if x["conv_w"] is None else torch.from_numpy(x["conv_w"]).pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        for _ in range(2):
            nys.forward_host(qh, kh, vh, mask=mh, conv_w=wh, m=w.m, n_iter=w.n_iter, out=oh)
        if world > 1:
            dist.barrier()
        e_ms = 0.0
        for _ in range(args.e2e_steps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            nys.forward_host(qh, kh, vh, mask=mh, conv_w=wh, m=w.m, n_iter=w.n_iter, out=oh)
            b.record(stream)
            b.synchronize()
            e_ms += a.elapsed_time(b)
        e_ms = max_over_ranks(e_ms, world, "cuda")
        elt = qh.element_size()
        h2d = 3 * qh.numel() * elt + (0 if mh is None else mh.numel()) + (0 if wh is None else wh.numel() * 4)
        e2e = {"value": round(job_throughput(w.tokens, world, args.e2e_steps, e_ms), 1), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(oh.numel() * elt),
               "steps": args.e2e_steps, "ms_per_step": round(e_ms / args.e2e_steps, 3)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not use_ex:
        cpu = cpu_baseline(w, x)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded numpy inputs, see workloads/)",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "d": w.d, "m": w.m,
                       "n_iter": w.n_iter, "conv": w.conv, "mask": w.lengths is not None,
                       "inputs": w.dist, "parallelism": "replicas" if world > 1 else "single",
                       "path": args.path, "inv_init": args.inv_init,
                       "l2": "not flushed" if args.no_flush else
                       "flushed before every step (256 MiB write, then a 256 MiB read of another buffer; untimed)"},
            "roofline": roof,
            "step_roofline": {"t_roof_us": round(t_roof * 1e6, 2), "frac": round(t_roof / (ms_per_step * 1e-3), 4),
                              "ideal_bytes": ideal_bytes, "flops": total_flops},
            "step_roofline_pipes": {"t_roof_us": round(t_pipes * 1e6, 2),
                                    "frac": round(t_pipes / (ms_per_step * 1e-3), 4),
                                    "note": "inverse (and kernel_2) at the tf32 tensor rate, the rest at bf16"},
            "step_roofline_exp": {"t_roof_us": round(t_exp_roof * 1e6, 2),
                                  "frac": round(t_exp_roof / (ms_per_step * 1e-3), 4),
                                  "t_exp_us": round(t_exp * 1e6, 2),
                                  "exponentials": step_exponentials(w, args.path),
                                  "note": "pipe-aware bound with every softmax exponential on the MUFU "
                                          f"unit at {MUFU_EX2_PER_CLK_SM}/clk/SM"},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
            "kernels": kernels,
            "kernels_source": f"separate untimed pass of {breakdown_steps} steps, every launch bracketed by "
                              "CUDA events; the timed loop brackets only the roofline kernel, in its last tenth of steps",
            "clocks": clocks, "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

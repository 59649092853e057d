"""Multi-process (N > 1) host logic of bench.py, on CPU with the gloo backend.

The forward has no exchange step, so N GPUs run N independent replicas; what
N > 1 adds is host plumbing: the rank environment, a barrier, the max over
ranks of the device-timed region, the whole-job throughput, and that rank 0
alone prints the JSON line. These tests run that plumbing as two gloo ranks
on 127.0.0.1; the NCCL path in bench.py calls the same helpers with
device "cuda".
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, times):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, local = bench.rank_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        total_ms = bench.max_over_ranks(times[r], w, "cpu")
        value = bench.job_throughput(1000, w, 4, total_ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "local": local, "total_ms": total_ms, "value": value}, f)


def test_rank_env_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5


def test_job_throughput_counts_every_rank():
    # 2 ranks x 3 steps x 1000 tokens in 6 ms of the slowest rank
    assert bench.job_throughput(1000, 2, 3, 6.0) == pytest.approx(1e6)


def test_max_over_ranks_gloo_world2(tmp_path):
    times = [12.5, 20.25]          # rank 1 is the slower one
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path), times), nprocs=2,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, x in enumerate(res):
        assert (x["world"], x["rank"], x["local"]) == (2, r, r)
        assert x["total_ms"] == 20.25                   # every rank sees the max
        assert x["value"] == pytest.approx(1000 * 2 * 4 / 20.25e-3)


def test_reference_arm_under_torchrun_world2():
    """torchrun with 2 ranks: every rank exits 0 and only rank 0 prints one JSON line."""
    env = dict(os.environ, NYS_REFERENCE_BUDGET_S="5", OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "2", "--warmup", "3", "--workload", "tiny_f32"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["workload"] == "tiny_f32"
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_kernel_source_digests_resolve():
    """Every kernel's traffic-validity digest finds its headers and launch functions, and
    differs from the digest of another kernel's sources."""
    digests = {k: bench.source_digest(k) for k in bench.KERNEL_SOURCES}
    assert all(len(d) == 16 for d in digests.values())
    assert digests["pinv"] != digests["output"] != digests["k3v_partial"]
    with open(os.path.join(ROOT, "nystr_self_attention_scale_b200", "csrc", "nys_attn.cu")) as f:
        src = f.read()
    text = bench._function_text(src, "launch_pinv_pair")
    assert text.lstrip().startswith("int launch_pinv_pair(") and text.rstrip().endswith("}")

"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare element by element.

Tolerances (element-wise over the whole output, after converting the GPU
result to float64):
  float32 path: max |gpu - oracle| <= 2e-3 and ||gpu - oracle||_F / ||oracle||_F <= 1e-4
  bf16 path:    ||gpu - oracle||_F / ||oracle||_F <= 2e-2 (bf16 in/out, fp32 accumulate)
"""
from __future__ import annotations

import numpy as np

TOL = {"f32": dict(max_abs=2e-3, rel_f=1e-4), "bf16": dict(max_abs=None, rel_f=2e-2)}

# (what, max-abs, rel-F) of every comparison made in this session, printed at the end of the
# run (tests/conftest.py), so that a GPU run's log records the measured errors.
MEASURED = []


def note(what, max_abs, rel_f):
    MEASURED.append((what, float(max_abs), float(rel_f)))


def to_device(x, torch):
    dt = torch.float32 if x["dtype"] == "f32" else torch.bfloat16
    dev = dict(q=torch.from_numpy(x["q"]).to(dt).cuda(), k=torch.from_numpy(x["k"]).to(dt).cuda(),
               v=torch.from_numpy(x["v"]).to(dt).cuda())
    dev["mask"] = None if x["mask"] is None else torch.from_numpy(x["mask"]).cuda()
    dev["conv_w"] = None if x["conv_w"] is None else torch.from_numpy(x["conv_w"]).cuda()
    return dev


def gpu_forward(x, nys, torch, m=None, n_iter=None, debug=False):
    dev = to_device(x, torch)
    kw = dict(mask=dev["mask"], conv_w=dev["conv_w"], m=m or x["m"],
              n_iter=x["n_iter"] if n_iter is None else n_iter)
    if debug:
        out, st = nys.forward_debug(dev["q"], dev["k"], dev["v"], **kw)
        torch.cuda.synchronize()
        return out, {k_: t.cpu().numpy().astype(np.float64) for k_, t in st.items()}
    out = nys.forward(dev["q"], dev["k"], dev["v"], **kw)
    torch.cuda.synchronize()
    return out


def oracle_heads(x, oracle, heads, rows=None, m=None, n_iter=None, stages=False):
    """Oracle output for a list of (b, h) heads: [len(heads), n_rows, d] (+ stages)."""
    outs, sts = [], []
    for b, h in heads:
        r = oracle.forward(x["q"][b:b + 1, h:h + 1], x["k"][b:b + 1, h:h + 1],
                           x["v"][b:b + 1, h:h + 1],
                           None if x["mask"] is None else x["mask"][b:b + 1],
                           None if x["conv_w"] is None else x["conv_w"][h:h + 1],
                           m=m or x["m"], n_iter=x["n_iter"] if n_iter is None else n_iter,
                           rows=rows, stages=stages)
        if stages:
            outs.append(r[0][0, 0])
            sts.append({k: v[0, 0] for k, v in r[1].items()})
        else:
            outs.append(r[0, 0])
    return (np.stack(outs), sts) if stages else np.stack(outs)


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    return float(np.max(np.abs(diff))), float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got, ref, dtype, what=""):
    tol = TOL[dtype]
    max_abs, rel_f = errors(got, ref)
    note(what, max_abs, rel_f)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert rel_f <= tol["rel_f"], f"{what}: rel-F {rel_f:.3e} > {tol['rel_f']:.1e} (max-abs {max_abs:.3e})"
    if tol["max_abs"] is not None:
        assert max_abs <= tol["max_abs"], f"{what}: max-abs {max_abs:.3e} > {tol['max_abs']:.1e}"
    return max_abs, rel_f


def sample_rows(n, lengths=None, count=48, seed=0):
    """Rows covering the ends, 128-row tile edges, the valid-length edges and random rows."""
    rs = {0, 1, n - 1, n - 2, min(127, n - 1), min(128, n - 1), n // 2}
    if lengths is not None:
        for L in lengths:
            for r in (int(L) - 1, int(L), int(L) + 1):
                if 0 <= r < n:
                    rs.add(r)
    rng = np.random.default_rng(seed)
    rs.update(int(r) for r in rng.integers(0, n, size=count))
    return sorted(rs)

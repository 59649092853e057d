"""The allocation-free entry point nys_attn_pinv_static.

nys_attn_pinv_static exists for callers that cannot allocate device memory
(for example an application that reserves all GPU memory up front and
forbids later allocations, or a loop that cannot afford an allocation's
latency or its failure): its scratch is a fixed array inside the library
instead of a cudaMallocAsync workspace. Here it is called through the C ABI
on the float32 landmarks that nys_attn_forward_debug produced, twice in a
row, and its Z must match:
  - the fp64 oracle's Z for the same landmarks (kernel_2 = softmax of the
    landmark product, then the iterative inverse, walkthrough 2.4 and 2.5),
    within the float32 parity bar: relative Frobenius <= 1e-4, and max-abs
    <= 1e-4 of the largest |Z| entry (Z's entries reach the hundreds on the
    degenerate case, so an absolute bound on them says nothing);
  - the Z of the regular float32 entry point, within the same bar;
and the second call must leave the device's free memory unchanged.

This file is collected last on purpose, so that a stop-at-first-failure run
has already run every other test when it gets here.
"""
import ctypes
import dataclasses

import numpy as np
import pytest

from parity import errors, note, to_device
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

REL_F = 1e-4          # the float32 parity bar
MAX_ABS_REL = 1e-4    # max |error| relative to max |Z|


@pytest.fixture(scope="module")
def nys():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nystr_self_attention_scale_b200 as nys_mod
    return nys_mod


def _call_static(nys, q_l, k_l, n_iter):
    B, H, m, d = q_l.shape
    z = torch.full((B, H, m, m), float("nan"), device="cuda", dtype=torch.float32)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    rc = nys.lib.nys_attn_pinv_static(ctypes.c_void_p(q_l.data_ptr()), ctypes.c_void_p(k_l.data_ptr()),
                                      ctypes.c_void_p(z.data_ptr()), B * H, m, d, n_iter,
                                      ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, nys.strerror(rc)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    return z, free_before, free_after


def _oracle_z(oracle_mod, q_l, k_l, n_iter, heads):
    """Z of the fp64 oracle from the same float32 landmarks, for the listed heads."""
    out = []
    for b, h in heads:
        ql = q_l[b, h].astype(np.float64)
        kl = k_l[b, h].astype(np.float64)
        k2 = oracle_mod.softmax_rows(ql @ kl.T)
        out.append(oracle_mod.iterative_inv(k2, n_iter))
    return np.stack(out)


def _check(got, ref, what):
    max_abs, rel = errors(got, ref)
    note(what, max_abs, rel)
    assert np.isfinite(got).all(), what
    assert rel <= REL_F, f"{what}: rel-F {rel:.3e}"
    assert max_abs <= MAX_ABS_REL * np.abs(ref).max(), f"{what}: max-abs {max_abs:.3e}"


@pytest.mark.parametrize("name,kw,heads", [
    ("default_f32_masked", dict(B=2, H=3), [(0, 0), (0, 2), (1, 1)]),   # m = 64, one launch
    # m = 256, 16 heads: three launches of at most 6 heads; heads on both sides of a boundary
    ("corr_f32", dict(B=2, H=8, n=4096), [(0, 0), (0, 5), (0, 6), (1, 7)]),
    ("degenerate_f32_it24", dict(), [(0, 0)]),                          # m = n = 256, 24 iterations
])
def test_static_scratch_matches_oracle_and_regular_entry_point(nys, oracle_mod, name, kw, heads):
    if name == "corr_f32":
        w = dataclasses.replace(WORKLOADS["n16384_bf16_corr"], name=name, dtype="f32")
    else:
        w = WORKLOADS[name]
    x = make_inputs(w, seed=11, **kw)
    dev = to_device(x, torch)
    _, st = nys.forward_debug(dev["q"], dev["k"], dev["v"], mask=dev["mask"], conv_w=dev["conv_w"],
                              m=w.m, n_iter=w.n_iter)
    torch.cuda.synchronize()
    regular = st["z"].double().cpu().numpy()
    q_l = st["q_l"].cpu().numpy()
    k_l = st["k_l"].cpu().numpy()
    ref = _oracle_z(oracle_mod, q_l, k_l, w.n_iter, heads)
    first, _, _ = _call_static(nys, st["q_l"], st["k_l"], w.n_iter)
    second, free_before, free_after = _call_static(nys, st["q_l"], st["k_l"], w.n_iter)
    assert free_after == free_before, (free_before, free_after)
    for tag, z in (("first", first), ("second", second)):
        z = z.double().cpu().numpy()
        got = np.stack([z[b, h] for b, h in heads])
        _check(got, ref, f"{name} {tag} call vs oracle")
        _check(z, regular, f"{name} {tag} call vs the regular entry point")
    assert torch.equal(first, second)


def test_static_scratch_rejects_bad_arguments(nys):
    q = torch.zeros(1, 1, 64, 64, device="cuda")
    z = torch.zeros(1, 1, 64, 64, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert nys.lib.nys_attn_pinv_static(None, p(q), p(z), 1, 64, 64, 6, None) == -1
    assert nys.lib.nys_attn_pinv_static(p(q), p(q), p(z), 0, 64, 64, 6, None) == -1
    assert nys.lib.nys_attn_pinv_static(p(q), p(q), p(z), 1, 64, 48, 6, None) == -2
    assert nys.lib.nys_attn_pinv_static(p(q), p(q), p(z), 1, 512, 64, 6, None) == -2
    assert nys.device_status() == 0

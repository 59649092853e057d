"""The allocation-free entry point nys_attn_pinv_static against the regular path.

nys_attn_pinv_static exists for callers that cannot allocate device memory
(for example an application that reserves all GPU memory up front and
forbids later allocations): its scratch is a fixed array inside the library
instead of a cudaMallocAsync workspace. Here it is called through the C ABI
on landmarks produced by nys_attn_forward_debug, twice in a row, and its Z
must match the Z that the regular entry point computed, within the float32
parity tolerance (max-abs 2e-3, relative Frobenius 1e-4).

This file is collected last on purpose, so that a stop-at-first-failure run
has already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest

from parity import TOL, errors, to_device
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


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
    rc = nys.lib.nys_attn_pinv_static(ctypes.c_void_p(q_l.data_ptr()), ctypes.c_void_p(k_l.data_ptr()),
                                      ctypes.c_void_p(z.data_ptr()), B * H, m, d, n_iter,
                                      ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, nys.strerror(rc)
    torch.cuda.synchronize()
    return z


# float32 workloads: there the regular entry point runs the same float32 inverse that
# nys_attn_pinv_static runs (the bf16 path uses a tf32 tensor-core inverse instead).
@pytest.mark.parametrize("name,kw", [
    ("default_f32_masked", dict(B=2, H=3)),                 # m = 64, one launch
    ("corr_f32", dict(B=2, H=8, n=4096)),                   # m = 256, 16 heads: several batches
    ("degenerate_f32_it24", dict()),                         # m = n = 256, 24 iterations
])
def test_static_scratch_matches_regular_entry_point(nys, name, kw):
    import dataclasses
    if name == "corr_f32":
        w = dataclasses.replace(WORKLOADS["n16384_bf16_corr"], name=name, dtype="f32")
    else:
        w = WORKLOADS[name]
    x = make_inputs(w, seed=11, **kw)
    dev = to_device(x, torch)
    _, st = nys.forward_debug(dev["q"], dev["k"], dev["v"], mask=dev["mask"], conv_w=dev["conv_w"],
                              m=w.m, n_iter=w.n_iter)
    torch.cuda.synchronize()
    ref = st["z"].double().cpu().numpy()
    first = _call_static(nys, st["q_l"], st["k_l"], w.n_iter).double().cpu().numpy()
    second = _call_static(nys, st["q_l"], st["k_l"], w.n_iter).double().cpu().numpy()
    for got in (first, second):
        assert np.isfinite(got).all()
        max_abs, rel = errors(got, ref)
        assert rel <= TOL["f32"]["rel_f"] and max_abs <= TOL["f32"]["max_abs"], (max_abs, rel)
    np.testing.assert_array_equal(first, second)


def test_static_scratch_rejects_bad_arguments(nys):
    q = torch.zeros(1, 1, 64, 64, device="cuda")
    z = torch.zeros(1, 1, 64, 64, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert nys.lib.nys_attn_pinv_static(None, p(q), p(z), 1, 64, 64, 6, None) == -1
    assert nys.lib.nys_attn_pinv_static(p(q), p(q), p(z), 0, 64, 64, 6, None) == -1
    assert nys.lib.nys_attn_pinv_static(p(q), p(q), p(z), 1, 64, 48, 6, None) == -2
    assert nys.lib.nys_attn_pinv_static(p(q), p(q), p(z), 1, 512, 64, 6, None) == -2
    assert nys.device_status() == 0

"""Index safety of the kernels: the workspace guard mode and guarded caller buffers.

compute-sanitizer is not available on the GPUs these tests run on, so the
index safety of the hand-written kernels is checked here, on small shapes that
still span several tiles and a ragged tail, in two ways:
  - the workspace guard mode (nys_attn_set_workspace_guard): every workspace
    buffer lies between guard zones, the workspace starts as 0xFF bytes (NaN),
    and a check after the call records NYS_ERR_GUARD in the device status word
    if a guard byte changed;
  - every caller buffer sits inside a larger allocation: inputs between NaN
    margins (the key mask between margins of 0, a padded key), so a read past
    either end of a buffer reaches the output; outputs between sentinel
    margins, which must come back unchanged.
The guarded call must return exactly (bitwise) what the unguarded call returns,
all of it finite, and both are compared with the oracle at the usual parity
bars (float32 max-abs 2e-3 and rel-F 1e-4; bf16 rel-F 2e-2).
"""
import ctypes
import dataclasses

import numpy as np
import pytest

from parity import assert_close, to_device
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MARGIN = 4096          # elements on each side of a guarded buffer (keeps 16-byte alignment)
SENTINEL = 7.0         # exactly representable in float32 and bf16


@pytest.fixture(scope="module")
def nys():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nystr_self_attention_scale_b200 as nys_mod
    assert nys_mod.device_status() == 0
    yield nys_mod
    nys_mod.set_workspace_guard(False)


def _embed(t, fill):
    """A copy of t inside a flat allocation with MARGIN elements of `fill` on each side."""
    flat = torch.full((t.numel() + 2 * MARGIN,), fill, dtype=t.dtype, device=t.device)
    flat[MARGIN:MARGIN + t.numel()] = t.reshape(-1)
    return flat, flat[MARGIN:MARGIN + t.numel()].view(t.shape)


def _margins_intact(flat, fill):
    ref = torch.full((MARGIN,), fill, dtype=flat.dtype, device=flat.device)
    return torch.equal(flat[:MARGIN], ref) and torch.equal(flat[-MARGIN:], ref)


def _call(nys, q, k, v, mask, conv_w, x, out, probs, inv_init, exact):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    B, H, n, d = q.shape
    rc = nys.lib.nys_attn_forward_ex(p(q), p(k), p(v), p(mask), p(conv_w), B, H, n, d, x["m"], x["n_iter"],
                                     nys.F32 if x["dtype"] == "f32" else nys.BF16, inv_init, 1 if exact else 0,
                                     p(out), p(probs), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, nys.strerror(rc)


def _run_both(nys, x, want_probs, inv_init, exact):
    dev = to_device(x, torch)
    q, k, v = dev["q"], dev["k"], dev["v"]
    B, H, n, d = q.shape
    pw = n if exact else x["m"]
    # unguarded, plain buffers
    out0 = torch.empty_like(q)
    probs0 = torch.empty(B, H, n, pw, device="cuda") if want_probs else None
    nys.set_workspace_guard(False)
    _call(nys, q, k, v, dev["mask"], dev["conv_w"], x, out0, probs0, inv_init, exact)
    torch.cuda.synchronize()
    # guarded: workspace guard mode plus margins around every caller buffer
    nan = float("nan")
    gq, gk, gv = (_embed(t, nan) for t in (q, k, v))
    gmask = None if dev["mask"] is None else _embed(dev["mask"], 0)
    gconv = None if dev["conv_w"] is None else _embed(dev["conv_w"], nan)
    gout = _embed(torch.empty_like(q), SENTINEL)
    gprobs = _embed(torch.empty(B, H, n, pw, device="cuda"), SENTINEL) if want_probs else None
    assert not nys.set_workspace_guard(True)
    try:
        _call(nys, gq[1], gk[1], gv[1], None if gmask is None else gmask[1], None if gconv is None else gconv[1],
              x, gout[1], None if gprobs is None else gprobs[1], inv_init, exact)
        torch.cuda.synchronize()
    finally:
        nys.set_workspace_guard(False)
    assert nys.device_status() == 0, "a workspace guard zone was overwritten"
    assert _margins_intact(gout[0], SENTINEL), "the output's margins changed"
    if want_probs:
        assert _margins_intact(gprobs[0], SENTINEL), "the attention weights' margins changed"
    for t, f in ((gq, nan), (gk, nan), (gv, nan), (gconv, nan), (gmask, 0)):
        if t is not None and f == 0:
            assert _margins_intact(t[0], 0)
        elif t is not None:
            assert torch.isnan(t[0][:MARGIN]).all() and torch.isnan(t[0][-MARGIN:]).all()
    out1 = gout[1]
    assert torch.isfinite(out1).all()
    assert torch.equal(out1, out0), "guarded and unguarded calls differ"
    if want_probs:
        assert torch.isfinite(gprobs[1]).all()
        assert torch.equal(gprobs[1], probs0)
    return out1, (gprobs[1] if want_probs else None)


CASES = [
    # name, make_inputs overrides, output_attentions, inv_init, exact
    ("tiny_f32", dict(), False, 0, False),                             # float32, m = 64, one head
    ("default_f32_masked", dict(B=2, H=2), True, 0, False),            # float32, masked, weights
    ("sweep_n1024_conv", dict(B=2, H=2), False, 0, False),             # bf16, m = 64
    ("longcls_bf16_masked", dict(B=2, n=1024), True, 0, False),        # bf16, m = 128, masked, d = 32
    ("n16384_bf16_corr", dict(B=1, H=2, n=2048), False, 0, False),     # bf16, m = 256, CTA pairs
    ("n16384_bf16_corr", dict(B=1, H=2, n=2048), True, 1, False),      # exact coefficient, weights
    ("exact_f32_ragged", dict(B=1, H=2, n=200), True, 0, True),        # path A, ragged n
    ("exact_bf16_masked", dict(B=2, H=2, n=1024), False, 0, True),     # path A, bf16
]


@pytest.mark.parametrize("name,kw,want_probs,inv_init,exact", CASES, ids=[
    f"{c[0]}{'-weights' if c[2] else ''}{'-exactinit' if c[3] else ''}" for c in CASES])
def test_guarded_call_is_exact_and_in_bounds(nys, oracle_mod, name, kw, want_probs, inv_init, exact):
    if name == "exact_f32_ragged":
        w = dataclasses.replace(WORKLOADS["tiny_f32"], lengths=(1, 200), zero_pad=True)
    elif name == "exact_bf16_masked":
        w = dataclasses.replace(WORKLOADS["tiny_f32"], dtype="bf16", lengths=(300, 1024), zero_pad=True)
    else:
        w = WORKLOADS[name]
    x = make_inputs(w, seed=41, **kw)
    out, probs = _run_both(nys, x, want_probs, inv_init, exact)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], x["conv_w"], m=x["m"], n_iter=x["n_iter"],
                           init_option=inv_init, exact=exact, probs=want_probs)
    ref, st = (r[0], r[1]) if want_probs else (r, None)
    assert_close(out.double().cpu().numpy(), ref, x["dtype"], f"guarded {name}")
    if want_probs:
        tol = "f32" if (exact or x["dtype"] == "f32") else "bf16"
        assert_close(probs.double().cpu().numpy(), st["probs"], tol, f"guarded {name} weights")


def test_guard_check_detects_a_changed_byte(nys):
    """The check itself: a clean buffer passes, one byte changed in a zone is reported."""
    assert nys.selftest_guard(False) == nys.OK
    assert nys.selftest_guard(True) == nys.ERR_GUARD
    assert nys.device_status() == 0   # the self-test read and cleared the word


def test_guard_mode_switch_and_workspace_size(nys):
    plain = nys.workspace_bytes(1, 2, 2048, 64, 256)
    assert not nys.set_workspace_guard(True)
    try:
        guarded = nys.workspace_bytes(1, 2, 2048, 64, 256)
        assert nys.set_workspace_guard(True)   # returns the previous setting
    finally:
        nys.set_workspace_guard(False)
    assert guarded - plain == 16 * 4096    # 15 buffers on the bf16 m = 256 path + a trailing zone
    assert nys.workspace_bytes(1, 2, 2048, 64, 256) == plain

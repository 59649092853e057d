"""GPU parity of the layer's other options, through nys_attn_forward_ex, against the oracle.

  - the exact Z_0 coefficient (walkthrough 2.5, second bullet; inv_coeff_init_option)
  - the exact branch, path A (walkthrough 2.1): softmax(Qs Ks^T + mask) V + conv
  - the attention weights returned for output_attentions (walkthrough 2.7)

Tolerances are the parity bars of tests/parity.py: float32 max-abs 2e-3 and
rel-F 1e-4; bf16 rel-F 2e-2.
"""
import dataclasses

import numpy as np
import pytest

from parity import assert_close, errors, note, sample_rows, to_device
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def nys():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nystr_self_attention_scale_b200 as nys_mod
    return nys_mod


@pytest.fixture(scope="module", autouse=True)
def _status_clean(nys):
    yield
    assert nys.device_status() == 0


def _run(nys, x, **kw):
    dev = to_device(x, torch)
    r = nys.forward_ex(dev["q"], dev["k"], dev["v"], mask=dev["mask"], conv_w=dev["conv_w"],
                       m=x["m"], n_iter=x["n_iter"], **kw)
    torch.cuda.synchronize()
    return r


def _oracle(oracle_mod, x, rows=None, **kw):
    return oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], x["conv_w"], m=x["m"],
                              n_iter=x["n_iter"], rows=rows, **kw)


# ------------------------------------------------------------------ exact Z_0 coefficient

@pytest.mark.parametrize("name,kw", [
    ("default_f32_masked", dict(B=2, H=2)),            # float32, m = 64
    ("sweep_n1024_conv", dict(B=2, H=2)),              # bf16, m = 64 (tensor-core inverse)
    ("longcls_bf16_masked", dict(B=2, n=1024)),        # bf16, m = 128
    ("n16384_bf16_corr", dict(B=1, H=2, n=2048)),      # bf16, m = 256 (CTA-pair inverse)
])
def test_exact_coefficient_matches_oracle(nys, oracle_mod, name, kw):
    x = make_inputs(WORKLOADS[name], seed=31, **kw)
    out = _run(nys, x, inv_coeff_init_option=True)
    ref = _oracle(oracle_mod, x, init_option=1)
    assert_close(out.double().cpu().numpy(), ref, x["dtype"], f"inv_init exact {name}")


# ------------------------------------------------------------------ exact branch (path A)

@pytest.mark.parametrize("dtype,B,H,n,d,lengths,conv", [
    ("f32", 2, 2, 512, 64, (200, 512), True),
    ("f32", 1, 3, 200, 32, (1, 200), True),      # ragged n, a sequence with one valid key
    ("f32", 1, 1, 96, 64, None, False),
    ("bf16", 2, 2, 1024, 64, (300, 1024), True),
    ("bf16", 1, 2, 4096, 32, (1024, 4096), True),
    ("bf16", 2, 1, 256, 64, None, False),
])
def test_exact_branch_matches_oracle(nys, oracle_mod, dtype, B, H, n, d, lengths, conv):
    w = dataclasses.replace(WORKLOADS["tiny_f32"], dtype=dtype, d=d, lengths=lengths,
                            zero_pad=lengths is not None, conv=conv)
    x = make_inputs(w, seed=32, B=B, H=H, n=n)
    out = _run(nys, x, exact=True)
    ref = _oracle(oracle_mod, x, exact=True)
    assert_close(out.double().cpu().numpy(), ref, dtype,
                 f"exact branch {dtype} B{B} H{H} n{n} d{d} lengths{lengths} conv{conv}")


def test_exact_branch_long_sequence_sampled(nys, oracle_mod):
    """n = 16384 bf16: two key splits per row block; sampled rows of two heads."""
    w = dataclasses.replace(WORKLOADS["n16384_bf16_corr"], dist="iid")
    x = make_inputs(w, seed=33, B=1, H=2, n=16384)
    out = _run(nys, x, exact=True)
    rows = sample_rows(x["n"])
    ref = _oracle(oracle_mod, x, rows=rows, exact=True)
    assert_close(out[:, :, rows].double().cpu().numpy(), ref, "bf16", "exact branch n=16384 sampled rows")


def test_exact_branch_equals_converged_nystrom_at_m_equals_n(nys):
    """m = n with a converged inverse is path A (A A^+ A = A): the GPU's two paths agree."""
    x = make_inputs(WORKLOADS["degenerate_f32_it24"], seed=0)
    dev = to_device(x, torch)
    a = nys.forward_ex(dev["q"], dev["k"], dev["v"], exact=True)
    b = nys.forward(dev["q"], dev["k"], dev["v"], m=256, n_iter=24)
    torch.cuda.synchronize()
    assert_close(b.double().cpu().numpy(), a.double().cpu().numpy(), "f32", "m=n Nystrom vs exact branch")


def test_exact_branch_ignores_landmark_arguments(nys):
    x = make_inputs(WORKLOADS["tiny_f32"], seed=34, n=256)
    dev = to_device(x, torch)
    a = nys.forward_ex(dev["q"], dev["k"], dev["v"], conv_w=dev["conv_w"], m=64, exact=True)
    b = nys.forward_ex(dev["q"], dev["k"], dev["v"], conv_w=dev["conv_w"], m=7, n_iter=0, exact=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------------------------------ attention weights

@pytest.mark.parametrize("name,kw,tol", [
    ("tiny_f32", dict(), "f32"),
    ("default_f32_masked", dict(B=2, H=2), "f32"),
    ("sweep_n1024_conv", dict(B=1, H=2), "bf16"),
    ("longcls_bf16_masked", dict(B=2, n=1024), "bf16"),
    ("n16384_bf16_corr", dict(B=1, H=2, n=2048), "bf16"),
])
def test_nystrom_attention_weights_match_oracle(nys, oracle_mod, name, kw, tol):
    """kernel_1 Z ([n, m] per head). On the bf16 path Z comes from the tf32 inverse, so the
    bf16 bar applies; the output itself is unchanged by asking for the weights."""
    x = make_inputs(WORKLOADS[name], seed=35, **kw)
    out, probs = _run(nys, x, output_attentions=True)
    plain = _run(nys, x)
    assert torch.equal(out, plain)
    _, st = _oracle(oracle_mod, x, probs=True)
    assert_close(probs.double().cpu().numpy(), st["probs"], tol, f"attention weights {name}")


@pytest.mark.parametrize("dtype,n,lengths", [("f32", 512, (100, 512)), ("bf16", 1024, (300, 1024))])
def test_exact_attention_weights_match_oracle(nys, oracle_mod, dtype, n, lengths):
    """softmax(Qs Ks^T + mask) ([n, n] per head), computed in float32 from the inputs: the
    float32 bar applies to both input types; padded keys get exactly 0."""
    w = dataclasses.replace(WORKLOADS["tiny_f32"], dtype=dtype, lengths=lengths, zero_pad=True)
    x = make_inputs(w, seed=36, B=2, H=2, n=n)
    out, probs = _run(nys, x, exact=True, output_attentions=True)
    _, st = _oracle(oracle_mod, x, exact=True, probs=True)
    got = probs.double().cpu().numpy()
    assert_close(got, st["probs"], "f32", f"exact attention weights {dtype} n{n}")
    for b in range(2):
        assert np.all(got[b][:, :, x["mask"][b] == 0] == 0.0)
    rs = got.sum(-1)
    ma, rel = errors(rs, np.ones_like(rs))
    note(f"exact weights row sums {dtype}", ma, rel)
    assert ma < 1e-5

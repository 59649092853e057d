"""Pins of the fp64 CPU oracle against facts the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a closed
form, an invariant, a textbook or library routine, or brute force on a
special case. Together they are chosen so that a dropped term, a wrong sign,
index or axis, or a transposed operand anywhere in the oracle fails at least
one of them. Citations name "Nystromformer source walkthrough"
(blog.gitcode.com) and its sections.
"""
import dataclasses

import numpy as np
import pytest
import scipy.special
import torch

from workloads import WORKLOADS, make_inputs


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- landmarks (2.2, 2.3)

@pytest.mark.parametrize("n,m,d", [(512, 64, 64), (4096, 128, 32), (256, 256, 64), (64, 4, 8)])
def test_landmarks_ramp_closed_form(oracle_mod, n, m, d):
    """Segment means of the ramp x[i, c] = i + 1000 c, scaled by d^-1/4 (2.2, 2.3)."""
    i = np.arange(n)[:, None]
    c = np.arange(d)[None, :]
    x = (i + 1000 * c).astype(np.float32)
    L = n // m
    j = np.arange(m)[:, None]
    expect = (j * L + (L - 1) / 2.0 + 1000.0 * c) * d ** -0.25
    got = oracle_mod.landmarks(x, m)
    np.testing.assert_allclose(got, expect, rtol=1e-14, atol=1e-12)


@pytest.mark.parametrize("n,m", [(512, 64), (64, 8), (256, 256)])
def test_landmarks_one_hot_membership(oracle_mod, n, m):
    """A single one-hot token t lands in landmark floor(t / L) only (2.3)."""
    d = 8
    L = n // m
    for t in (0, 1, L - 1, L, n // 2 + 3, n - 1):
        x = np.zeros((n, d), np.float32)
        x[t, 5] = 1.0
        got = oracle_mod.landmarks(x, m)
        nz = np.argwhere(got != 0)
        assert nz.tolist() == [[t // L, 5]]
        assert got[t // L, 5] == pytest.approx(d ** -0.25 / L, rel=1e-15)


# ---------------------------------------------------------------- softmax (2.4)

def test_softmax_matches_library_and_sums_to_one(oracle_mod):
    s = _rng(1).standard_normal((37, 129)) * 4
    got = oracle_mod.softmax_rows(s)
    np.testing.assert_allclose(got, scipy.special.softmax(s, axis=1), rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(got.sum(1), 1.0, atol=1e-12)


def test_softmax_mask_entries_are_exact_zero(oracle_mod):
    s = _rng(2).standard_normal((9, 50))
    keep = (_rng(3).random(50) > 0.4).astype(np.uint8)
    keep[0] = 1
    got = oracle_mod.softmax_rows(s, keep)
    assert np.all(got[:, keep == 0] == 0.0)
    ref = scipy.special.softmax(s[:, keep == 1], axis=1)
    np.testing.assert_allclose(got[:, keep == 1], ref, rtol=1e-13)


# ---------------------------------------------------------------- pseudoinverse (2.5)

def _phi_closed_form(a, c, n_iter):
    """Z_k = V diag(g_k) U^T with A = U S V^T, g_0 = c s, phi = s g,
    g_{k+1} = g_k (13 - 15 phi + 7 phi^2 - phi^3) / 4 (derived from the update of 2.5)."""
    u, sv, vt = np.linalg.svd(a)
    g = c * sv
    for _ in range(n_iter):
        phi = sv * g
        g = g * (13 - 15 * phi + 7 * phi ** 2 - phi ** 3) / 4
    return vt.T @ np.diag(g) @ u.T


def _kernel2_like(m, seed, scale=1.0):
    s = _rng(seed).standard_normal((m, m)) * scale
    return scipy.special.softmax(s, axis=1)


@pytest.mark.parametrize("m,n_iter,seed", [(16, 6, 0), (64, 6, 1), (64, 0, 2), (64, 1, 3),
                                           (128, 6, 4), (33, 11, 5)])
def test_iterative_inv_svd_closed_form(oracle_mod, m, n_iter, seed):
    a = _kernel2_like(m, seed)
    c = 1.0 / (np.linalg.norm(a, 1) * np.linalg.norm(a, np.inf))
    z = oracle_mod.iterative_inv(a, n_iter)
    ref = _phi_closed_form(a, c, n_iter)
    assert np.linalg.norm(z - ref) <= 1e-10 * np.linalg.norm(ref)


def test_iterative_inv_nonsymmetric_general_matrix(oracle_mod):
    """The closed form holds for any nonnegative matrix, not only row-stochastic ones
    (for nonnegative entries the column/row sums are the 1- and inf-norms)."""
    a = _rng(7).random((24, 24)) + 3 * np.eye(24)
    c = 1.0 / (np.linalg.norm(a, 1) * np.linalg.norm(a, np.inf))
    z = oracle_mod.iterative_inv(a, 6)
    ref = _phi_closed_form(a, c, 6)
    assert np.linalg.norm(z - ref) <= 1e-10 * np.linalg.norm(ref)


def test_init_coeff_is_inverse_of_one_times_inf_norm(oracle_mod):
    a = _rng(8).random((40, 40))
    assert oracle_mod.init_coeff(a) == pytest.approx(
        1.0 / (np.linalg.norm(a, 1) * np.linalg.norm(a, np.inf)), rel=1e-14)


def test_init_coeff_exact_is_inverse_of_one_norm(oracle_mod):
    """The exact-coefficient option (walkthrough 2.5, second bullet): c = 1 / ||A||_1."""
    a = _rng(18).random((40, 40))
    assert oracle_mod.init_coeff(a, init_option=1) == pytest.approx(1.0 / np.linalg.norm(a, 1), rel=1e-14)


@pytest.mark.parametrize("n_iter", [0, 1, 6])
def test_iterative_inv_exact_coefficient_closed_form(oracle_mod, n_iter):
    """With Z_0 = A^T / ||A||_1 every iterate is the SVD closed form at c = 1 / ||A||_1. The
    coefficient presumes rows summing to at most 1 (a softmax kernel); this matrix is a
    softmax kernel with rows scaled to sums in [0.5, 0.9], so its column sums, its row sums
    and the two coefficients all differ while the iteration still converges."""
    a = _kernel2_like(24, 19, scale=1.5) * np.linspace(0.5, 0.9, 24)[:, None]
    assert np.linalg.norm(a, 1) > 1.2 * np.linalg.norm(a, np.inf)
    assert abs(oracle_mod.init_coeff(a, 1) / oracle_mod.init_coeff(a, 0) - 1.0) > 0.05
    z = oracle_mod.iterative_inv(a, n_iter, init_option=1)
    ref = _phi_closed_form(a, 1.0 / np.linalg.norm(a, 1), n_iter)
    assert np.linalg.norm(z - ref) <= 1e-10 * np.linalg.norm(ref)


def test_exact_coefficient_on_a_softmax_kernel_is_the_default(oracle_mod):
    """For kernel_2 (rows normalised by the softmax) the row factor of the default
    coefficient is 1, so both options give the same Z up to rounding."""
    a = _kernel2_like(64, 20, scale=2.0)
    z0 = oracle_mod.iterative_inv(a, 6)
    z1 = oracle_mod.iterative_inv(a, 6, init_option=1)
    assert np.linalg.norm(z1 - z0) <= 1e-12 * np.linalg.norm(z0)


def test_iterative_inv_converges_to_library_pinv(oracle_mod):
    """Well-conditioned kernel: many iterations reach numpy's SVD pseudoinverse."""
    s = _rng(9).standard_normal((48, 48)) + 4.0 * np.eye(48)
    a = scipy.special.softmax(s, axis=1)  # diagonal-peaked rows: well conditioned
    assert np.linalg.cond(a) < 50
    z = oracle_mod.iterative_inv(a, 40)
    ref = np.linalg.pinv(a)
    assert np.linalg.norm(z - ref) <= 1e-10 * np.linalg.norm(ref)
    assert np.linalg.norm(a @ z @ a - a) <= 1e-10 * np.linalg.norm(a)


def test_iterative_inv_rank_deficient_converges_to_pinv(oracle_mod):
    """Exactly singular input: the iteration keeps the null space at zero (Moore-Penrose)."""
    blk = _rng(10).random((10, 10)) + 4.0 * np.eye(10)
    a = np.block([[blk, blk], [blk, blk]])  # rank 10 of 20, nonnegative
    z = oracle_mod.iterative_inv(a, 40)
    ref = np.linalg.pinv(a, rcond=1e-9)
    assert np.linalg.norm(z - ref) <= 1e-9 * np.linalg.norm(ref)
    assert np.linalg.norm(z @ a @ z - z) <= 1e-9 * np.linalg.norm(z)


# ---------------------------------------------------------------- conv (2.6)

@pytest.mark.parametrize("n,d", [(512, 64), (40, 8), (65, 3)])
def test_dwconv_matches_torch_conv2d(oracle_mod, n, d):
    r = _rng(11)
    H = 3
    v = r.standard_normal((H, n, d)).astype(np.float32)
    w = (r.standard_normal((H, 65)) * 0.02).astype(np.float32)
    ref = torch.nn.functional.conv2d(torch.from_numpy(v.astype(np.float64))[None],
                                     torch.from_numpy(w.astype(np.float64)).view(H, 1, 65, 1),
                                     padding=(32, 0), groups=H)[0].numpy()
    for h in range(H):
        np.testing.assert_allclose(oracle_mod.dwconv(v[h], w[h]), ref[h], rtol=1e-12, atol=1e-14)


def test_forward_conv_term_is_torch_conv2d(oracle_mod):
    """forward(with conv) - forward(without) equals the library Conv2d of V (2.6)."""
    w = WORKLOADS["tiny_f32"]
    x = make_inputs(w, seed=3, H=2, n=256)
    a = oracle_mod.forward(x["q"], x["k"], x["v"], None, x["conv_w"], m=32)
    b = oracle_mod.forward(x["q"], x["k"], x["v"], None, None, m=32)
    ref = torch.nn.functional.conv2d(torch.from_numpy(x["v"].astype(np.float64)),
                                     torch.from_numpy(x["conv_w"].astype(np.float64)).view(2, 1, 65, 1),
                                     padding=(32, 0), groups=2).numpy()
    np.testing.assert_allclose(a - b, ref, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- whole forward

def _exact_attention(q, k, v, mask=None):
    d = q.shape[-1]
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / np.sqrt(d)
    if mask is not None:
        s = np.where(mask[None, :] > 0, s, -np.inf)
    return scipy.special.softmax(s, axis=1) @ v.astype(np.float64)


def test_m_equals_n_reduces_to_exact_attention(oracle_mod):
    """m = n: landmarks are the rows, k1 = k2 = k3 = A, and A A^+ A = A, so the
    attention term equals softmax(QK^T / sqrt(d)) V once Z has converged (2.1, 2.4)."""
    w = WORKLOADS["degenerate_f32_it24"]
    x = make_inputs(w, seed=0)
    out = oracle_mod.forward(x["q"], x["k"], x["v"], None, None, m=256, n_iter=24)
    ref = _exact_attention(x["q"][0, 0], x["k"][0, 0], x["v"][0, 0])
    rel = np.linalg.norm(out[0, 0] - ref) / np.linalg.norm(ref)
    assert rel < 1e-9


def test_m_equals_n_small_exact(oracle_mod):
    r = _rng(12)
    n, d = 32, 16
    q, k, v = (r.standard_normal((1, 1, n, d)).astype(np.float32) for _ in range(3))
    out = oracle_mod.forward(q, k, v, None, None, m=n, n_iter=30)
    ref = _exact_attention(q[0, 0], k[0, 0], v[0, 0])
    assert np.linalg.norm(out[0, 0] - ref) / np.linalg.norm(ref) < 1e-10


def test_m_equals_n_six_iterations_matches_closed_form(oracle_mod):
    """At the default 6 iterations the m = n output is A Z_6 A V with Z_6 the SVD
    closed form, not yet exact attention."""
    w = WORKLOADS["degenerate_f32_it6"]
    x = make_inputs(w, seed=0)
    out = oracle_mod.forward(x["q"], x["k"], x["v"], None, None, m=256, n_iter=6)
    q, k, v = (x[t][0, 0].astype(np.float64) for t in ("q", "k", "v"))
    a = scipy.special.softmax(q @ k.T / 8.0, axis=1)
    c = 1.0 / (np.linalg.norm(a, 1) * np.linalg.norm(a, np.inf))
    ref = a @ _phi_closed_form(a, c, 6) @ a @ v
    assert np.linalg.norm(out[0, 0] - ref) / np.linalg.norm(ref) < 1e-9


def test_mask_equals_deleting_padded_keys(oracle_mod):
    """kernel_3 with padded keys masked equals kernel_3 over the valid keys only (2.4)."""
    w = WORKLOADS["default_f32_masked"]
    x = make_inputs(w, seed=5, B=2, H=1, n=128)
    _, st = oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], None, m=16, stages=True)
    for b in range(2):
        valid = x["mask"][b] > 0
        ks = x["k"][b, 0][valid].astype(np.float64) * 64 ** -0.25
        p = scipy.special.softmax(st["ql"][b, 0] @ ks.T, axis=1)
        ref = p @ x["v"][b, 0][valid].astype(np.float64)
        np.testing.assert_allclose(st["k3v"][b, 0], ref, rtol=1e-11, atol=1e-13)


def test_linear_in_v(oracle_mod):
    w = WORKLOADS["tiny_f32"]
    x = make_inputs(w, seed=6, n=128)
    # dyadic values with few bits, so 2 v1 - 3 v2 is exact in float32
    v1 = (np.round(x["v"] * 8) / 8).astype(np.float32)
    v2 = (np.round(_rng(13).standard_normal(x["v"].shape) * 8) / 8).astype(np.float32)
    f = lambda v: oracle_mod.forward(x["q"], x["k"], v, None, x["conv_w"], m=16)
    lhs = f((2.0 * v1 - 3.0 * v2).astype(np.float32))
    rhs = 2.0 * f(v1) - 3.0 * f(v2)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-9, atol=1e-10)


def test_heads_independent_and_rows_sampling(oracle_mod):
    w = WORKLOADS["default_f32_masked"]
    x = make_inputs(w, seed=7, B=2, H=3, n=128)
    full = oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], x["conv_w"], m=16)
    for b, h in ((0, 0), (1, 2)):
        one = oracle_mod.forward(x["q"][b:b + 1, h:h + 1], x["k"][b:b + 1, h:h + 1],
                                 x["v"][b:b + 1, h:h + 1], x["mask"][b:b + 1],
                                 x["conv_w"][h:h + 1], m=16)
        np.testing.assert_array_equal(one[0, 0], full[b, h])
    rows = [0, 5, 64, 127]
    part = oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], x["conv_w"], m=16, rows=rows)
    np.testing.assert_allclose(part, full[:, :, rows], rtol=1e-13, atol=1e-15)


def test_kernel_rows_sum_to_one(oracle_mod):
    w = WORKLOADS["default_f32_masked"]
    x = make_inputs(w, seed=8, B=1, H=1, n=128)
    _, st = oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], None, m=16, stages=True)
    np.testing.assert_allclose(st["k2"][0, 0].sum(1), 1.0, atol=1e-12)
    # landmarks of the scaled inputs (2.3) recomputed by numpy reshape-mean
    ql = (x["q"][0, 0].astype(np.float64) * 64 ** -0.25).reshape(16, 8, 64).mean(1)
    np.testing.assert_allclose(st["ql"][0, 0], ql, rtol=1e-13, atol=1e-15)


def test_rejects_bad_shapes(oracle_mod):
    q = np.zeros((1, 1, 100, 8), np.float32)
    with pytest.raises(ValueError):
        oracle_mod.forward(q, q, q, m=64)  # 100 % 64 != 0


# ---------------------------------------------------------------- exact branch (2.1) and the
# returned attention weights (2.7)

def _sdpa(q, k, v, mask=None):
    """torch's scaled_dot_product_attention in float64 (scale 1/sqrt(d)): the library routine
    whose definition path A of walkthrough 2.1 names."""
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    am = None if mask is None else torch.from_numpy(mask[None, :] > 0)
    return torch.nn.functional.scaled_dot_product_attention(t(q)[None], t(k)[None], t(v)[None],
                                                            attn_mask=am)[0].numpy()


@pytest.mark.parametrize("masked", [False, True])
def test_exact_path_is_library_attention_plus_conv(oracle_mod, masked):
    w = dataclasses.replace(WORKLOADS["default_f32_masked"], lengths=(40, 150))
    x = make_inputs(w, seed=21, B=2, H=2, n=192)
    mask = x["mask"] if masked else None
    assert mask is None or (mask == 0).any(axis=1).all()
    out, st = oracle_mod.forward(x["q"], x["k"], x["v"], mask, x["conv_w"], exact=True, probs=True)
    conv = torch.nn.functional.conv2d(torch.from_numpy(x["v"].astype(np.float64)),
                                      torch.from_numpy(x["conv_w"].astype(np.float64)).view(2, 1, 65, 1),
                                      padding=(32, 0), groups=2).numpy()
    for b in range(2):
        for h in range(2):
            mk = None if mask is None else mask[b]
            ref = _sdpa(x["q"][b, h], x["k"][b, h], x["v"][b, h], mk)
            np.testing.assert_allclose(out[b, h], ref + conv[b, h], rtol=1e-10, atol=1e-12)
            if mk is not None:
                assert np.all(st["probs"][b, h][:, mk == 0] == 0.0)
            np.testing.assert_allclose(st["probs"][b, h].sum(1), 1.0, atol=1e-12)


def test_exact_path_equals_nystrom_at_m_equals_n(oracle_mod):
    """m = n with a converged inverse reproduces path A (A A^+ A = A, walkthrough 2.1)."""
    r = _rng(22)
    n, d = 48, 16
    q, k, v = (r.standard_normal((1, 1, n, d)).astype(np.float32) for _ in range(3))
    a = oracle_mod.forward(q, k, v, None, None, exact=True)
    b = oracle_mod.forward(q, k, v, None, None, m=n, n_iter=30)
    assert np.linalg.norm(a - b) / np.linalg.norm(a) < 1e-9


def test_probs_are_kernel1_times_z(oracle_mod):
    """The returned weights (2.7) times kernel_3 V give the attention term (2.4), and at m = n
    with a converged inverse they are A A^+ = I for the nonsingular A of these inputs."""
    w = WORKLOADS["default_f32_masked"]
    x = make_inputs(w, seed=23, B=1, H=2, n=128)
    out, st = oracle_mod.forward(x["q"], x["k"], x["v"], x["mask"], None, m=16, stages=True, probs=True)
    for h in range(2):
        np.testing.assert_allclose(st["probs"][0, h] @ st["k3v"][0, h], out[0, h], rtol=1e-10, atol=1e-12)
    r = _rng(24)
    q, k, v = (r.standard_normal((1, 1, 32, 16)).astype(np.float32) for _ in range(3))
    _, st = oracle_mod.forward(q, k, v, None, None, m=32, n_iter=30, probs=True)
    np.testing.assert_allclose(st["probs"][0, 0], np.eye(32), atol=1e-9)

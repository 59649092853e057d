"""Python access to the fp64 CPU oracle (``nys_oracle.c``).

TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package. The product path
(the CUDA library and its binding) never does.

The oracle follows "Nystromformer source walkthrough" (blog.gitcode.com),
sections 2.2-2.6; see the C file for the step-by-step citations.

``build()`` compiles the C file with gcc into ``oracle/libnys_oracle.so``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nys_oracle.c")
LIB = os.path.join(HERE, "libnys_oracle.so")
TAPS = 65

_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        ip = ctypes.POINTER(ctypes.c_int)
        i = ctypes.c_int
        lib.nys_oracle_landmarks.argtypes = [fp, i, i, i, dp]
        lib.nys_oracle_softmax_rows.argtypes = [dp, i, i, u8p]
        lib.nys_oracle_iterative_inv.argtypes = [dp, i, i, dp]
        lib.nys_oracle_iterative_inv_opt.argtypes = [dp, i, i, i, dp]
        lib.nys_oracle_init_coeff.argtypes = [dp, i]
        lib.nys_oracle_init_coeff.restype = ctypes.c_double
        lib.nys_oracle_init_coeff_exact.argtypes = [dp, i]
        lib.nys_oracle_init_coeff_exact.restype = ctypes.c_double
        lib.nys_oracle_dwconv_add.argtypes = [fp, fp, i, i, dp]
        lib.nys_oracle_forward.argtypes = [fp, fp, fp, u8p, fp, i, i, i, i, i, i, i, i, ip, i, i,
                                           dp, dp, dp, dp, dp, dp, dp]
        lib.nys_oracle_forward.restype = ctypes.c_int
        lib.nys_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray], ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def max_threads() -> int:
    return int(_load().nys_oracle_max_threads())


def landmarks(x: np.ndarray, m: int) -> np.ndarray:
    """Segment means of d^-1/4 * x for one head; x is [n, d]."""
    x = _f32(x)
    n, d = x.shape
    out = np.empty((m, d), np.float64)
    _load().nys_oracle_landmarks(_ptr(x, ctypes.c_float), n, d, m, _ptr(out, ctypes.c_double))
    return out


def softmax_rows(s: np.ndarray, keep: Optional[np.ndarray] = None) -> np.ndarray:
    s = np.array(s, dtype=np.float64, order="C", copy=True)
    rows, cols = s.shape
    keep_arr = None if keep is None else np.ascontiguousarray(keep, dtype=np.uint8)
    _load().nys_oracle_softmax_rows(_ptr(s, ctypes.c_double), rows, cols,
                                    _ptr(keep_arr, ctypes.c_uint8))
    return s


def iterative_inv(a: np.ndarray, n_iter: int = 6, init_option: int = 0) -> np.ndarray:
    """Iterative inverse of walkthrough 2.5; init_option 0 = default Z_0 scalar,
    1 = the exact coefficient 1 / ||a||_1 (inv_coeff_init_option = True)."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    m = a.shape[0]
    z = np.empty((m, m), np.float64)
    _load().nys_oracle_iterative_inv_opt(_ptr(a, ctypes.c_double), m, n_iter, int(init_option),
                                         _ptr(z, ctypes.c_double))
    return z


def init_coeff(a: np.ndarray, init_option: int = 0) -> float:
    a = np.ascontiguousarray(a, dtype=np.float64)
    fn = _load().nys_oracle_init_coeff_exact if init_option else _load().nys_oracle_init_coeff
    return float(fn(_ptr(a, ctypes.c_double), a.shape[0]))


def dwconv(v: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The depthwise 65-tap sequence convolution of one head's V ([n, d])."""
    v = _f32(v)
    w = _f32(w)
    n, d = v.shape
    out = np.zeros((n, d), np.float64)
    _load().nys_oracle_dwconv_add(_ptr(v, ctypes.c_float), _ptr(w, ctypes.c_float), n, d,
                                  _ptr(out, ctypes.c_double))
    return out


def forward(q, k, v, mask=None, conv_w=None, m: int = 64, n_iter: int = 6,
            rows: Optional[Sequence[int]] = None, threads: int = 0, stages: bool = False,
            init_option: int = 0, exact: bool = False, probs: bool = False):
    """Oracle forward over [B, H, n, d] float32 inputs; returns float64 output.

    ``rows`` selects query rows (same for every head): output [B, H, len(rows), d].
    With ``stages=True`` also returns a dict of per-head Q_l, K_l, kernel_2, Z and
    kernel_3 V (Nystrom path only); with ``probs=True`` the dict also holds "probs",
    the attention weights of walkthrough 2.7 ([B, H, rows, m] = kernel_1 Z, or
    [B, H, rows, n] on the exact path). ``init_option`` selects the Z_0 scalar
    (0 default, 1 exact coefficient); ``exact=True`` takes path A (2.1).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, n, d = q.shape
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    nr = n if rows_arr is None else len(rows_arr)
    out = np.empty((B, H, nr, d), np.float64)
    st = None
    if stages or probs:
        st = {}
    if stages and not exact:
        st.update(ql=np.empty((B, H, m, d)), kl=np.empty((B, H, m, d)),
                  k2=np.empty((B, H, m, m)), z=np.empty((B, H, m, m)),
                  k3v=np.empty((B, H, m, d)))
    if probs:
        st["probs"] = np.empty((B, H, nr, n if exact else m))
    mask_arr = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    w_arr = None if conv_w is None else _f32(conv_w)
    dp = ctypes.c_double
    g = (lambda key: _ptr(st[key], dp) if st is not None and key in st else None)
    rc = _load().nys_oracle_forward(
        _ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float),
        _ptr(mask_arr, ctypes.c_uint8), _ptr(w_arr, ctypes.c_float), B, H, n, d, m, n_iter,
        int(init_option), 1 if exact else 0,
        _ptr(rows_arr, ctypes.c_int), nr, int(threads), _ptr(out, dp),
        g("ql"), g("kl"), g("k2"), g("z"), g("k3v"), g("probs"))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return (out, st) if (stages or probs) else out

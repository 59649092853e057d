"""Python binding of the B200 Nystromformer self-attention forward library.

Argument marshalling only: every step of the forward runs in the CUDA
library ``libnys_attn.so`` (see ``include/nys_attn.h`` for the C ABI). torch
is used for device memory and streams. There is no CPU fallback: importing
this package fails loudly when the library is missing and cannot be built.

    import nystr_self_attention_scale_b200 as nys
    out = nys.forward(q, k, v, mask=None, conv_w=None, m=64, n_iter=6)

q, k, v: CUDA tensors [B, H, n, d], float32 or bfloat16, contiguous.
mask: [B, n] uint8/bool CUDA tensor (1 = valid key) or None.
conv_w: [H, 65] float32 CUDA tensor (the depthwise conv weight) or None.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from . import build as _build

LIB_PATH = _build.LIB
CONV_TAPS = 65
DEFAULT_N_ITER = 6
DEFAULT_NUM_LANDMARKS = 64

F32, BF16 = 0, 1
INV_INIT_DEFAULT, INV_INIT_EXACT = 0, 1
_STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape or dtype", -3: "CUDA error",
           -4: "device workspace allocation failed", -5: "bounded device wait timed out",
           -6: "problem exceeds the library's fixed static scratch",
           -7: "a workspace guard zone was overwritten (guard mode)"}
OK, ERR_TIMEOUT, ERR_GUARD = 0, -5, -7


class NysError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, 'unknown status')} ({status})")


def _load() -> ctypes.CDLL:
    if os.environ.get("NYS_NO_BUILD") != "1":
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library missing: {LIB_PATH} (build with "
                          "python -m nystr_self_attention_scale_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    fwd = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.nys_attn_forward.argtypes = fwd + [vp]
    lib.nys_attn_forward_host.argtypes = fwd + [vp]
    lib.nys_attn_forward_debug.argtypes = fwd + [vp, vp, vp, vp, vp, vp]
    lib.nys_attn_forward_ex.argtypes = fwd[:-1] + [i, i, vp, vp, vp]
    for f in ("nys_attn_forward", "nys_attn_forward_host", "nys_attn_forward_debug",
              "nys_attn_forward_ex", "nys_attn_device_status", "nys_attn_version"):
        getattr(lib, f).restype = ctypes.c_int
    lib.nys_attn_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.nys_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.nys_attn_profile_enable.argtypes = [i]
    lib.nys_attn_profile_enable.restype = i
    lib.nys_attn_profile_read.argtypes = [i, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    lib.nys_attn_profile_mask.argtypes = [ctypes.c_uint]
    lib.nys_attn_profile_mask.restype = i
    lib.nys_attn_profile_read.restype = i
    lib.nys_attn_kernel_count.restype = i
    lib.nys_attn_kernel_name.argtypes = [i]
    lib.nys_attn_kernel_name.restype = ctypes.c_char_p
    lib.nys_attn_pinv_static.argtypes = [vp, vp, vp, i, i, i, i, vp]
    lib.nys_attn_pinv_static.restype = i
    lib.nys_attn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_int)]
    lib.nys_attn_selftest_wait_timeout.restype = i
    lib.nys_attn_set_workspace_guard.argtypes = [i]
    lib.nys_attn_set_workspace_guard.restype = i
    lib.nys_attn_selftest_guard.argtypes = [i, ctypes.POINTER(ctypes.c_int)]
    lib.nys_attn_selftest_guard.restype = i
    lib.nys_attn_selftest_exp2.argtypes = [ctypes.POINTER(ctypes.c_float)]
    lib.nys_attn_selftest_exp2.restype = i
    lib.nys_strerror.argtypes = [i]
    lib.nys_strerror.restype = ctypes.c_char_p
    return lib


lib = _load()


def strerror(status: int) -> str:
    return lib.nys_strerror(int(status)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise NysError(rc, what)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _shape(q, k, v):
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, H, n, d] shape")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k, v must share one dtype")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    return tuple(int(x) for x in q.shape)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _prep_device(q, k, v, mask, conv_w):
    import torch
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("forward() takes CUDA tensors; use forward_host() for host buffers")
    B, H, n, d = _shape(q, k, v)
    if mask is not None:
        if mask.shape != (B, n) or not mask.is_cuda:
            raise ValueError("mask must be a [B, n] CUDA tensor")
        mask = mask.to(torch.uint8).contiguous()
    if conv_w is not None:
        if tuple(conv_w.shape) not in ((H, CONV_TAPS), (H, 1, CONV_TAPS, 1)) or not conv_w.is_cuda:
            raise ValueError("conv_w must be a [H, 65] CUDA tensor")
        conv_w = conv_w.reshape(H, CONV_TAPS).to(torch.float32).contiguous()
    return (B, H, n, d), mask, conv_w


def forward(q, k, v, mask=None, conv_w=None, m: int = DEFAULT_NUM_LANDMARKS,
            n_iter: int = DEFAULT_N_ITER, out=None, stream=None):
    """Nystromformer attention forward on device tensors; returns out [B, H, n, d]."""
    import torch
    (B, H, n, d), mask, conv_w = _prep_device(q, k, v, mask, conv_w)
    if out is None:
        out = torch.empty_like(q)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.nys_attn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), _ptr(conv_w), B, H, n, d,
                                  int(m), int(n_iter), _dtype_code(q), _ptr(out), s.cuda_stream)
    _check(rc, "nys_attn_forward")
    return out


def takes_exact_path(num_landmarks: int, segment_means_seq_len: int) -> bool:
    """The layer's branch rule (walkthrough 2.1, 3.1): path A, exact attention, when the
    number of landmarks equals the segment-means sequence length."""
    return int(num_landmarks) == int(segment_means_seq_len)


def forward_ex(q, k, v, mask=None, conv_w=None, m: int = DEFAULT_NUM_LANDMARKS,
               n_iter: int = DEFAULT_N_ITER, inv_coeff_init_option: bool = False,
               exact: bool = False, output_attentions: bool = False, out=None, stream=None):
    """forward() with the layer's other options (nys_attn_forward_ex): the exact Z_0
    coefficient, the exact branch (path A), and the returned attention weights
    ([B, H, n, m], or [B, H, n, n] on the exact path, float32). Returns out, or
    (out, weights) when output_attentions is set."""
    import torch
    (B, H, n, d), mask, conv_w = _prep_device(q, k, v, mask, conv_w)
    if out is None:
        out = torch.empty_like(q)
    probs = None
    if output_attentions:
        probs = torch.empty(B, H, n, n if exact else int(m), device=q.device, dtype=torch.float32)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.nys_attn_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), _ptr(conv_w), B, H, n, d,
                                     int(m), int(n_iter), _dtype_code(q),
                                     INV_INIT_EXACT if inv_coeff_init_option else INV_INIT_DEFAULT,
                                     1 if exact else 0, _ptr(out), _ptr(probs), s.cuda_stream)
    _check(rc, "nys_attn_forward_ex")
    return (out, probs) if output_attentions else out


def forward_debug(q, k, v, mask=None, conv_w=None, m: int = DEFAULT_NUM_LANDMARKS,
                  n_iter: int = DEFAULT_N_ITER):
    """forward() plus the float32 stages: q_l, k_l, z, k3v, w (per head)."""
    import torch
    (B, H, n, d), mask, conv_w = _prep_device(q, k, v, mask, conv_w)
    out = torch.empty_like(q)
    f = dict(device=q.device, dtype=torch.float32)
    st = dict(q_l=torch.empty(B, H, m, d, **f), k_l=torch.empty(B, H, m, d, **f),
              z=torch.empty(B, H, m, m, **f), k3v=torch.empty(B, H, m, d, **f),
              w=torch.empty(B, H, m, d, **f))
    s = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.nys_attn_forward_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), _ptr(conv_w), B, H,
                                        n, d, int(m), int(n_iter), _dtype_code(q), _ptr(out),
                                        _ptr(st["q_l"]), _ptr(st["k_l"]), _ptr(st["z"]),
                                        _ptr(st["k3v"]), _ptr(st["w"]), s.cuda_stream)
    _check(rc, "nys_attn_forward_debug")
    return out, st


def forward_host(q, k, v, mask=None, conv_w=None, m: int = DEFAULT_NUM_LANDMARKS,
                 n_iter: int = DEFAULT_N_ITER, out=None, stream=None):
    """Same operation on host (CPU, ideally pinned) tensors; the library copies
    inputs in, runs, copies the result back and synchronises before returning."""
    import torch
    B, H, n, d = _shape(q, k, v)
    if q.is_cuda:
        raise ValueError("forward_host() takes host tensors")
    if mask is not None:
        mask = mask.to(torch.uint8).contiguous()
    if conv_w is not None:
        conv_w = conv_w.reshape(H, CONV_TAPS).to(torch.float32).contiguous()
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    s = stream if stream is not None else torch.cuda.current_stream()
    rc = lib.nys_attn_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), _ptr(conv_w), B, H, n, d,
                                   int(m), int(n_iter), _dtype_code(q), _ptr(out), s.cuda_stream)
    _check(rc, "nys_attn_forward_host")
    return out


def device_status() -> int:
    """Synchronise and return (and clear) the library's device status word."""
    return int(lib.nys_attn_device_status())


def selftest_exp2() -> float:
    """Maximum relative error of the library's FMA-pipe 2^x against CUDA's exp2f on [-125, 8]."""
    err = ctypes.c_float(0.0)
    _check(lib.nys_attn_selftest_exp2(ctypes.byref(err)), "nys_attn_selftest_exp2")
    return float(err.value)


def selftest_wait_timeout(limit_ns: int = 1_000_000) -> int:
    """Run the bounded-wait self-test (a wait nothing completes, limited to `limit_ns`);
    returns 0 when the wait ran out (the expected result) and 1 if it completed."""
    done = ctypes.c_int(-1)
    _check(lib.nys_attn_selftest_wait_timeout(int(limit_ns), ctypes.byref(done)),
           "nys_attn_selftest_wait_timeout")
    return int(done.value)


def set_workspace_guard(enable: bool) -> bool:
    """Turn the workspace guard mode on or off for later calls; returns the previous setting.

    While it is on, every workspace buffer lies between guard zones, the workspace starts as
    0xFF bytes (NaN), and a check after each call records ERR_GUARD in the device status word
    if a guard byte changed (read it with device_status())."""
    prev = int(lib.nys_attn_set_workspace_guard(1 if enable else 0))
    _check(min(prev, 0), "nys_attn_set_workspace_guard")
    return bool(prev)


def selftest_guard(corrupt: bool) -> int:
    """Run the guard check on a small buffer, with one guard byte changed from the host if
    `corrupt`; returns the status word it left (OK, or ERR_GUARD when corrupt)."""
    st = ctypes.c_int(1)
    _check(lib.nys_attn_selftest_guard(1 if corrupt else 0, ctypes.byref(st)), "nys_attn_selftest_guard")
    return int(st.value)


def workspace_bytes(B, H, n, d, m, dtype_code=BF16) -> int:
    return int(lib.nys_attn_workspace_bytes(B, H, n, d, m, dtype_code))


def version() -> int:
    return int(lib.nys_attn_version())


def profile_enable(on: bool = True) -> None:
    """Start (or stop) per-kernel CUDA-event timing; clears the counters."""
    lib.nys_attn_profile_enable(1 if on else 0)


def profile_mask(kernels=None) -> None:
    """Time only the named kernels (an iterable of names from profile_read()), or all of
    them when `kernels` is None."""
    if kernels is None:
        mask = 0xFFFFFFFF
    else:
        names = [lib.nys_attn_kernel_name(k).decode() for k in range(lib.nys_attn_kernel_count())]
        mask = 0
        for name in kernels:
            mask |= 1 << names.index(name)
    _check(lib.nys_attn_profile_mask(mask), "profile_mask")


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since profile_enable()."""
    out = {}
    for kid in range(lib.nys_attn_kernel_count()):
        n = ctypes.c_int(0)
        ms = ctypes.c_double(0.0)
        _check(lib.nys_attn_profile_read(kid, ctypes.byref(n), ctypes.byref(ms)), "profile_read")
        out[lib.nys_attn_kernel_name(kid).decode()] = (n.value, ms.value)
    return out


def _check_pinv_static_args(q_l, k_l, out):
    """Shape, dtype, device and layout checks of pinv_static() (no CUDA call): q_l and k_l
    float32 [B, H, m, d] on one device, out (if given) a contiguous float32 [B, H, m, m] on
    the same device. A wrong buffer here would make the kernel read or write out of bounds."""
    import torch
    if q_l.dim() != 4 or q_l.dtype != torch.float32:
        raise ValueError("q_l must be a float32 [B, H, m, d] tensor")
    if k_l.dtype != torch.float32 or tuple(k_l.shape) != tuple(q_l.shape):
        raise ValueError("k_l must be a float32 tensor of q_l's shape")
    if k_l.device != q_l.device:
        raise ValueError("k_l must be on q_l's device")
    if out is not None:
        B, H, m, _ = (int(t) for t in q_l.shape)
        if out.dtype != torch.float32 or tuple(out.shape) != (B, H, m, m):
            raise ValueError("out must be a float32 [B, H, m, m] tensor")
        if not out.is_contiguous():
            raise ValueError("out must be contiguous")
        if out.device != q_l.device:
            raise ValueError("out must be on q_l's device")


def pinv_static(q_l, k_l, n_iter: int = DEFAULT_N_ITER, out=None, stream=None):
    """kernel_2 + iterative inverse from float32 landmarks [B, H, m, d] -> Z [B, H, m, m],
    through the allocation-free entry point (scratch is a fixed array inside the library)."""
    import torch
    _check_pinv_static_args(q_l, k_l, out)
    if not q_l.is_cuda:
        raise ValueError("q_l, k_l must be CUDA tensors")
    B, H, m, d = (int(t) for t in q_l.shape)
    q_l, k_l = q_l.contiguous(), k_l.contiguous()
    if out is None:
        out = torch.empty(B, H, m, m, device=q_l.device, dtype=torch.float32)
    s = stream if stream is not None else torch.cuda.current_stream(q_l.device)
    with torch.cuda.device(q_l.device):
        rc = lib.nys_attn_pinv_static(_ptr(q_l), _ptr(k_l), _ptr(out), B * H, m, d, int(n_iter),
                                      s.cuda_stream)
    _check(rc, "nys_attn_pinv_static")
    return out

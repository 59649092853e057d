"""Host-side checks of the C ABI library (no GPU needed).

The shared library must build for sm_100a, load, export every function that
include/nys_attn.h declares, and reject bad arguments before touching the
device. No compute call is made here.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def _declared():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for mt in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(nys_\w+)\s*\(", text, re.M):
            names.add(mt.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    import nystr_self_attention_scale_b200 as nys
    return nys.lib


def test_header_declares_the_entry_points():
    names = _declared()
    for required in ("nys_attn_forward", "nys_attn_forward_host", "nys_attn_forward_debug",
                     "nys_strerror", "nys_attn_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    import nystr_self_attention_scale_b200 as nys
    out = subprocess.run(["nm", "-D", "--defined-only", nys.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        getattr(lib, n)


def test_library_is_sm100a():
    import nystr_self_attention_scale_b200 as nys
    log = open(os.path.join(os.path.dirname(nys.LIB_PATH), "build.log")).read()
    assert "arch=compute_100a,code=sm_100a" in log


def test_strerror_texts(lib):
    import nystr_self_attention_scale_b200 as nys
    assert nys.strerror(0) == "ok"
    assert "invalid" in nys.strerror(-1)
    assert "unsupported" in nys.strerror(-2)
    assert nys.strerror(12345) == "unknown status"


def _call(lib, B=1, H=1, n=512, d=64, m=64, n_iter=6, dtype=0, null=False):
    p = None if null else ctypes.c_void_p(16)  # never dereferenced: checks fail first
    return lib.nys_attn_forward(p, p, p, None, None, B, H, n, d, m, n_iter, dtype, p, None)


@pytest.mark.parametrize("kw,code", [
    (dict(null=True), -1),
    (dict(B=0), -1), (dict(H=-1), -1), (dict(n=0), -1), (dict(d=0), -1), (dict(m=0), -1),
    (dict(n=500, m=64), -1),          # n % m != 0
    (dict(n=64, m=128), -1),          # m > n
    (dict(n_iter=-1), -1),
    (dict(d=48), -2), (dict(d=128), -2),
    (dict(m=512, n=1024), -2),
    (dict(dtype=7), -2),
    (dict(dtype=1, m=32), -2),        # bf16 tensor path: m in {64, 128, 256}
    (dict(dtype=1, n=192, m=64), -2), # bf16 tensor path: n % 128 == 0
])
def test_rejects_before_launch(lib, kw, code):
    assert _call(lib, **kw) == code


def test_host_entry_validates_too(lib):
    p = ctypes.c_void_p(16)
    assert lib.nys_attn_forward_host(p, p, p, None, None, 1, 1, 100, 64, 64, 6, 0, p, None) == -1


def test_workspace_bytes(lib):
    import nystr_self_attention_scale_b200 as nys
    assert nys.workspace_bytes(1, 1, 100, 64, 64) == 0
    small = nys.workspace_bytes(1, 1, 512, 64, 64, 0)
    big = nys.workspace_bytes(4, 8, 16384, 64, 256)
    assert 0 < small < big


def test_defaults_match_the_pages():
    """Defaults printed by the pages (see tests/golden/config_defaults.txt)."""
    import nystr_self_attention_scale_b200 as nys
    rows = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "config_defaults.txt")):
        line = line.split("#", 1)[0].strip()
        if line:
            key, val = line.split("=", 1)
            rows[key.strip()] = val.strip()
    assert int(rows["num_landmarks"]) == nys.DEFAULT_NUM_LANDMARKS
    assert int(rows["conv_kernel_size"]) == nys.CONV_TAPS
    assert int(rows["iterative_inv_n_iter"]) == nys.DEFAULT_N_ITER
    hdr = open(os.path.join(ROOT, "include", "nys_attn.h")).read()
    assert f"#define NYS_CONV_TAPS {rows['conv_kernel_size']}" in hdr
    assert f"#define NYS_DEFAULT_N_ITER {rows['iterative_inv_n_iter']}" in hdr


def test_host_plan_covers_every_slice_once(lib):
    """The host entry's chunk plan: at most 8 chunks, each contiguous in a [B, H, n, d]
    tensor (whole batch elements, or a head range of one), covering every slice once."""
    import ctypes
    lib.nys_attn_host_plan.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    lib.nys_attn_host_plan.restype = ctypes.c_int
    buf = (ctypes.c_int * 32)()
    for B in range(1, 40):
        for H in range(1, 20):
            n = lib.nys_attn_host_plan(B, H, buf, 8)
            assert 1 <= n <= 8, (B, H, n)
            seen = []
            for c in range(n):
                b0, nb, h0, nh = buf[4 * c:4 * c + 4]
                assert nb >= 1 and nh >= 1 and (nb == 1 or (h0 == 0 and nh == H)), (B, H, c)
                seen += [(b, h) for b in range(b0, b0 + nb) for h in range(h0, h0 + nh)]
            assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)], (B, H)
    assert lib.nys_attn_host_plan(0, 1, buf, 8) == -1
    assert lib.nys_attn_host_plan(1, 1, buf, 7) == -1
    assert lib.nys_attn_host_plan(1, 1, None, 8) == -1


def test_pinv_static_binding_rejects_bad_buffers():
    """pinv_static() checks its buffers before calling the library: a k_l of another dtype,
    shape or device, or an `out` of the wrong shape, dtype, layout or device, would make the
    kernel read or write out of bounds (checked here on CPU tensors: no CUDA call is made)."""
    import torch
    import nystr_self_attention_scale_b200 as nys
    check = nys._check_pinv_static_args
    q = torch.zeros(2, 3, 64, 32)
    check(q, q.clone(), None)
    check(q, q.clone(), torch.zeros(2, 3, 64, 64))
    bad = [
        (q.double(), q, None),                              # q_l not float32
        (q[0], q[0], None),                                 # not 4-D
        (q, q.to(torch.bfloat16), None),                    # k_l dtype
        (q, torch.zeros(2, 3, 64, 64), None),               # k_l shape
        (q, q, torch.zeros(2, 3, 64, 32)),                  # out shape
        (q, q, torch.zeros(2, 3, 64, 64, dtype=torch.float64)),   # out dtype
        (q, q, torch.zeros(2, 3, 64, 128)[..., ::2]),       # out strided
        (q, q, torch.zeros(2, 3, 64, 64, device="meta")),   # out on another device
        (q, q.to("meta"), None),                            # k_l on another device
    ]
    for args in bad:
        with pytest.raises(ValueError):
            check(*args)


@pytest.mark.parametrize("kw,code", [
    (dict(inv_init=2), -1),                      # neither Z_0 option
    (dict(inv_init=-1), -1),
    (dict(exact=1, null=True), -1),
    (dict(exact=1, d=48), -2),
    (dict(exact=1, dtype=1, n=192), -2),         # bf16 exact branch: n % 128 == 0
    (dict(exact=1, B=0), -1),
    (dict(n=500, m=64), -1),                     # Nystrom path checks as nys_attn_forward
])
def test_forward_ex_rejects_before_launch(lib, kw, code):
    p = None if kw.pop("null", False) else ctypes.c_void_p(16)
    a = dict(B=1, H=1, n=512, d=64, m=64, n_iter=6, dtype=0, inv_init=0, exact=0)
    a.update(kw)
    assert lib.nys_attn_forward_ex(p, p, p, None, None, a["B"], a["H"], a["n"], a["d"], a["m"],
                                   a["n_iter"], a["dtype"], a["inv_init"], a["exact"], p, None,
                                   None) == code

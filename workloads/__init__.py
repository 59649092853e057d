"""Seeded synthetic inputs for the Nystromformer attention forward.

This module is shared by the CPU oracle's tests, the GPU parity tests, the
smoke check and the benchmark. It draws random numbers and lays them out;
it holds none of the attention arithmetic.

Recipe (every workload): numpy ``default_rng(seed)``; draw order Q, K, V,
conv weights, then per-sequence valid lengths; values are drawn in float32
and, for bf16 workloads, rounded to bf16 with round-to-nearest-even. The
returned float32 arrays hold exactly the values the device sees, so both
sides start from identical bits.

Shapes follow the head split of the Nystromformer self-attention
("Nystromformer source walkthrough", section 2.2): ``[B, H, n, d]``
row-major. The key mask is ``[B, n]`` uint8, 1 = valid key, 0 = padded
(the model API's attention-mask convention, HF docs, NystromformerModel
forward, ``attention_mask``). Conv weights are ``[H, 65]`` float32, the
depthwise Conv2d weight ``[H, 1, 65, 1]`` flattened (walkthrough section 2.6).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

CONV_TAPS = 65


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16"
    B: int
    H: int
    n: int
    d: int
    m: int
    n_iter: int = 6
    conv: bool = True
    lengths: Optional[tuple] = None   # (lo, hi) inclusive valid-length range, or None = no mask
    zero_pad: bool = False            # zero Q/K/V rows at padded positions
    dist: str = "iid"                 # "iid" N(0,1) or "correlated"

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.n

    def describe(self) -> str:
        parts = [f"{self.dtype} B={self.B} H={self.H} n={self.n} d={self.d} m={self.m}",
                 f"n_iter={self.n_iter}", "conv65" if self.conv else "noconv"]
        if self.lengths:
            parts.append(f"valid_len~U[{self.lengths[0]},{self.lengths[1]}]")
        if self.dist != "iid":
            parts.append(self.dist)
        return " ".join(parts)


def _c5(n: int, conv: bool) -> Workload:
    return Workload(f"sweep_n{n}_{'conv' if conv else 'noconv'}", "bf16", 8, 8, n, 64, 64,
                    conv=conv)


# The five workload families: the default-config shapes in fp32, the long
# sequence classification shape, the n=16384 correlated-token shape, the
# n sweep, and the degenerate n = m case.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "f32", 1, 1, 512, 64, 64),
    "default_f32_masked": Workload("default_f32_masked", "f32", 8, 12, 512, 64, 64,
                                   lengths=(256, 512), zero_pad=True),
    "longcls_bf16_masked": Workload("longcls_bf16_masked", "bf16", 32, 2, 4096, 32, 128,
                                    lengths=(1024, 4096), zero_pad=True),
    "n16384_bf16_corr": Workload("n16384_bf16_corr", "bf16", 4, 8, 16384, 64, 256,
                                 dist="correlated"),
    # the headline shape at B*H = 128: more CTA pairs of the m = 256 inverse than one wave
    "n16384_bf16_corr_bh128": Workload("n16384_bf16_corr_bh128", "bf16", 16, 8, 16384, 64, 256,
                                       dist="correlated"),
    "degenerate_f32_it24": Workload("degenerate_f32_it24", "f32", 1, 1, 256, 64, 256,
                                    n_iter=24, conv=False),
    "degenerate_f32_it6": Workload("degenerate_f32_it6", "f32", 1, 1, 256, 64, 256,
                                   n_iter=6, conv=False),
}
for _n in (1024, 4096, 16384, 65536):
    for _conv in (True, False):
        _w = _c5(_n, _conv)
        WORKLOADS[_w.name] = _w

HEADLINE = "n16384_bf16_corr"


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    if dist == "iid":
        return rng.standard_normal(shape, dtype=np.float32)
    if dist == "correlated":
        # 0.5 * N(0,1) per element plus one N(0,1) value per token shared by all d lanes
        z = rng.standard_normal(shape, dtype=np.float32)
        s = rng.standard_normal(shape[:-1] + (1,), dtype=np.float32)
        return (np.float32(0.5) * z + s).astype(np.float32)
    raise ValueError(dist)


def make_inputs(w: Workload, seed: int = 0, B: Optional[int] = None, H: Optional[int] = None,
                n: Optional[int] = None) -> dict:
    """Draw the inputs of workload ``w`` (optionally with B/H/n overridden).

    Returns a dict with float32 arrays ``q, k, v`` ([B,H,n,d], values exactly
    representable in ``w.dtype``), ``bits`` (uint16 views for bf16, else None),
    ``conv_w`` ([H,65] float32 or None), ``mask`` ([B,n] uint8 or None) and
    ``lengths`` ([B] int64 or None).
    """
    B = B or w.B
    H = H or w.H
    n = n or w.n
    rng = np.random.default_rng(seed)
    shape = (B, H, n, w.d)
    q = _draw(rng, shape, w.dist)
    k = _draw(rng, shape, w.dist)
    v = _draw(rng, shape, w.dist)
    conv_w = None
    if w.conv:
        conv_w = (rng.standard_normal((H, CONV_TAPS), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    mask = None
    lengths = None
    if w.lengths is not None:
        lo, hi = w.lengths
        lengths = rng.integers(lo, hi + 1, size=B).astype(np.int64)
        pos = np.arange(n)[None, :]
        mask = (pos < lengths[:, None]).astype(np.uint8)
        if w.zero_pad:
            keep = mask[:, None, :, None].astype(np.float32)
            q *= keep
            k *= keep
            v *= keep
    bits = None
    if w.dtype == "bf16":
        bits = {}
        for name, arr in (("q", q), ("k", k), ("v", v)):
            b = f32_to_bf16_bits(arr)
            bits[name] = b
        q, k, v = (bf16_bits_to_f32(bits["q"]).reshape(shape),
                   bf16_bits_to_f32(bits["k"]).reshape(shape),
                   bf16_bits_to_f32(bits["v"]).reshape(shape))
    return dict(q=q, k=k, v=v, bits=bits, conv_w=conv_w, mask=mask, lengths=lengths,
                B=B, H=H, n=n, d=w.d, m=w.m, n_iter=w.n_iter, dtype=w.dtype)

"""Seeded synthetic inputs shaped like video-DiT self-attention activations.

This module is shared by the CUDA path's tests/bench and by the oracle's tests.
It holds no routing, masking or attention arithmetic: only the random draws,
the positional "feature" signal mixed into Q/K and the fp32 -> bf16 encoding
of the drawn values.  The long-horizon workload's fixed window-plus-anchor
mask is not drawn here: tests take it from the oracle (oracle/masks.py) and
the benchmark from the library's own device producer.

Layout of every Q/K/V tensor: [B, N, H, d] in C order, N = T*Hs*Ws tokens in
raster order (frame t, then row y, then column x), i.e. the layout a video DiT
hands to its attention layer.

Workloads (sizes follow the pages' Wan2.1 / Wan2.2 setups: FVAttn review,
section 5 "experimental setup" -- 720p, 21 latent frames x 3600 tokens; the
long-horizon fixed mask follows the LVSA wiki page, "TL;DR" and "Key points"):

  1 tiny        B1 H2  d64  T4 x16x16  =   1024 tokens, block 64,  fp32
  2 480p        B1 H12 d128 T21x30x52  =  32760 tokens, block 128, bf16
  3 720p        B1 H40 d128 T21x45x80  =  75600 tokens, block 128, bf16 (p 0.8/0.9/0.95)
  4 skewed      config-3 shapes, 36 concentrated heads + 4 near-dense heads
  5 long        B1 H12 d128 T126x30x52 = 196560 tokens, block 128, bf16, fixed mask

Generator recipe (numpy PCG64, seed = 1000*config + sub):
  draw c_h [H] ~ U[0,2], then s_h [H] (log-uniform [1/4, 4]), then z_q, z_k, z_v
  ~ N(0,1) fp32 [B,N,H,d] in that order;
  Q = s_h * (z_q + c_h * f(t,y,x)), K = z_k + c_h * f(t,y,x), V = z_v,
  rounded once to bf16 (round to nearest even).  Tiny keeps fp32, uses no
  feature term and fixed scales s = (0.5, 3.0).  Config 4 fixes s_h = 4 on heads
  0..35 and 1/4 on heads 36..39.  Config 5 uses plain N(0,1) draws.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload", "CONFIGS", "workload", "make_inputs", "features",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "seed_for",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    B: int
    H: int
    d: int
    T: int
    Hs: int
    Ws: int
    block: int
    dtype: str              # "f32" or "bf16": the dtype routing reads
    ps: tuple               # Top-p values exercised (empty: fixed mask, no routing)
    k_floor: int

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def nb(self) -> int:
        return -(-self.N // self.block)

    @property
    def rows(self) -> int:
        return self.B * self.H * self.nb


CONFIGS = {
    1: Workload(1, "tiny_1024", 1, 2, 64, 4, 16, 16, 64, "f32", (0.9,), 2),
    2: Workload(2, "wan21_480p_32760", 1, 12, 128, 21, 30, 52, 128, "bf16", (0.9,), 4),
    3: Workload(3, "wan22_720p_75600", 1, 40, 128, 21, 45, 80, 128, "bf16", (0.8, 0.9, 0.95), 4),
    4: Workload(4, "skewed_720p_75600", 1, 40, 128, 21, 45, 80, 128, "bf16", (0.95,), 8),
    5: Workload(5, "long_fixed_196560", 1, 12, 128, 126, 30, 52, 128, "bf16", (), 0),
}


def workload(cid: int, **override) -> Workload:
    """Return config `cid`, optionally with fields replaced (for small variants)."""
    w = CONFIGS[cid]
    return dataclasses.replace(w, **override) if override else w


def f32_to_bf16_bits_reference(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns the uint16 bit patterns.

    The definition written out on the bit patterns (add 0x7FFF plus the lowest
    kept bit, drop the low 16 bits).  Inputs here are finite, so no NaN
    handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """As f32_to_bf16_bits_reference (same bits, checked by the tests), through
    torch's multi-threaded CPU conversion, which rounds the same way."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def features(T: int, Hs: int, Ws: int, d: int) -> np.ndarray:
    """Sinusoidal (t, y, x) features, fp32 [T*Hs*Ws, d], raster token order.

    The d/2 sin/cos pairs are split into a t group (the remainder) and equal
    y and x groups (d/2 // 3 pairs each): for d=128 that is 22/21/21 pairs,
    i.e. 44/42/42 dims.  Within a group of P pairs over coordinate u, pair m
    is (sin(u*w_m), cos(u*w_m)) with w_m = 10000**(-m/P).
    """
    pairs = d // 2
    py = px = pairs // 3
    pt = pairs - py - px
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hs), np.arange(Ws), indexing="ij")
    out = np.empty((T * Hs * Ws, d), dtype=np.float64)
    col = 0
    for u, P in ((t.ravel(), pt), (y.ravel(), py), (x.ravel(), px)):
        w = 10000.0 ** (-np.arange(P) / P)
        ang = u[:, None].astype(np.float64) * w[None, :]
        out[:, col:col + 2 * P:2] = np.sin(ang)
        out[:, col + 1:col + 2 * P:2] = np.cos(ang)
        col += 2 * P
    return out.astype(np.float32)


def _head_params(w: Workload, rng: np.random.Generator):
    c = rng.uniform(0.0, 2.0, size=w.H)
    s = np.exp(rng.uniform(math.log(0.25), math.log(4.0), size=w.H))
    if w.cid == 1:
        c = np.zeros(w.H)
        s = np.array([0.5, 3.0][: w.H] + [1.0] * max(0, w.H - 2))
    elif w.cid == 4:
        s = np.where(np.arange(w.H) < w.H - 4, 4.0, 0.25)
    elif w.cid == 5:
        c = np.zeros(w.H)
        s = np.ones(w.H)
    return c.astype(np.float32), s.astype(np.float32)


def make_inputs(w: Workload | int, sub: int = 0, seed: int | None = None) -> dict:
    """Draw Q, K, V for workload `w`.

    Returns {"q","k","v": arrays [B,N,H,d]} -- fp32 for the tiny workload,
    uint16 bf16 bit patterns otherwise -- plus the per-head "c" and "s" and the
    seed used.  Deterministic in (config, sub, seed).
    """
    if isinstance(w, int):
        w = CONFIGS[w]
    seed = 1000 * w.cid + sub if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    c, s = _head_params(w, rng)
    shape = (w.B, w.N, w.H, w.d)
    use_feat = bool(np.any(c != 0))
    f = features(w.T, w.Hs, w.Ws, w.d)[None, :, None, :] if use_feat else None
    out = {"c": c, "s": s, "seed": seed}
    for name in ("q", "k", "v"):
        z = rng.standard_normal(size=shape, dtype=np.float32)
        if name != "v" and use_feat:
            z += c[None, None, :, None] * f
        if name == "q":
            z *= s[None, None, :, None]
        out[name] = z if w.dtype == "f32" else f32_to_bf16_bits(z)
        del z
    return out


def seed_for(cid: int, p_index: int = 0) -> int:
    """Seed of config `cid` at its `p_index`-th Top-p value: 1000*cid + 1 + p_index
    (config 3: 3001/3002/3003 for p = 0.8/0.9/0.95)."""
    return 1000 * cid + 1 + p_index

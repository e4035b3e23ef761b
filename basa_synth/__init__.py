"""Seeded synthetic inputs for shifted-window attention workloads.

This module only draws random numbers and rounds them to the storage dtype. It
holds none of the attention arithmetic, so both the CPU oracle side (tests,
``bench.py``'s CPU baseline) and the CUDA side (parity tests, bench) can take
their inputs from it without sharing any of the method's computation.

Tensors use the token layout ``[B, T, Hg, Wg, H, d]`` (batch, time, grid rows,
grid columns, heads, head dim), row-major.  A 2D image grid has ``T == 1``.

Recipe (per workload):
  * ``numpy.random.Generator(PCG64(seed))`` standard normal draws in float64,
    cast to float32, then rounded to the storage dtype (bfloat16 with
    round-to-nearest-even, done by ``torch.Tensor.to``).  The rounded tensor is
    the one both sides see.
  * seeds: ``seed = 1000 * workload + 10 * block + {q: 0, k: 1, v: 2, head scale: 3}``.
  * optional per-head query scale: one factor ``u_h ~ U(0.5, 2)`` per head
    multiplies every query vector of that head.
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_qkv", "make_text_qkv", "to_storage", "seed_for",
           "workload_inputs", "text_inputs"]


@dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic shifted-window attention workload."""

    name: str
    B: int
    T: int
    Hg: int
    Wg: int
    H: int
    d: int
    dtype: str                      # "f32", "bf16" or "e4m3" (bf16 output)
    window: Tuple[int, int, int]    # (wt, wh, ww)
    shifts: Tuple[Tuple[int, int, int], ...]  # one (st, sh, sw) per DiT block
    pool: Tuple[int, int, int] = (0, 0, 0)     # (pt, ph, pw); zeros = no global memory
    head_scale: Optional[Tuple[float, float]] = None  # U(lo, hi) per-head |q| factor
    text: int = 0                   # text tokens of a joint text + image block (0 = none)

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def m(self) -> int:
        return self.window[0] * self.window[1] * self.window[2]

    @property
    def P(self) -> int:
        if self.pool == (0, 0, 0):
            return 0
        pt, ph, pw = self.pool
        return (self.T // pt) * (self.Hg // ph) * (self.Wg // pw)

    def shape(self):
        return (self.B, self.T, self.Hg, self.Wg, self.H, self.d)

    def describe(self) -> dict:
        out = asdict(self)
        out["N"] = self.N
        out["m"] = self.m
        out["P"] = self.P
        return out


# The five workloads: a small fp32 correctness grid, two FLUX-like image grids,
# a Wan-like video grid and a 4-block shift schedule with pooled global memory.
WORKLOADS = {
    "grid16_f32": Workload("grid16_f32", 1, 1, 16, 16, 2, 64, "f32",
                           (1, 8, 8), ((0, 4, 4),)),
    "flux1024": Workload("flux1024", 1, 1, 64, 64, 24, 128, "bf16",
                         (1, 16, 16), ((0, 0, 0), (0, 8, 8))),
    "flux2048": Workload("flux2048", 1, 1, 128, 128, 24, 128, "bf16",
                         (1, 16, 16), ((0, 8, 8),), head_scale=(0.5, 2.0)),
    "wan_video": Workload("wan_video", 1, 21, 45, 80, 40, 128, "bf16",
                          (7, 9, 16), ((3, 4, 8),)),
    "flux2048_gm4": Workload("flux2048_gm4", 2, 1, 128, 128, 24, 128, "bf16",
                             (1, 16, 16),
                             ((0, 0, 0), (0, 8, 0), (0, 0, 8), (0, 8, 8)),
                             pool=(1, 4, 4)),
    # a FLUX-like joint (double-stream) block: 1024^2 image tokens plus 512 text
    # tokens (the T5 prompt length FLUX uses); q, k, v ~ N(0, 1) for both streams
    "flux1024_text512": Workload("flux1024_text512", 1, 1, 64, 64, 24, 128, "bf16",
                                 (1, 16, 16), ((0, 8, 8),), text=512),
    # the flux2048 block with q, k, v stored as fp8 e4m3 (the same draws rounded
    # to e4m3 instead of bf16; descale factors 1)
    "flux2048_e4m3": Workload("flux2048_e4m3", 1, 1, 128, 128, 24, 128, "e4m3",
                              (1, 16, 16), ((0, 8, 8),), head_scale=(0.5, 2.0)),
}

WORKLOAD_INDEX = {"grid16_f32": 0, "flux1024": 1, "flux2048": 2, "wan_video": 3,
                  "flux2048_gm4": 4, "flux1024_text512": 5, "flux2048_e4m3": 2}


def seed_for(workload_index: int, block: int, which: str) -> int:
    off = {"q": 0, "k": 1, "v": 2, "head_scale": 3}[which]
    return 1000 * workload_index + 10 * block + off


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round a float array to the storage dtype (RNE for bf16 and e4m3) as a CPU tensor."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "e4m3":  # OCP fp8 e4m3 (torch.float8_e4m3fn); |x| here stays far below 448
        return t.to(torch.float8_e4m3fn)
    if dtype == "f32":
        return t
    raise ValueError(f"unknown dtype {dtype!r}")


def make_qkv(shape: Sequence[int], dtype: str, seed_q: int, seed_k: int, seed_v: int,
             head_scale: Optional[Tuple[float, float]] = None, seed_hs: int = 0,
             q_mult: float = 1.0):
    """Return CPU tensors (q, k, v) of ``shape`` in the storage dtype.

    ``q_mult`` multiplies q before rounding (used for large-logit stability cases).
    """
    def draw(seed):
        g = np.random.Generator(np.random.PCG64(seed))
        return g.standard_normal(size=tuple(shape), dtype=np.float64)

    q = draw(seed_q) * q_mult
    if head_scale is not None:
        g = np.random.Generator(np.random.PCG64(seed_hs))
        u = g.uniform(head_scale[0], head_scale[1], size=(shape[4],))
        q = q * u.reshape((1, 1, 1, 1, -1, 1))
    k = draw(seed_k)
    v = draw(seed_v)
    return to_storage(q, dtype), to_storage(k, dtype), to_storage(v, dtype)


def workload_inputs(w: Workload, block: int = 0, q_mult: float = 1.0):
    """Seeded (q, k, v) CPU tensors for block ``block`` of workload ``w``."""
    i = WORKLOAD_INDEX.get(w.name, 9)
    return make_qkv(w.shape(), w.dtype, seed_for(i, block, "q"), seed_for(i, block, "k"),
                    seed_for(i, block, "v"), head_scale=w.head_scale,
                    seed_hs=seed_for(i, block, "head_scale"), q_mult=q_mult)


def make_text_qkv(B: int, L: int, H: int, d: int, dtype: str, seed_q: int, seed_k: int,
                  seed_v: int):
    """Return CPU text-token tensors (qt, kt, vt) of shape [B, L, H, d]."""
    def draw(seed):
        g = np.random.Generator(np.random.PCG64(seed))
        return g.standard_normal(size=(B, L, H, d), dtype=np.float64)

    return to_storage(draw(seed_q), dtype), to_storage(draw(seed_k), dtype), \
        to_storage(draw(seed_v), dtype)


def text_inputs(w: Workload, block: int = 0):
    """Seeded text tokens (qt, kt, vt) of a joint workload; seeds offset by 5."""
    i = WORKLOAD_INDEX.get(w.name, 9)
    return make_text_qkv(w.B, w.text, w.H, w.d, w.dtype, seed_for(i, block, "q") + 5,
                         seed_for(i, block, "k") + 5, seed_for(i, block, "v") + 5)

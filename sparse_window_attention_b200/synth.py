"""Seeded synthetic inputs for the BASA forward path.

This module only draws random numbers and builds random fields. It holds none of
the operator's arithmetic (no windows, no pooling, no routing, no softmax), so the
CUDA path and the CPU oracle can both be fed from it without sharing method code.

Every tensor is drawn in float32 from ``numpy.random.Generator(PCG64(seed + off))``
with a fixed offset per tensor (``SEED_OFFSETS``) and a fixed draw order, then
rounded to bfloat16 (round-to-nearest-even, done by ``torch.Tensor.to``) or kept
in float32. The same bytes go to the GPU and, widened to float64, to the oracle.

Field recipes (they stand in for DiT activations; the pages measure on FLUX.1-dev
and Wan2.1 activations of COCO2014 / VBench prompts, which are not available):

* ``iid``: X ~ N(0, 1).
* ``sinusoid``: X = 0.5 N(0,1) + sin(2 pi (a y / H + b x / W) + phi), with integer
  a, b ~ U{-3..3} and phi ~ U[0, 2 pi) drawn per (head, channel). The field is
  periodic across the grid edges.
* ``block_mean``: X = 0.5 N(0,1) + mu[h, block(t, y, x)], mu ~ N(0,1)^d drawn per
  (head, block), where block() is the raster index of the cell that holds the
  token on a lattice of cells of a given size whose origin is offset by a given
  amount (cells wrap around the grid edges).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

SEED_OFFSETS = {"q": 0, "k": 1, "v": 2, "k_text": 3, "v_text": 4, "mu_q": 5, "mu_k": 6}


def rng_for(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed + SEED_OFFSETS[name]))


def iid_normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def sinusoid_field(rng: np.random.Generator, heads: int, T: int, H: int, W: int, d: int) -> np.ndarray:
    """[heads, T*H*W, d] float32 smooth field, periodic over (H, W); constant over T."""
    a = rng.integers(-3, 4, size=(heads, d)).astype(np.float32)
    b = rng.integers(-3, 4, size=(heads, d)).astype(np.float32)
    phi = rng.uniform(0.0, 2.0 * np.pi, size=(heads, d)).astype(np.float32)
    y = (np.arange(H, dtype=np.float32) / np.float32(H))[:, None]
    x = (np.arange(W, dtype=np.float32) / np.float32(W))[None, :]
    out = np.empty((heads, T, H, W, d), dtype=np.float32)
    two_pi = np.float32(2.0 * np.pi)
    for h in range(heads):
        arg = two_pi * (y[:, :, None] * a[h][None, None, :] + x[:, :, None] * b[h][None, None, :]) + phi[h]
        out[h] = np.sin(arg)[None]
    return out.reshape(heads, T * H * W, d)


def block_labels(T: int, H: int, W: int, cell, offset) -> np.ndarray:
    """Raster label of the lattice cell holding each token (cells wrap at the edges)."""
    ct, cy, cx = cell
    ot, oy, ox = offset
    nt, ny, nx = T // ct, H // cy, W // cx
    t = ((np.arange(T) - ot) % T) // ct
    y = ((np.arange(H) - oy) % H) // cy
    x = ((np.arange(W) - ox) % W) // cx
    lab = (t[:, None, None] * ny + y[None, :, None]) * nx + x[None, None, :]
    return lab.reshape(-1), nt * ny * nx


def block_mean_field(rng: np.random.Generator, heads: int, T: int, H: int, W: int, d: int, cell, offset) -> np.ndarray:
    lab, ncell = block_labels(T, H, W, cell, offset)
    mu = rng.standard_normal(size=(heads, ncell, d), dtype=np.float32)
    return mu[:, lab, :]


@dataclass
class Workload:
    """Shape of one BASA layer call (one layer at one shift)."""

    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    heads: int
    d: int
    grid: tuple  # (T, H, W)
    window: tuple  # (wt, wh, ww)
    shift: tuple  # (st, sy, sx)
    pool: tuple  # (pt, ph, pw) or (0, 0, 0)
    n_text: int
    routed_k: int
    field: str  # "iid", "sinusoid" or "block_mean"
    route_radius: int = 0  # routing candidates: 0 = all other windows, r = window-grid radius r

    @property
    def N(self) -> int:
        T, H, W = self.grid
        return T * H * W

    def with_shift(self, shift) -> "Workload":
        return Workload(**{**self.__dict__, "shift": tuple(shift)})


# Workload shapes (B=1). Shift cycles are listed in SHIFT_CYCLES.
WORKLOADS = {
    "tiny": Workload("tiny", "f32", 1, 2, 64, (1, 32, 32), (1, 8, 8), (0, 4, 4), (1, 4, 4), 0, 0, "iid"),
    "flux1k": Workload("flux1k", "bf16", 1, 24, 128, (1, 64, 64), (1, 16, 16), (0, 0, 0), (1, 8, 8), 512, 0, "sinusoid"),
    "flux2k": Workload("flux2k", "bf16", 1, 24, 128, (1, 128, 128), (1, 32, 32), (0, 0, 0), (1, 8, 8), 512, 0, "sinusoid"),
    "flux4k": Workload("flux4k", "bf16", 1, 24, 128, (1, 256, 256), (1, 32, 32), (0, 16, 16), (1, 16, 16), 512, 0, "sinusoid"),
    "wan": Workload("wan", "bf16", 1, 12, 128, (21, 30, 52), (3, 6, 13), (0, 3, 6), (3, 6, 13), 0, 4, "block_mean"),
    # The pages' own video configuration at the Wan2.1-1.3B latent grid of 1664x960, 81
    # frames: windows keep the full temporal extent, pooling is spatial only, and one
    # routed window is chosen among the radius-one neighbours (BASA §3.2, §3.3, §A.2 and
    # Table 3, row w=(15,26), p=(4,4)).
    "wan_video": Workload("wan_video", "bf16", 1, 12, 128, (21, 60, 104), (21, 15, 26), (0, 7, 13), (1, 4, 4), 0, 1,
                          "block_mean", route_radius=1),
}

SHIFT_CYCLES = {
    "tiny": [(0, 4, 4)],
    "flux1k": [(0, 0, 0), (0, 8, 0), (0, 0, 8), (0, 8, 8)],
    "flux2k": [(0, 0, 0), (0, 16, 0), (0, 0, 16), (0, 16, 16)],
    "flux4k": [(0, 16, 16)],
    "wan": [(0, 3, 6)],
    "wan_video": [(0, 0, 0), (0, 7, 13)],
}


def _to_dtype(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.clone()


def make_inputs(wl: Workload, seed: int = 0, heads=None):
    """Return (q, k, v) CPU tensors: q [B,h,N,d]; k, v [B,h,N+n_text,d].

    ``heads`` optionally restricts generation to a subset of heads (the draws for the
    other heads are still made, so a head's values do not depend on the subset).
    """
    T, H, W = wl.grid
    N, d, B, nh = wl.N, wl.d, wl.B, wl.heads
    keep = list(range(nh)) if heads is None else list(heads)
    out = {}
    for name in ("q", "k", "v"):
        rng = rng_for(seed, name)
        if wl.field == "iid":
            vis = iid_normal(rng, (B, nh, N, d))
        elif wl.field == "sinusoid":
            noise = iid_normal(rng, (B, nh, N, d), 0.5)
            vis = noise + sinusoid_field(rng, nh, T, H, W, d)[None]
        elif wl.field == "block_mean":
            if name == "v":
                vis = iid_normal(rng, (B, nh, N, d))
            else:
                noise = iid_normal(rng, (B, nh, N, d), 0.5)
                mrng = rng_for(seed, "mu_" + name)
                vis = noise + block_mean_field(mrng, nh, T, H, W, d, wl.window, wl.shift)[None]
        else:
            raise ValueError(wl.field)
        if name != "q" and wl.n_text > 0:
            trng = rng_for(seed, name + "_text")
            txt = iid_normal(trng, (B, nh, wl.n_text, d), 0.5 if wl.field != "iid" else 1.0)
            vis = np.concatenate([vis, txt], axis=2)
        out[name] = _to_dtype(vis[:, keep], wl.dtype)
    return out["q"], out["k"], out["v"]

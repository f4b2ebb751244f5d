"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare with the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_MAX_ABS = 1e-4
ROUTE_SCORE_TOL = 1e-3


def geometry(wl, shift=None) -> O.Geometry:
    return O.Geometry(grid=wl.grid, window=wl.window, shift=tuple(shift if shift is not None else wl.shift),
                      pool=wl.pool, n_text=wl.n_text, routed_k=wl.routed_k, route_radius=wl.route_radius)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def assert_outputs_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    d = np.abs(gpu - ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite GPU output"
    if dtype == "bf16":
        assert d.max() <= BF16_MAX_ABS, f"{what}: max abs {d.max():.3e} > {BF16_MAX_ABS}"
        assert d.mean() <= BF16_MEAN_ABS, f"{what}: mean abs {d.mean():.3e} > {BF16_MEAN_ABS}"
    else:
        assert d.max() <= F32_MAX_ABS, f"{what}: max abs {d.max():.3e} > {F32_MAX_ABS}"
    return float(d.max()), float(d.mean())


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def assert_pool_close(gpu: np.ndarray, ref: np.ndarray, dtype: str):
    """bf16: within one bf16 ulp of the exact mean (rounding once from a float32
    sum); float32: within 1e-6 relative."""
    if dtype == "bf16":
        bad = np.abs(gpu - ref) > bf16_ulp(ref)
        assert not bad.any(), f"{bad.sum()} pooled values off by more than one bf16 ulp"
    else:
        np.testing.assert_allclose(gpu, ref, rtol=1e-6, atol=1e-6)


def check_routes(gpu_idx: np.ndarray, ref_idx: np.ndarray, S: np.ndarray):
    """Routing acceptance: ids equal in order, except that a pick whose oracle
    score lies within 1e-3 * max(1, |k-th score|) of the oracle's k-th score is
    accepted either way (near-ties may fall differently in float32). Returns the
    number of (b, head, window) rows whose ids differ from the oracle's."""
    B, h, nw, k = ref_idx.shape
    differing = 0
    for b in range(B):
        for hh in range(h):
            for w in range(nw):
                g, r = gpu_idx[b, hh, w], ref_idx[b, hh, w]
                if np.array_equal(g, r):
                    continue
                differing += 1
                assert len(set(g.tolist())) == k and w not in g and g.min() >= 0 and g.max() < nw
                sk = S[b, hh, w, r[-1]]
                tol = ROUTE_SCORE_TOL * max(1.0, abs(sk))
                for pos in range(k):
                    if g[pos] != r[pos]:
                        assert abs(S[b, hh, w, g[pos]] - sk) <= tol, (b, hh, w, g, r)
    return differing


def gpu_inputs(wl, seed=0, device="cuda"):
    q, k, v = synth.make_inputs(wl, seed)
    return (q, k, v), (q.to(device), k.to(device), v.to(device))


def oracle_pool_for_gpu(k64, v64, geo, dtype):
    """Oracle pooled K/V, rounded to the kernel's element type (oracle-side rounding)."""
    kp, vp = O.pool_kv(k64, v64, geo)
    if dtype == "bf16":
        kp, vp = O.round_to_bf16(kp), O.round_to_bf16(vp)
    return kp, vp


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return (t.to(torch.bfloat16) if dtype == "bf16" else t).to(device)

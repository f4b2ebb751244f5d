"""GPU parity of the bfloat16 backward (tensor cores): basa_window_attn_bwd against the
oracle's basa_attention_backward (float64), with the oracle's routing, on small shapes
with every key group and on the FLUX 1024^2, FLUX 2048^2 and Wan workload shapes
(oracle on a subset of heads), plus run-to-run bitwise determinism.

Tolerance, from the arithmetic of the kernels: P and dS are rounded once to bfloat16
(relative error <= 2^-9) before the tensor-core products, D = dout . out uses the
forward's bfloat16 output, and dq, dk, dv are rounded once to bfloat16 (<= 2^-9).
Every output element is a sum of >= 64 products, each carrying one such rounding, so
its expected relative L2 error is a few times 2^-9 / sqrt(3) ~ 1.1e-3; the bound is
1e-2 on the relative L2 error of each tensor (global) and 5e-2 on each row's (rows
with a norm below 5% of the tensor's RMS row norm are held to that absolute floor
instead, since a row that small carries the errors of its large terms).
BASA §3.4 (dense-teacher adaptation trains through this operator).
"""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload
REL_L2 = 1e-2
ROW_REL = 5e-2
ROW_FLOOR = 0.05

SMALL = [
    # pooled + text + routing with every window type wrapping (3-D shift)
    W("wrap3d", "bf16", 1, 2, 128, (4, 8, 12), (2, 4, 4), (1, 2, 3), (2, 4, 4), 77, 3, "block_mean"),
    # odd windows (117-row tiles), batch 2, text and routing
    W("odd", "bf16", 2, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean"),
    # own window only
    W("own_only", "bf16", 1, 2, 128, (1, 32, 32), (1, 16, 16), (0, 8, 8), (0, 0, 0), 0, 0, "iid"),
    # pooled keys not a multiple of 128 (144), ragged text (200 rows = two tiles)
    W("ragged", "bf16", 1, 2, 128, (1, 48, 48), (1, 16, 16), (0, 8, 8), (1, 4, 4), 200, 0, "sinusoid"),
    # video variant: full-T windows, spatial pooling, radius-one routing
    W("video", "bf16", 1, 2, 128, (5, 24, 32), (5, 6, 8), (2, 3, 4), (1, 2, 2), 0, 3, "block_mean", route_radius=1),
    # one window routed to by many (most of the grid): a long query list for one key tile
    W("hub", "bf16", 1, 1, 128, (1, 64, 64), (1, 8, 8), (0, 4, 4), (0, 0, 0), 0, 2, "iid"),
]


def _heads(wl):
    return list(range(wl.heads)) if wl.heads <= 4 else sorted({0, wl.heads // 2, wl.heads - 1})


def _compare(name, g, r):
    g2 = g.reshape(-1, g.shape[-1])
    r2 = r.reshape(-1, r.shape[-1])
    err = g2 - r2
    rel = np.linalg.norm(err) / max(np.linalg.norm(r2), 1e-30)
    assert np.isfinite(g2).all(), f"{name}: non-finite"
    assert rel <= REL_L2, f"{name}: relative L2 error {rel:.3e} > {REL_L2}"
    rn = np.linalg.norm(r2, axis=1)
    en = np.linalg.norm(err, axis=1)
    floor = ROW_FLOOR * np.sqrt(np.mean(rn ** 2))
    worst = np.max(en / np.maximum(rn, floor))
    assert worst <= ROW_REL, f"{name}: worst row relative error {worst:.3e} > {ROW_REL}"
    return rel, worst


def _hub_route(geo, hub):
    """Routing where every window picks window `hub` first (then its lowest other id)."""
    r = np.zeros((1, 1, geo.n_win, geo.routed_k), dtype=np.int32)
    for w in range(geo.n_win):
        picks = [hub] if w != hub else []
        u = 0
        while len(picks) < geo.routed_k:
            if u != w and u not in picks:
                picks.append(u)
            u += 1
        r[0, 0, w] = picks
    return r


def run_backward(wl, seed=0, twice=False):
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl, seed)
    geo = PT.geometry(wl)
    hs = _heads(wl)
    q64, k64, v64 = PT.to64(q[:, hs]), PT.to64(k[:, hs]), PT.to64(v[:, hs])
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                      route_radius=wl.route_radius)
    route = None
    if geo.has_pool:
        layer.pool_kv(kd, vd, wl.shift)
    if geo.routed_k:
        if wl.name == "hub":
            route_all = _hub_route(geo, hub=27)
        else:
            layer.route(qd, kd, wl.shift)
            torch.cuda.synchronize()
            route_all = layer.route_idx.cpu().numpy()
            route_all[:, hs] = O.route_windows(q64, k64, geo)[0]
        layer.route_idx.copy_(torch.from_numpy(route_all))
        route = route_all[:, hs]
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out, lse, wl.shift, B.BASA_KEYS_ALL)
    rng = np.random.default_rng(seed + 17)
    dout = torch.from_numpy(rng.standard_normal(q.shape, dtype=np.float32)).to(torch.bfloat16)
    dq, dk, dv = layer.backward(qd, kd, vd, out, lse, dout.cuda(), wl.shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    if twice:
        dq2, dk2, dv2 = layer.backward(qd, kd, vd, out, lse, dout.cuda(), wl.shift)
        torch.cuda.synchronize()
        assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2), "not deterministic"
    do64 = PT.to64(dout[:, hs])
    rq, rk, rv = O.basa_attention_backward(q64, k64, v64, geo, do64, route_idx=route)
    res = {}
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        res[name] = _compare(f"{wl.name} {name}", PT.to64(g[:, hs]), r)
    return res


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_backward_bf16_small(wl):
    run_backward(wl, twice=True)


def test_backward_bf16_flux1k():
    run_backward(synth.WORKLOADS["flux1k"].with_shift((0, 8, 8)), twice=True)


def test_backward_bf16_flux2k():
    run_backward(synth.WORKLOADS["flux2k"].with_shift((0, 16, 16)))


def test_backward_bf16_wan():
    run_backward(synth.WORKLOADS["wan"], twice=True)

"""Route ids outside [0, nWin) are reported by the kernels that read them.

The attention kernels (bf16 and float32 forward, bf16 backward) check each route id
they load; one outside the window range sets BASA_DEVERR_BAD_ROUTE in the device
error word and the routed window is read from the query's own window instead, so
nothing is accessed out of bounds. The bf16 forward's output then equals the oracle
run with the same substitution (the own window listed twice).
"""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload


def _bad_routes(layer, geo, wl):
    """Valid routes with a few ids replaced by -1, nWin and 10^6; returns the device
    ids and the ids the kernels are expected to use instead."""
    layer.route(*_inputs(wl)[1][:2], wl.shift)
    torch.cuda.synchronize()
    route = layer.route_idx.cpu().numpy().copy()
    fixed = route.copy()
    for (b, h, w, r), bad in zip([(0, 0, 0, 0), (0, 1, 3, 1), (0, 0, geo.n_win - 1, 0)], (-1, geo.n_win, 10 ** 6)):
        route[b, h, w, r] = bad
        fixed[b, h, w, r] = w
    return route, fixed


_CACHE = {}


def _inputs(wl):
    if wl.name not in _CACHE:
        _CACHE[wl.name] = PT.gpu_inputs(wl, seed=11)
    return _CACHE[wl.name]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bad_route_id_is_reported_and_contained(dtype):
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    wl = W(f"badroute_{dtype}", dtype, 1, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean")
    geo = PT.geometry(wl)
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
    (q, k, v), (qd, kd, vd) = _inputs(wl)
    layer.pool_kv(kd, vd, wl.shift)
    route, fixed = _bad_routes(layer, geo, wl)
    layer.route_idx.copy_(torch.from_numpy(route))
    layer.dev_err.zero_()
    out = torch.full_like(qd, float("nan"))
    layer.attention(qd, kd, vd, out, wl.shift)
    torch.cuda.synchronize()
    word = layer.device_error()
    assert word & B.BASA_DEVERR_BAD_ROUTE, word
    assert B.basa_device_error_status(word) == 6  # BASA_ERR_BAD_INDEX
    q64, k64, v64 = PT.to64(q), PT.to64(k), PT.to64(v)
    kp, vp = PT.oracle_pool_for_gpu(k64, v64, geo, wl.dtype)
    ref = O.basa_attention(q64, k64, v64, geo, kp=kp, vp=vp, route_idx=fixed)
    PT.assert_outputs_close(PT.to64(out), ref, wl.dtype, "attention with substituted routes")
    # the layer is usable afterwards: valid routes, clean error word
    layer.route_idx.copy_(torch.from_numpy(fixed))
    layer.dev_err.zero_()
    layer.attention(qd, kd, vd, out, wl.shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0


def test_bad_route_id_in_backward_is_reported():
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    wl = W("badroute_bwd", "bf16", 1, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean")
    geo = PT.geometry(wl)
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
    _, (qd, kd, vd) = _inputs(wl)
    layer.pool_kv(kd, vd, wl.shift)
    route, _ = _bad_routes(layer, geo, wl)
    layer.route_idx.copy_(torch.from_numpy(route))
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out, lse, wl.shift, B.BASA_KEYS_ALL)
    torch.cuda.synchronize()
    layer.dev_err.zero_()
    dq, dk, dv = layer.backward(qd, kd, vd, out, lse, torch.randn_like(qd), wl.shift)
    torch.cuda.synchronize()
    assert layer.device_error() & B.BASA_DEVERR_BAD_ROUTE
    assert all(torch.isfinite(t.float()).all() for t in (dq, dk, dv))

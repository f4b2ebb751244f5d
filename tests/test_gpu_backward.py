"""GPU parity of the backward (float32): basa_window_attn_bwd against the oracle's
basa_attention_backward, with the oracle's routing and the GPU forward's lse."""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = [
    W("f32_d128", "f32", 1, 2, 128, (2, 16, 16), (1, 8, 8), (1, 4, 2), (2, 4, 4), 9, 2, "block_mean"),
    W("no_pool", "f32", 2, 2, 128, (1, 24, 16), (1, 8, 8), (0, 5, 3), (0, 0, 0), 0, 1, "iid"),
    W("video_r1", "f32", 1, 1, 128, (4, 12, 16), (4, 4, 4), (0, 2, 2), (1, 2, 2), 3, 2, "block_mean", route_radius=1),
    W("own_only", "f32", 1, 2, 128, (1, 16, 16), (1, 8, 8), (0, 4, 4), (0, 0, 0), 0, 0, "iid"),
]
TOL = 2e-4


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_backward_matches_oracle(wl):
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl)
    geo = PT.geometry(wl)
    q64, k64, v64 = PT.to64(q), PT.to64(k), PT.to64(v)
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                      route_radius=wl.route_radius)
    route = None
    if geo.has_pool:
        layer.pool_kv(kd, vd, wl.shift)
    if geo.routed_k:
        route = O.route_windows(q64, k64, geo)[0]
        layer.route_idx.copy_(torch.from_numpy(route))
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out, lse, wl.shift, B.BASA_KEYS_ALL)
    rng = np.random.default_rng(17)
    dout = torch.from_numpy(rng.standard_normal(q.shape, dtype=np.float32))
    dq, dk, dv = layer.backward(qd, kd, vd, out, lse, dout.cuda(), wl.shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    rq, rk, rv = O.basa_attention_backward(q64, k64, v64, geo, dout.numpy().astype(np.float64), route_idx=route)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = np.abs(PT.to64(g) - r).max()
        assert err <= TOL, f"{wl.name} {name}: max abs {err:.3e}"

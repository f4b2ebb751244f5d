"""GPU parity of the branch form (BASA §A.1): attention over selected key groups
with its log-sum-exp, and the merge of branches into the joint softmax, against
the oracle's branch_attention / merge_branches / basa_attention."""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload
LSE_TOL = {"bf16": 1e-3, "f32": 1e-5}

CASES = [
    synth.WORKLOADS["flux1k"].with_shift((0, 8, 8)),
    synth.WORKLOADS["wan"],
    synth.WORKLOADS["tiny"],
    W("text77", "bf16", 1, 2, 128, (1, 48, 48), (1, 16, 16), (0, 8, 8), (1, 4, 4), 77, 0, "sinusoid"),
    W("odd", "bf16", 2, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean"),
    W("f32_d128", "f32", 1, 2, 128, (2, 16, 16), (1, 8, 8), (1, 4, 2), (2, 4, 4), 9, 2, "block_mean"),
]


def _setup(wl):
    from sparse_window_attention_b200.layer import BasaLayer

    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl)
    geo = PT.geometry(wl)
    hs = list(range(wl.heads)) if wl.heads <= 4 else [0, wl.heads - 1]
    q64, k64, v64 = PT.to64(q[:, hs]), PT.to64(k[:, hs]), PT.to64(v[:, hs])
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                      route_radius=wl.route_radius)
    kp_or = vp_or = route_or = None
    if geo.has_pool:
        kp_or, vp_or = PT.oracle_pool_for_gpu(k64, v64, geo, wl.dtype)
        layer.pool_kv(kd, vd, wl.shift)
        layer.kp[:, hs] = PT.to_device(kp_or, wl.dtype)
        layer.vp[:, hs] = PT.to_device(vp_or, wl.dtype)
    if geo.routed_k:
        route_or, _ = O.route_windows(q64, k64, geo)
        layer.route(qd, kd, wl.shift)
        layer.route_idx[:, hs] = torch.from_numpy(route_or).to(layer.route_idx.device)
    torch.cuda.synchronize()
    return layer, geo, hs, (qd, kd, vd), (q64, k64, v64), (kp_or, vp_or, route_or)


def _splits(geo):
    glob = (O.KEYS_POOLED if geo.has_pool else 0) | (O.KEYS_TEXT if geo.n_text else 0)
    out = []
    if glob:
        out.append([O.KEYS_WINDOWS, glob])
    if geo.has_pool and geo.n_text:
        out.append([O.KEYS_WINDOWS, O.KEYS_POOLED, O.KEYS_TEXT])
    return out


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_branch_form_matches_joint_softmax(wl):
    layer, geo, hs, (qd, kd, vd), (q64, k64, v64), (kp_or, vp_or, route_or) = _setup(wl)
    shift = wl.shift
    # the whole key list with its lse: same output as the plain call, lse as the oracle's
    ref_out, ref_lse = O.branch_attention(q64, k64, v64, geo, O.KEYS_ALL, kp=kp_or, vp=vp_or, route_idx=route_or)
    out_plain = torch.empty_like(qd)
    layer.attention(qd, kd, vd, out_plain, shift)
    out_all = torch.empty_like(qd)
    lse_all = torch.full(qd.shape[:-1], float("nan"), dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out_all, lse_all, shift, O.KEYS_ALL)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert torch.equal(out_all, out_plain)
    assert not torch.isnan(lse_all).any()
    np.testing.assert_allclose(lse_all[:, hs].cpu().numpy(), ref_lse, rtol=0, atol=LSE_TOL[wl.dtype])
    PT.assert_outputs_close(PT.to64(out_all[:, hs]), ref_out, wl.dtype, "keys=all")
    for parts in _splits(geo):
        outs, lses = [], []
        for keys in parts:
            o = torch.full_like(qd, float("nan"))
            lse = torch.full(qd.shape[:-1], float("nan"), dtype=torch.float32, device=qd.device)
            layer.attention_lse(qd, kd, vd, o, lse, shift, keys)
            torch.cuda.synchronize()
            assert layer.device_error() == 0
            bo, bl = O.branch_attention(q64, k64, v64, geo, keys, kp=kp_or, vp=vp_or, route_idx=route_or)
            PT.assert_outputs_close(PT.to64(o[:, hs]), bo, wl.dtype, f"branch {keys}")
            np.testing.assert_allclose(lse[:, hs].cpu().numpy(), bl, rtol=0, atol=LSE_TOL[wl.dtype])
            outs.append(o)
            lses.append(lse)
        merged = torch.empty_like(qd)
        merged_lse = torch.empty_like(lses[0])
        layer.merge(outs, lses, merged, merged_lse)
        torch.cuda.synchronize()
        PT.assert_outputs_close(PT.to64(merged[:, hs]), ref_out, wl.dtype, f"merge {parts}")
        np.testing.assert_allclose(merged_lse[:, hs].cpu().numpy(), ref_lse, rtol=0, atol=LSE_TOL[wl.dtype])
        # in place: the merged result may overwrite the first branch
        layer.merge(outs, lses, outs[0], None)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], merged)


def test_layer_forward_in_branch_form():
    """The whole layer (pooling, routing, branches, merge) against the oracle."""
    wl = W("odd", "bf16", 2, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean")
    from sparse_window_attention_b200.layer import BasaLayer

    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl)
    geo = PT.geometry(wl)
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
    out = layer.forward_branches(qd, kd, vd, wl.shift, [O.KEYS_WINDOWS, O.KEYS_POOLED | O.KEYS_TEXT])
    torch.cuda.synchronize()
    q64, k64, v64 = PT.to64(q), PT.to64(k), PT.to64(v)
    assert (layer.route_idx.cpu().numpy() == O.route_windows(q64, k64, geo)[0]).all()
    PT.assert_outputs_close(PT.to64(out), O.basa_attention(q64, k64, v64, geo), wl.dtype, "branch-form layer")

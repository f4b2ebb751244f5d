"""GPU parity: the CUDA path through the C ABI against the oracle, element by
element, on the same seeded inputs.

* The five workload shapes at full size (large ones checked on a subset of
  heads, every window of those heads), in the launch configuration bench.py times.
* Small shapes that span several tiles with ragged tails and the degenerate cases.
Attention parity is decoupled from pooling/routing parity: the attention kernel
is also fed the oracle's pooled K/V (rounded to bf16 by the oracle) and the
oracle's routed ids; the end-to-end test then runs the three kernels in a row.
"""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload


def _layer(wl):
    from sparse_window_attention_b200.layer import BasaLayer

    return BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                     route_radius=wl.route_radius)


def _heads(wl):
    return list(range(wl.heads)) if wl.heads <= 4 else sorted({0, wl.heads // 2, wl.heads - 1})


def run_parity(wl, shift, seed=0, e2e=True):
    """Pool, route and attention parity for one workload at one shift."""
    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl, seed)
    geo = PT.geometry(wl, shift)
    hs = _heads(wl)
    q64, k64, v64 = PT.to64(q[:, hs]), PT.to64(k[:, hs]), PT.to64(v[:, hs])
    layer = _layer(wl)
    report = {}
    kp_or = vp_or = None
    kp_dev = vp_dev = None
    if geo.has_pool:
        layer.pool_kv(kd, vd, shift)
        torch.cuda.synchronize()
        kp_ex, vp_ex = O.pool_kv(k64, v64, geo)
        PT.assert_pool_close(PT.to64(layer.kp[:, hs]), kp_ex, wl.dtype)
        PT.assert_pool_close(PT.to64(layer.vp[:, hs]), vp_ex, wl.dtype)
        kp_or, vp_or = PT.oracle_pool_for_gpu(k64, v64, geo, wl.dtype)
        # the kernel gets the oracle's rounded pooled K/V for every head; only `hs` are compared
        kp_dev = layer.kp.clone()
        vp_dev = layer.vp.clone()
        kp_dev[:, hs] = PT.to_device(kp_or, wl.dtype)
        vp_dev[:, hs] = PT.to_device(vp_or, wl.dtype)
    route_or = route_dev = None
    if geo.routed_k:
        layer.route(qd, kd, shift)
        torch.cuda.synchronize()
        route_or, S = O.route_windows(q64, k64, geo)
        report["route_rows_differing"] = PT.check_routes(layer.route_idx[:, hs].cpu().numpy(), route_or, S)
        # GPU scores agree with the oracle's for the chosen ids
        gs = layer.route_score[:, hs].cpu().numpy().astype(np.float64)
        gi = layer.route_idx[:, hs].cpu().numpy()
        ref = np.take_along_axis(S, gi.astype(np.int64), axis=3)
        assert np.all(np.abs(gs - ref) <= PT.ROUTE_SCORE_TOL * np.maximum(1.0, np.abs(ref)))
        route_dev = layer.route_idx.clone()
        route_dev[:, hs] = torch.from_numpy(route_or).to(route_dev.device)
    out = torch.full_like(qd, float("nan"))
    layer.attention(qd, kd, vd, out, shift, kp=kp_dev, vp=vp_dev, route_idx=route_dev)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.basa_attention(q64, k64, v64, geo, kp=kp_or, vp=vp_or, route_idx=route_or)
    report["attn"] = PT.assert_outputs_close(PT.to64(out[:, hs]), ref, wl.dtype, f"{wl.name} attention")
    if e2e:
        out2 = layer.forward(qd, kd, vd, shift)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        ref2 = O.basa_attention(q64, k64, v64, geo)  # float64 pooling, oracle routing
        g2 = PT.to64(out2[:, hs])
        if geo.routed_k:
            same = (layer.route_idx[:, hs].cpu().numpy() == O.route_windows(q64, k64, geo)[0]).all(axis=-1)
            win = O.window_of_token(geo)
            keep = same[:, :, win]  # [B, h, N] queries whose window was routed like the oracle's
            assert keep.mean() > 0.99
            g2 = np.where(keep[..., None], g2, ref2)
        report["e2e"] = PT.assert_outputs_close(g2, ref2, wl.dtype, f"{wl.name} end to end")
    return report


# ----------------------------------------------------------------- full-size workloads


@pytest.mark.parametrize("shift", synth.SHIFT_CYCLES["flux1k"])
def test_flux1k_every_shift(shift):
    run_parity(synth.WORKLOADS["flux1k"], shift)


@pytest.mark.parametrize("shift", synth.SHIFT_CYCLES["flux2k"])
def test_flux2k_every_shift(shift):
    run_parity(synth.WORKLOADS["flux2k"], shift, e2e=shift == (0, 16, 16))


def test_flux4k():
    run_parity(synth.WORKLOADS["flux4k"], (0, 16, 16))


def test_wan():
    r = run_parity(synth.WORKLOADS["wan"], (0, 3, 6))
    assert r["route_rows_differing"] == 0


def test_tiny_f32():
    run_parity(synth.WORKLOADS["tiny"], (0, 4, 4))


def sampled_rows(geo, n_random, seed):
    """Query tokens to check on a large grid: random ones plus the first and last
    tokens (shifted-frame raster order) of every window, which sit in the first and
    last, ragged, query tiles."""
    rng = np.random.default_rng(seed)
    win = O.window_of_token(geo)
    picks = set(rng.choice(geo.N, size=n_random, replace=False).tolist())
    for w in range(geo.n_win):
        members = np.nonzero(win == w)[0]  # original indices; shifted order differs
        picks.update(members[[0, len(members) // 2, -1]].tolist())
    return np.array(sorted(picks))


_LARGE = {}  # the last large workload's inputs, reused across its shifts


def _large_inputs(wl, seed):
    key = (wl.name, seed)
    if key not in _LARGE:
        _LARGE.clear()
        (q, k, v), dev = PT.gpu_inputs(wl, seed)
        hs = _heads(wl)
        _LARGE[key] = (dev, (PT.to64(q[:, hs]), PT.to64(k[:, hs]), PT.to64(v[:, hs])))
    return _LARGE[key]


def run_sampled_parity(wl, shift, n_random=96, seed=0):
    """Full-size pool and routing parity on a head subset, attention parity on
    sampled query rows (the oracle computes them one by one)."""
    (qd, kd, vd), (q64, k64, v64) = _large_inputs(wl, seed)
    geo = PT.geometry(wl, shift)
    hs = _heads(wl)
    layer = _layer(wl)
    layer.pool_kv(kd, vd, shift)
    layer.route(qd, kd, shift)
    torch.cuda.synchronize()
    kp_ex, vp_ex = O.pool_kv(k64, v64, geo)
    PT.assert_pool_close(PT.to64(layer.kp[:, hs]), kp_ex, wl.dtype)
    PT.assert_pool_close(PT.to64(layer.vp[:, hs]), vp_ex, wl.dtype)
    route_or, S = O.route_windows(q64, k64, geo)
    differing = PT.check_routes(layer.route_idx[:, hs].cpu().numpy(), route_or, S)
    kp_or, vp_or = PT.oracle_pool_for_gpu(k64, v64, geo, wl.dtype)
    kp_dev, vp_dev, route_dev = layer.kp.clone(), layer.vp.clone(), layer.route_idx.clone()
    kp_dev[:, hs] = PT.to_device(kp_or, wl.dtype)
    vp_dev[:, hs] = PT.to_device(vp_or, wl.dtype)
    route_dev[:, hs] = torch.from_numpy(route_or).to(route_dev.device)
    out = torch.full_like(qd, float("nan"))
    layer.attention(qd, kd, vd, out, shift, kp=kp_dev, vp=vp_dev, route_idx=route_dev)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert not torch.isnan(out).any()  # every query row was written
    rows = sampled_rows(geo, n_random, seed)
    for j in range(len(hs)):
        ref = O.attention_rows(q64, k64, v64, geo, 0, j, rows, kp=kp_or, vp=vp_or, route_idx=route_or)
        PT.assert_outputs_close(PT.to64(out[0, hs[j]][rows]), ref, wl.dtype, f"{wl.name} head {hs[j]}")
    return differing


@pytest.mark.parametrize("shift", synth.SHIFT_CYCLES["wan_video"])
def test_wan_video_full_size(shift):
    """The pages' video configuration at 21x60x104: 15x26 spatial windows over all
    frames, spatial-only 4x4 pooling, one routed window among radius-one neighbours."""
    differing = run_sampled_parity(synth.WORKLOADS["wan_video"], shift)
    assert differing == 0


# ----------------------------------------------------------------- fused pool + routing pass


def run_fused_parity(wl, shift, seed=0, large=False):
    """basa_pool_route (one read of q, k, v) against the oracle's pooling and routing."""
    from sparse_window_attention_b200 import binding as B

    if large:
        (qd, kd, vd), (q64, k64, v64) = _large_inputs(wl, seed)
    else:
        (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl, seed)
        hs0 = _heads(wl)
        q64, k64, v64 = PT.to64(q[:, hs0]), PT.to64(k[:, hs0]), PT.to64(v[:, hs0])
    geo = PT.geometry(wl, shift)
    hs = _heads(wl)
    layer = _layer(wl)
    assert layer.fused_bytes(shift) > 0, "shape not supported by the fused pass"
    layer.kp.fill_(float("nan"))
    layer.vp.fill_(float("nan"))
    layer.route_idx.fill_(-1)
    layer.pool_route(qd, kd, vd, shift)
    torch.cuda.synchronize()
    assert not torch.isnan(layer.kp).any() and not torch.isnan(layer.vp).any()
    kp_ex, vp_ex = O.pool_kv(k64, v64, geo)
    PT.assert_pool_close(PT.to64(layer.kp[:, hs]), kp_ex, wl.dtype)
    PT.assert_pool_close(PT.to64(layer.vp[:, hs]), vp_ex, wl.dtype)
    route_or, S = O.route_windows(q64, k64, geo)
    differing = PT.check_routes(layer.route_idx[:, hs].cpu().numpy(), route_or, S)
    gs = layer.route_score[:, hs].cpu().numpy().astype(np.float64)
    ref = np.take_along_axis(S, layer.route_idx[:, hs].cpu().numpy().astype(np.int64), axis=3)
    assert np.all(np.abs(gs - ref) <= PT.ROUTE_SCORE_TOL * np.maximum(1.0, np.abs(ref)))
    # the window means at the head of the workspace match the oracle's
    T, H, W = wl.grid
    nwin = geo.n_win
    means = layer.fused_workspace[: 2 * wl.B * wl.heads * nwin * wl.d * 4].view(torch.float32)
    means = means.view(2, wl.B, wl.heads, nwin, wl.d)[:, :, hs].cpu().numpy().astype(np.float64)
    qm, km = O.window_means(q64, k64, geo)
    np.testing.assert_allclose(means[0], qm, rtol=0, atol=1e-5 * max(1.0, np.abs(qm).max()))
    np.testing.assert_allclose(means[1], km, rtol=0, atol=1e-5 * max(1.0, np.abs(km).max()))
    return differing


FUSED = [
    W("wrap3d", "bf16", 1, 2, 128, (4, 8, 12), (2, 4, 4), (1, 2, 3), (2, 4, 4), 0, 11, "block_mean"),
    W("odd", "bf16", 2, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean"),
    W("rows", "bf16", 1, 2, 128, (1, 4, 80), (1, 1, 40), (0, 1, 17), (1, 2, 8), 0, 1, "iid"),
    # window wider than the box on every axis, the box spanning the whole t axis
    W("whole_t", "bf16", 1, 2, 128, (5, 24, 32), (5, 6, 8), (2, 3, 4), (5, 2, 2), 0, 3, "block_mean", route_radius=1),
    # pool patches larger than windows along x, pooled box wider than the grid's windows
    W("wide_pool", "bf16", 1, 2, 128, (2, 16, 48), (1, 4, 6), (1, 1, 5), (2, 4, 12), 3, 2, "iid"),
    W("f32_d128", "f32", 1, 2, 128, (2, 16, 16), (1, 8, 8), (1, 4, 2), (2, 4, 4), 9, 2, "block_mean"),
    W("f32_d64", "f32", 2, 3, 64, (1, 24, 16), (1, 8, 8), (0, 5, 3), (1, 4, 4), 0, 1, "iid"),
    W("bf16_d64", "bf16", 1, 2, 64, (1, 24, 16), (1, 8, 8), (0, 5, 3), (1, 4, 4), 0, 1, "iid"),
]


@pytest.mark.parametrize("wl", FUSED, ids=[w.name for w in FUSED])
def test_fused_pool_route_small(wl):
    run_fused_parity(wl, wl.shift)


def test_fused_pool_route_wan():
    assert run_fused_parity(synth.WORKLOADS["wan"], (0, 3, 6)) == 0


@pytest.mark.parametrize("shift", synth.SHIFT_CYCLES["wan_video"])
def test_fused_pool_route_wan_video(shift):
    assert run_fused_parity(synth.WORKLOADS["wan_video"], shift, large=True) == 0
    if shift == synth.SHIFT_CYCLES["wan_video"][-1]:
        _LARGE.clear()


# ----------------------------------------------------------------- small shapes, edge cases

SMALL = [
    # ragged text (77 rows) and a pooled count that is not a multiple of 128 (144)
    W("text77", "bf16", 1, 2, 128, (1, 48, 48), (1, 16, 16), (0, 8, 8), (1, 4, 4), 77, 0, "sinusoid"),
    # no pooled keys, no text, no routing: own window only
    W("own_only", "bf16", 2, 2, 128, (1, 64, 64), (1, 16, 16), (0, 8, 8), (0, 0, 0), 0, 0, "iid"),
    # window = whole grid, shift 0: dense attention (closed form)
    W("dense", "bf16", 1, 2, 128, (1, 16, 24), (1, 16, 24), (0, 0, 0), (0, 0, 0), 0, 0, "iid"),
    # 3-D with a shift in t, y and x (all eight window types), routing to every other window
    W("wrap3d", "bf16", 1, 2, 128, (4, 8, 12), (2, 4, 4), (1, 2, 3), (2, 4, 4), 0, 11, "block_mean"),
    # odd window extents, two query tiles of 117 rows, batch 2
    W("odd", "bf16", 2, 2, 128, (3, 12, 26), (3, 6, 13), (0, 3, 6), (3, 6, 13), 5, 2, "block_mean"),
    # single-row boxes: window 1 x 1 x 40 (40-token pieces), shift 17
    W("rows", "bf16", 1, 2, 128, (1, 4, 80), (1, 1, 40), (0, 1, 17), (1, 2, 8), 0, 1, "iid"),
    # float32 variants: head_dim 128, routing, text
    W("f32_d128", "f32", 1, 2, 128, (2, 16, 16), (1, 8, 8), (1, 4, 2), (2, 4, 4), 9, 2, "block_mean"),
    W("f32_d64", "f32", 2, 3, 64, (1, 24, 16), (1, 8, 8), (0, 5, 3), (1, 4, 4), 0, 1, "iid"),
    # video variant: windows over all frames, spatial-only pooling, radius-one routing
    W("video", "bf16", 1, 2, 128, (5, 24, 32), (5, 6, 8), (0, 3, 4), (1, 2, 2), 0, 1, "block_mean", route_radius=1),
    # the same with a temporal shift (every window wraps in t) and the most routed
    # windows radius one allows on a 4x4 window grid (a corner has 3 neighbours)
    W("video_tshift", "bf16", 1, 2, 128, (5, 24, 32), (5, 6, 8), (2, 3, 4), (1, 2, 2), 0, 3, "block_mean",
      route_radius=1),
    # radius two on a 6x6 window grid, float32
    W("f32_radius2", "f32", 1, 2, 64, (1, 24, 24), (1, 4, 4), (0, 2, 1), (1, 4, 4), 0, 8, "iid", route_radius=2),
    # 1152 windows per head: staging of the candidates' means in several chunks
    W("many_windows", "bf16", 1, 1, 128, (1, 128, 144), (1, 4, 4), (0, 2, 2), (0, 0, 0), 0, 2, "block_mean"),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_small_shapes(wl):
    run_parity(wl, wl.shift)


def test_max_routed_k():
    wl = W("k16", "bf16", 1, 1, 128, (1, 40, 40), (1, 8, 8), (0, 4, 4), (1, 8, 8), 0, 16, "block_mean")
    run_parity(wl, wl.shift)


def test_empty_batch_launches_nothing():
    from sparse_window_attention_b200 import binding as B

    p = B.make_params(0, 24, 128, (1, 64, 64), (1, 16, 16), (0, 8, 8), (1, 8, 8), 512, 0, "bf16")
    assert B.basa_window_attn_fwd(None, None, None, None, None, None, None, p, check=False) == 0
    torch.cuda.synchronize()


def test_repeat_calls_are_deterministic():
    wl = synth.WORKLOADS["flux1k"]
    _, (qd, kd, vd) = PT.gpu_inputs(wl)
    layer = _layer(wl)
    a = layer.forward(qd, kd, vd, (0, 8, 8)).clone()
    b = layer.forward(qd, kd, vd, (0, 8, 8))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ----------------------------------------------------------------- every head of a full-size workload


@pytest.mark.parametrize("name,shift", [("wan", (0, 3, 6)), ("flux2k", (0, 16, 16))])
def test_every_head_full_size(name, shift):
    """Pooling and routing compared on EVERY head of a full-size workload, and the
    attention on sampled query rows of every head (a bug tied to the (batch, head)
    index, e.g. a middle head's route-id or tensor-map offset, shows up here)."""
    wl = synth.WORKLOADS[name]
    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl, 0)
    geo = PT.geometry(wl, shift)
    layer = _layer(wl)
    out = layer.forward(qd, kd, vd, shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    rng = np.random.default_rng(5)
    win = O.window_of_token(geo)
    for h in range(wl.heads):
        q64, k64, v64 = PT.to64(q[:, h:h + 1]), PT.to64(k[:, h:h + 1]), PT.to64(v[:, h:h + 1])
        kp_ex, vp_ex = O.pool_kv(k64, v64, geo)
        PT.assert_pool_close(PT.to64(layer.kp[:, h:h + 1]), kp_ex, wl.dtype)
        PT.assert_pool_close(PT.to64(layer.vp[:, h:h + 1]), vp_ex, wl.dtype)
        route = None
        if geo.routed_k:
            route, S = O.route_windows(q64, k64, geo)
            assert PT.check_routes(layer.route_idx[:, h:h + 1].cpu().numpy(), route, S) == 0, f"head {h}"
        # the kernel's own pooled K/V and routes, widened, are the oracle's inputs here:
        # this checks the attention of head h, given what the earlier kernels produced
        kp_g = PT.to64(layer.kp[:, h:h + 1])
        vp_g = PT.to64(layer.vp[:, h:h + 1])
        rows = np.unique(np.concatenate([rng.choice(wl.N, size=24, replace=False),
                                         [np.nonzero(win == rng.integers(geo.n_win))[0][-1]]]))
        ref = O.attention_rows(q64, k64, v64, geo, 0, 0, rows, kp=kp_g, vp=vp_g, route_idx=route)
        PT.assert_outputs_close(PT.to64(out[0, h][rows]), ref, wl.dtype, f"{name} head {h}")

"""GPU parity of the online softmax's rescale path.

The bfloat16 attention kernel keeps a running row max m and raises it only when a
key tile's max exceeds m by more than 8 (log2 units of the scaled score); only then
is the O accumulator in tensor memory multiplied by 2^(m_old - m_new) and the row
sum rescaled with it. On the workload fields the first key tiles already hold the
row max, so this branch would never run. The inputs here are built so that it runs,
often several times per row, in every mode it has:

* ``text staircase``: one channel of every even query is 16 and the same channel of
  text tile j (rows 128 j .. 128 j + 127 of the text keys) is 5 (j + 1), so each text
  tile lifts the even rows' max by ~10 log2 units (four rescales per row), while odd
  rows stay below the threshold: some lanes of a warp rescale and others do not.
* ``pooled key dominant``: the keys of one pool patch carry a large component along
  the queries' shared direction, so the pooled key (after the window tiles) wins.
* ``Q x 6`` on the FLUX 1024^2 shape: a wide score range everywhere.
* ``Wan, routed windows far above the own window``: the per-window means of the Wan
  field scaled x 3, so the routed windows' keys score far above the own window's.

Each case is compared element by element with the oracle (bf16 tolerances), and the
cases that must rescale assert it on the CPU from the oracle-side scores: for the
sampled rows, a later key group's max exceeds the max of every key before it by
more than 8 log2 units. BASA §A.1: one softmax over the concatenated keys.
"""
import math

import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload
LOG2E = 1.0 / math.log(2.0)
THRESH_LOG2 = 8.0


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _layer(wl):
    from sparse_window_attention_b200.layer import BasaLayer

    return BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                     route_radius=wl.route_radius)


def run_attn_parity(wl, q, k, v, heads):
    """Attention with the oracle's pooled K/V and routes, then the whole layer (GPU
    pooling and routing), both against the oracle on `heads`."""
    geo = PT.geometry(wl)
    shift = wl.shift
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    q64, k64, v64 = PT.to64(q[:, heads]), PT.to64(k[:, heads]), PT.to64(v[:, heads])
    layer = _layer(wl)
    kp_or = vp_or = route_or = None
    kp_dev = vp_dev = route_dev = None
    if geo.has_pool:
        layer.pool_kv(kd, vd, shift)
        torch.cuda.synchronize()
        kp_or, vp_or = PT.oracle_pool_for_gpu(k64, v64, geo, wl.dtype)
        kp_dev, vp_dev = layer.kp.clone(), layer.vp.clone()
        kp_dev[:, heads] = PT.to_device(kp_or, wl.dtype)
        vp_dev[:, heads] = PT.to_device(vp_or, wl.dtype)
    if geo.routed_k:
        layer.route(qd, kd, shift)
        torch.cuda.synchronize()
        route_or, _ = O.route_windows(q64, k64, geo)
        route_dev = layer.route_idx.clone()
        route_dev[:, heads] = torch.from_numpy(route_or).to(route_dev.device)
    out = torch.full_like(qd, float("nan"))
    layer.attention(qd, kd, vd, out, shift, kp=kp_dev, vp=vp_dev, route_idx=route_dev)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.basa_attention(q64, k64, v64, geo, kp=kp_or, vp=vp_or, route_idx=route_or)
    PT.assert_outputs_close(PT.to64(out[:, heads]), ref, wl.dtype, f"{wl.name} attention")
    out2 = layer.forward(qd, kd, vd, shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref2 = O.basa_attention(q64, k64, v64, geo)
    g2 = PT.to64(out2[:, heads])
    if geo.routed_k:
        same = (layer.route_idx[:, heads].cpu().numpy() == O.route_windows(q64, k64, geo)[0]).all(axis=-1)
        keep = same[:, :, O.window_of_token(geo)]
        assert keep.mean() > 0.99
        g2 = np.where(keep[..., None], g2, ref2)
    PT.assert_outputs_close(g2, ref2, wl.dtype, f"{wl.name} end to end")
    return geo, q64, k64, v64, kp_or, route_or


def _log2_scores(qrow, keys, d):
    return (keys @ qrow) / math.sqrt(d) * LOG2E


def test_text_staircase_rescales_every_text_tile():
    wl = W("stair", "bf16", 1, 2, 128, (1, 64, 64), (1, 16, 16), (0, 8, 8), (1, 8, 8), 512, 0, "sinusoid")
    q, k, v = synth.make_inputs(wl, seed=3)
    qf, kf = q.float().numpy(), k.float().numpy()
    ch = 5
    qf[:, :, 0::2, ch] = 16.0
    tile = np.arange(wl.n_text) // 128
    kf[:, :, wl.N:, ch] = 5.0 * (tile + 1)
    q, k = _bf16(qf), _bf16(kf)
    geo, q64, k64, _, kp_or, _ = run_attn_parity(wl, q, k, v, [0, 1])
    # even rows: every text tile lifts the max over everything before it by > 8 log2 units
    win = O.window_of_token(geo)
    rng = np.random.default_rng(0)
    rows = rng.choice(np.arange(0, wl.N, 2), size=64, replace=False)
    for h in range(2):
        for i in rows:
            own = k64[0, h, np.nonzero(win == win[i])[0]]
            before = np.concatenate([own, kp_or[0, h]])
            m = _log2_scores(q64[0, h, i], before, wl.d).max()
            for j in range(4):
                t = k64[0, h, wl.N + 128 * j: wl.N + 128 * (j + 1)]
                mt = _log2_scores(q64[0, h, i], t, wl.d).max()
                if j > 0:
                    assert mt > m + THRESH_LOG2, (h, i, j, mt, m)
                m = max(m, mt)


def test_pooled_key_dominates():
    wl = W("pool_dom", "bf16", 1, 2, 128, (1, 64, 64), (1, 16, 16), (0, 8, 0), (1, 8, 8), 0, 0, "sinusoid")
    q, k, v = synth.make_inputs(wl, seed=4)
    qf, kf = q.float().numpy(), k.float().numpy()
    ch = 9
    qf[:, :, :, ch] = 12.0
    # pool patch (3, 5) of the unshifted grid: rows 24..31, columns 40..47
    grid = kf[:, :, : wl.N].reshape(1, 2, 64, 64, wl.d)
    grid[:, :, 24:32, 40:48, ch] = 20.0
    q, k = _bf16(qf), _bf16(kf)
    geo, q64, k64, _, kp_or, _ = run_attn_parity(wl, q, k, v, [0, 1])
    # queries whose window does not contain the patch: the pooled key lifts the max
    win = O.window_of_token(geo)
    patch_tok = (np.arange(24, 32)[:, None] * 64 + np.arange(40, 48)[None, :]).ravel()
    far = np.nonzero(~np.isin(win, np.unique(win[patch_tok])))[0]
    rows = np.random.default_rng(1).choice(far, size=64, replace=False)
    for h in range(2):
        for i in rows:
            own = k64[0, h, np.nonzero(win == win[i])[0]]
            m_own = _log2_scores(q64[0, h, i], own, wl.d).max()
            m_pool = _log2_scores(q64[0, h, i], kp_or[0, h], wl.d).max()
            assert m_pool > m_own + THRESH_LOG2, (h, i, m_pool, m_own)


def test_flux1k_queries_scaled():
    wl = synth.WORKLOADS["flux1k"].with_shift((0, 8, 8))
    q, k, v = synth.make_inputs(wl, seed=0)
    q = _bf16(q.float().numpy() * 6.0)
    run_attn_parity(wl, q, k, v, [0, 12, 23])


def test_wan_routed_windows_far_above_own():
    wl = synth.WORKLOADS["wan"]
    T, H, Wd = wl.grid
    q, k, v = synth.make_inputs(wl, seed=0)
    # the field's per-window means, drawn again from their own streams, added twice more
    mq = synth.block_mean_field(synth.rng_for(0, "mu_q"), wl.heads, T, H, Wd, wl.d, wl.window, wl.shift)[None]
    mk = synth.block_mean_field(synth.rng_for(0, "mu_k"), wl.heads, T, H, Wd, wl.d, wl.window, wl.shift)[None]
    q = _bf16(q.float().numpy() + 2.0 * mq)
    k = _bf16(k.float().numpy() + 2.0 * mk)
    hs = [0, 6, 11]
    geo, q64, k64, _, _, route_or = run_attn_parity(wl, q, k, v, hs)
    win = O.window_of_token(geo)
    rows = np.random.default_rng(2).choice(wl.N, size=128, replace=False)
    lifted = 0
    for j in range(len(hs)):
        for i in rows:
            w = win[i]
            own = k64[0, j, np.nonzero(win == w)[0]]
            routed = k64[0, j, np.nonzero(np.isin(win, route_or[0, j, w]))[0]]
            m_own = _log2_scores(q64[0, j, i], own, wl.d).max()
            m_rt = _log2_scores(q64[0, j, i], routed, wl.d).max()
            lifted += m_rt > m_own + THRESH_LOG2
    assert lifted >= 0.5 * len(hs) * len(rows), lifted

"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: a hand-written fixture, a closed
form, a library routine, an invariant, or an independent brute force.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import basa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _qkv(geo, B=1, h=2, d=8, seed=0, scale=1.0):
    N = geo.N
    q = _rand((B, h, N, d), seed, scale)
    k = _rand((B, h, N + geo.n_text, d), seed + 1, scale)
    v = _rand((B, h, N + geo.n_text, d), seed + 2)
    return q, k, v


def _parse_dims(s):
    return tuple(int(x) for x in s.split("x"))


def _membership_by_partition(geo):
    """Window id of each original token, read off the roll + partition path."""
    idx = np.arange(geo.N, dtype=np.float64).reshape(1, 1, geo.N, 1)
    Xw = O.window_partition(O.cyclic_shift(O.to_grid(idx, geo.grid), geo.shift), geo.window)
    ids = np.empty(geo.N, dtype=np.int64)
    for w in range(geo.n_win):
        ids[Xw[0, 0, w, :, 0].astype(np.int64)] = w
    return ids


# ---------------------------------------------------------------- shift / windows


def test_shift_membership_golden():
    """Hand-derived window membership (tests/golden/shift_membership.txt)."""
    lines = [l for l in open(os.path.join(GOLDEN, "shift_membership.txt")) if l.strip() and not l.startswith("#")]
    assert len(lines) >= 5
    for line in lines:
        lhs, rhs = line.split("|")
        g, w, s = lhs.split()
        geo = O.Geometry(grid=_parse_dims(g), window=_parse_dims(w), shift=tuple(int(x) for x in s.split(",")))
        expect = np.array([int(x) for x in rhs.split()])
        np.testing.assert_array_equal(_membership_by_partition(geo), expect)
        np.testing.assert_array_equal(O.window_of_token(geo), expect)


def test_partition_roundtrip():
    geo = O.Geometry(grid=(4, 6, 10), window=(2, 3, 5), shift=(1, 2, 3))
    x = _rand((2, 3, geo.N, 4), 5)
    X = O.to_grid(x, geo.grid)
    back = O.inverse_cyclic_shift(O.window_unpartition(O.window_partition(O.cyclic_shift(X, geo.shift), geo.window), geo.grid, geo.window), geo.shift)
    np.testing.assert_array_equal(back, X)


# ---------------------------------------------------------------- pooling


def test_pool_of_token_index_is_patch_centre():
    """K[n] = n: the mean of an axis-aligned patch of a raster grid is the index of
    its centre, (t0 + (pt-1)/2) H W + (y0 + (ph-1)/2) W + x0 + (pw-1)/2 (an
    arithmetic series), so any wrong patch membership or order fails."""
    geo = O.Geometry(grid=(4, 6, 8), window=(2, 3, 4), pool=(2, 3, 2))
    T, H, W = geo.grid
    pt, ph, pw = geo.pool
    n = np.arange(geo.N, dtype=np.float64)
    k = np.broadcast_to(n[None, None, :, None], (1, 1, geo.N, 3)).copy()
    kp, vp = O.pool_kv(k, k, geo)
    expect = []
    for t0 in range(0, T, pt):
        for y0 in range(0, H, ph):
            for x0 in range(0, W, pw):
                expect.append((t0 + (pt - 1) / 2) * H * W + (y0 + (ph - 1) / 2) * W + x0 + (pw - 1) / 2)
    np.testing.assert_allclose(kp[0, 0, :, 0], expect, rtol=0, atol=1e-9)
    np.testing.assert_allclose(vp[0, 0, :, 2], expect, rtol=0, atol=1e-9)


def test_pool_constant_field_and_ignores_shift_and_text():
    geo = O.Geometry(grid=(1, 8, 8), window=(1, 4, 4), shift=(0, 3, 1), pool=(1, 2, 4), n_text=5)
    k = np.full((1, 2, geo.N + 5, 4), 0.75)
    k[:, :, geo.N:] = 100.0  # text rows must not enter the pooled tokens
    kp, _ = O.pool_kv(k, k, geo)
    assert kp.shape == (1, 2, 8, 4)
    np.testing.assert_array_equal(kp, 0.75)


# ---------------------------------------------------------------- routing


def _within_radius(geo, w, u):
    """Chebyshev distance of window-grid coordinates, computed from scratch."""
    if geo.route_radius == 0:
        return True
    nWt, nWy, nWx = geo.win_grid
    cw = (w // (nWy * nWx), (w // nWx) % nWy, w % nWx)
    cu = (u // (nWy * nWx), (u // nWx) % nWy, u % nWx)
    return max(abs(a - b) for a, b in zip(cw, cu)) <= geo.route_radius


def _brute_route(q, k, geo):
    """Explicit loops: window member lists by coordinates, means, scores, sort."""
    T, H, W = geo.grid
    wt, wh, ww = geo.window
    st, sy, sx = geo.shift
    nWt, nWy, nWx = geo.win_grid
    B, h, _, d = q.shape
    members = []
    for jt in range(nWt):
        for jy in range(nWy):
            for jx in range(nWx):
                toks = []
                for a in range(wt):
                    for b_ in range(wh):
                        for c in range(ww):
                            t = (jt * wt + a + st) % T
                            y = (jy * wh + b_ + sy) % H
                            x = (jx * ww + c + sx) % W
                            toks.append((t * H + y) * W + x)
                members.append(toks)
    out = np.zeros((B, h, len(members), geo.routed_k), dtype=np.int64)
    for b in range(B):
        for hh in range(h):
            qm = [q[b, hh, m].mean(axis=0) for m in members]
            km = [k[b, hh, m].mean(axis=0) for m in members]
            for w in range(len(members)):
                cands = [(-float(np.dot(qm[w], km[u])), u) for u in range(len(members))
                         if u != w and _within_radius(geo, w, u)]
                cands.sort()
                out[b, hh, w] = [u for _, u in cands[: geo.routed_k]]
    return out


@pytest.mark.parametrize(
    "geo",
    [
        O.Geometry(grid=(1, 8, 12), window=(1, 4, 3), shift=(0, 1, 2), routed_k=3),
        O.Geometry(grid=(4, 4, 6), window=(2, 2, 3), shift=(1, 1, 2), routed_k=2),
        O.Geometry(grid=(1, 12, 15), window=(1, 3, 3), shift=(0, 1, 2), routed_k=3, route_radius=1),
        O.Geometry(grid=(6, 8, 8), window=(2, 2, 2), shift=(1, 1, 1), routed_k=7, route_radius=1),
        O.Geometry(grid=(1, 12, 15), window=(1, 2, 3), shift=(0, 1, 2), routed_k=8, route_radius=2),
    ],
)
def test_route_matches_brute_force(geo):
    q, k, _ = _qkv(geo, B=2, h=2, d=6, seed=11)
    idx, S = O.route_windows(q, k, geo)
    np.testing.assert_array_equal(idx, _brute_route(q, k, geo))


def test_route_planted_winner_and_self_excluded():
    """Window u* gets keys aligned with every query mean: it must win everywhere
    (except for itself, which is never its own candidate)."""
    geo = O.Geometry(grid=(1, 8, 8), window=(1, 4, 4), shift=(0, 2, 2), routed_k=1)
    d = 4
    q = np.zeros((1, 1, geo.N, d))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, geo.N, d))
    win = O.window_of_token(geo)
    star = 2
    k[0, 0, win == star, 0] = 5.0
    k[0, 0, win == 1, 0] = 3.0  # runner-up
    idx, _ = O.route_windows(q, k, geo)
    for w in range(geo.n_win):
        assert idx[0, 0, w, 0] == (1 if w == star else star)


def test_route_ties_go_to_lower_id():
    """All scores equal: the chosen windows are the lowest ids other than w, in order."""
    geo = O.Geometry(grid=(1, 8, 8), window=(1, 2, 2), shift=(0, 1, 1), routed_k=4)
    q = np.ones((1, 1, geo.N, 3))
    k = np.ones((1, 1, geo.N, 3))
    idx, _ = O.route_windows(q, k, geo)
    for w in range(geo.n_win):
        expect = [u for u in range(geo.n_win) if u != w][:4]
        np.testing.assert_array_equal(idx[0, 0, w], expect)


def _planted_id_scores(geo):
    """Q means along e0 everywhere; K mean of window u is u along e0, so the score
    of u against any query window is proportional to u."""
    d = 3
    q = np.zeros((1, 1, geo.N, d))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, geo.N, d))
    k[0, 0, :, 0] = O.window_of_token(geo).astype(np.float64)
    return q, k


@pytest.mark.parametrize(
    "geo",
    [
        O.Geometry(grid=(1, 16, 16), window=(1, 4, 4), shift=(0, 2, 3), routed_k=1, route_radius=1),
        O.Geometry(grid=(6, 6, 9), window=(2, 2, 3), shift=(1, 1, 2), routed_k=1, route_radius=1),
        O.Geometry(grid=(21, 12, 20), window=(21, 3, 4), shift=(0, 1, 2), routed_k=1, route_radius=1),
    ],
)
def test_route_radius_picks_best_neighbour_in_closed_form(geo):
    """With score(w, u) increasing in u, the best radius-one candidate of window
    (jt, jy, jx) is the block's far corner (min(j+1, n-1) on every axis), or, for
    the grid's last window, the window just before it (BASA §A.2: candidate-window
    radius one). Wrap-around or a one-sided block would pick other windows."""
    q, k = _planted_id_scores(geo)
    idx, _ = O.route_windows(q, k, geo)
    nt, ny, nx = geo.win_grid
    for w in range(geo.n_win):
        jt, jy, jx = w // (ny * nx), (w // nx) % ny, w % nx
        best = (min(jt + 1, nt - 1) * ny + min(jy + 1, ny - 1)) * nx + min(jx + 1, nx - 1)
        if best == w:  # last window of the grid: the highest other id in its block
            best = w - 1
        assert idx[0, 0, w, 0] == best, (w, idx[0, 0, w, 0], best)


def test_route_radius_covering_the_grid_equals_global_routing():
    geo = O.Geometry(grid=(4, 8, 12), window=(2, 2, 3), shift=(1, 1, 2), routed_k=5)
    q, k, _ = _qkv(geo, B=1, h=2, d=6, seed=5)
    g0 = O.route_windows(q, k, geo)[0]
    for r in (max(geo.win_grid) - 1, max(geo.win_grid), 50):
        g1 = O.route_windows(q, k, O.Geometry(**{**geo.__dict__, "route_radius": r}))[0]
        np.testing.assert_array_equal(g0, g1)


def test_route_radius_candidates_lie_in_the_block():
    geo = O.Geometry(grid=(1, 20, 24), window=(1, 4, 4), shift=(0, 3, 1), routed_k=3, route_radius=1)
    q, k, _ = _qkv(geo, B=1, h=3, d=8, seed=9)
    idx, S = O.route_windows(q, k, geo)
    for w in range(geo.n_win):
        n_cand = sum(1 for u in range(geo.n_win) if u != w and _within_radius(geo, w, u))
        assert np.isfinite(S[0, 0, w]).sum() == n_cand
        for u in idx[0, :, w].ravel():
            assert _within_radius(geo, w, int(u)) and u != w


def test_full_temporal_windows_ignore_the_temporal_shift():
    """Windows that span all frames hold the same tokens whatever the temporal shift,
    and spatial-only pooling ignores the shift: the output cannot depend on st
    (BASA §3.2 spatial-only pooling and §A.2 full temporal extent, the video setup)."""
    base = O.Geometry(grid=(4, 6, 8), window=(4, 3, 4), shift=(0, 1, 2), pool=(1, 2, 2), routed_k=1, route_radius=1)
    q, k, v = _qkv(base, B=1, h=2, d=8, seed=13)
    ref = O.basa_attention(q, k, v, base)
    for st in (1, 3):
        geo = O.Geometry(**{**base.__dict__, "shift": (st, 1, 2)})
        np.testing.assert_allclose(O.basa_attention(q, k, v, geo), ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- attention


TINY_GEOS = [
    O.Geometry(grid=(1, 8, 8), window=(1, 4, 4), shift=(0, 2, 2), pool=(1, 2, 2), n_text=3, routed_k=2),
    O.Geometry(grid=(4, 4, 6), window=(2, 2, 3), shift=(1, 1, 2), routed_k=2),
    O.Geometry(grid=(2, 6, 4), window=(1, 3, 2), shift=(1, 4, 3), pool=(2, 3, 2), n_text=2, routed_k=1),
    O.Geometry(grid=(1, 6, 6), window=(1, 3, 3), shift=(0, 1, 0), pool=(1, 3, 3)),
]


@pytest.mark.parametrize("geo", TINY_GEOS)
def test_attention_matches_dense_masked_brute_force(geo):
    q, k, v = _qkv(geo, B=2, h=2, d=8, seed=3)
    route = O.route_windows(q, k, geo)[0] if geo.routed_k else None
    a = O.basa_attention(q, k, v, geo, route_idx=route)
    b = O.dense_masked_attention(q, k, v, geo, route_idx=route)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_closed_form_whole_grid_is_dense_sdpa():
    """window = grid, shift 0, no pooling, no text, no routing -> dense attention,
    checked against torch's scaled_dot_product_attention in float64."""
    geo = O.Geometry(grid=(2, 4, 6), window=(2, 4, 6))
    q, k, v = _qkv(geo, B=2, h=3, d=16, seed=7)
    a = O.basa_attention(q, k, v, geo)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(a, ref, rtol=0, atol=1e-12)


def test_closed_form_text_only_keys_are_sdpa_over_concat():
    """window = grid plus text keys -> SDPA over [visual ; text] keys."""
    geo = O.Geometry(grid=(1, 4, 4), window=(1, 4, 4), n_text=5)
    q, k, v = _qkv(geo, B=1, h=2, d=8, seed=9)
    a = O.basa_attention(q, k, v, geo)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(a, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("r", [(0, 2, 4), (1, 6, 2)])
def test_shift_equivariance(r):
    """Rolling the inputs by r and adding r to the shift rolls the output by r.
    r is a multiple of the pool patch, so the pooled set only permutes."""
    geo = O.Geometry(grid=(2, 12, 8), window=(1, 4, 4), shift=(1, 1, 3), pool=(1, 2, 2), n_text=2, routed_k=2)
    q, k, v = _qkv(geo, B=1, h=2, d=8, seed=21)
    out = O.basa_attention(q, k, v, geo)

    def roll(x):
        N = geo.N
        Xg = O.to_grid(x[:, :, :N], geo.grid)
        rolled = np.roll(Xg, shift=r, axis=(2, 3, 4)).reshape(x.shape[0], x.shape[1], N, -1)
        return np.concatenate([rolled, x[:, :, N:]], axis=2)

    geo2 = O.Geometry(grid=geo.grid, window=geo.window, shift=tuple((s + a) % g for s, a, g in zip(geo.shift, r, geo.grid)), pool=geo.pool, n_text=geo.n_text, routed_k=geo.routed_k)
    out2 = O.basa_attention(roll(q), roll(k), roll(v), geo2)
    np.testing.assert_allclose(out2, roll(out), rtol=0, atol=1e-12)
    r1 = O.route_windows(q, k, geo)[0]
    r2 = O.route_windows(roll(q), roll(k), geo2)[0]
    np.testing.assert_array_equal(np.sort(r1, axis=-1), np.sort(r2, axis=-1))


@pytest.mark.parametrize("geo", TINY_GEOS)
def test_softmax_rows_sum_to_one(geo):
    """V = 1 everywhere (pooled V is then 1 too) -> every output is exactly 1."""
    q, k, _ = _qkv(geo, B=1, h=2, d=8, seed=4, scale=3.0)
    v = np.ones_like(k)
    np.testing.assert_allclose(O.basa_attention(q, k, v, geo), 1.0, rtol=0, atol=1e-12)


def _key_set_by_coordinates(geo, route, b, hh, i):
    """Visual keys of query token i, enumerated from coordinates (no oracle helpers)."""
    T, H, W = geo.grid
    wt, wh, ww = geo.window
    st, sy, sx = geo.shift
    nWt, nWy, nWx = geo.win_grid
    t, y, x = i // (H * W), (i // W) % H, i % W
    jt, jy, jx = ((t - st) % T) // wt, ((y - sy) % H) // wh, ((x - sx) % W) // ww
    w = (jt * nWy + jy) * nWx + jx
    wins = [w] + ([int(u) for u in route[b, hh, w]] if geo.routed_k else [])
    keys = []
    for u in wins:
        ut, uy, ux = u // (nWy * nWx), (u // nWx) % nWy, u % nWx
        for a in range(wt):
            for c in range(wh):
                for e in range(ww):
                    keys.append((((ut * wt + a + st) % T) * H + (uy * wh + c + sy) % H) * W + (ux * ww + e + sx) % W)
    return keys


@pytest.mark.parametrize("geo", TINY_GEOS)
def test_constant_scores_give_mean_of_key_values(geo):
    """Q = 0 -> uniform weights -> out_i = mean of V over i's key list
    (own + routed windows, pooled tokens, text tokens), with duplicates counted."""
    _, k, v = _qkv(geo, B=1, h=2, d=5, seed=8)
    q = np.zeros((1, 2, geo.N, 5))
    rng = np.random.default_rng(1)
    route = None
    if geo.routed_k:
        route = np.stack([np.stack([rng.choice([u for u in range(geo.n_win) if u != w], geo.routed_k, replace=False) for w in range(geo.n_win)]) for _ in range(2)])[None].astype(np.int32)
    out = O.basa_attention(q, k, v, geo, route_idx=route)
    T, H, W = geo.grid
    for hh in range(2):
        pooled_rows = []
        if geo.has_pool:
            pt, ph, pw = geo.pool
            for t0 in range(0, T, pt):
                for y0 in range(0, H, ph):
                    for x0 in range(0, W, pw):
                        toks = [((t0 + a) * H + y0 + c) * W + x0 + e for a in range(pt) for c in range(ph) for e in range(pw)]
                        pooled_rows.append(v[0, hh, toks].mean(axis=0))
        for i in range(geo.N):
            rows = [v[0, hh, j] for j in _key_set_by_coordinates(geo, route, 0, hh, i)]
            rows += pooled_rows
            rows += [v[0, hh, geo.N + j] for j in range(geo.n_text)]
            np.testing.assert_allclose(out[0, hh, i], np.mean(rows, axis=0), rtol=0, atol=1e-12)


def test_attention_rows_match_full_oracle():
    geo = TINY_GEOS[0]
    q, k, v = _qkv(geo, B=1, h=2, d=8, seed=12)
    route = O.route_windows(q, k, geo)[0]
    kp, vp = O.pool_kv(k, v, geo)
    full = O.basa_attention(q, k, v, geo, kp=kp, vp=vp, route_idx=route)
    toks = [0, 5, 17, 63]
    rows = O.attention_rows(q, k, v, geo, 0, 1, toks, kp=kp, vp=vp, route_idx=route)
    np.testing.assert_allclose(rows, full[0, 1, toks], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- bf16 rounding


def test_round_to_bf16_matches_torch():
    """The oracle's bf16 rounding equals torch's float32 -> bfloat16 conversion
    (round to nearest, ties to even), including exact ties."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-3, 3, 10000), np.array([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -(1.0 + 2.0**-8), 0.0])]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to_bf16(x), ref)


# ---------------------------------------------------------------- measurement model


def test_flop_model_reproduces_table3():
    """Algorithmic FLOPs 4 d heads N keys reproduce the BASA Table 3 accounting."""
    from sparse_window_attention_b200 import accounting as A

    g = json.load(open(os.path.join(GOLDEN, "table3_wan_efficiency.json")))
    T, H, W = g["latent_grid"]
    N = T * H * W
    nh, d = g["heads"], g["head_dim"]
    win = T * 15 * 26  # full temporal extent, 15x26 spatial window
    pooled = T * (H // 4) * (W // 4)  # spatial-only pooling keeps all frames
    keys = A.keys_per_query(win, 1, pooled, 0)
    rows = g["rows"]
    assert A.sparsity(keys, N) == pytest.approx(rows["basa_w15x26_p4x4"]["sparsity"], abs=1e-12)
    sparse_tf = A.attn_flops(1, nh, N, d, keys) / 1e12
    dense_tf = A.dense_attn_flops(1, nh, N, d, N) / 1e12
    # the printed TFLOPs sit 0.6% above 4 d h N keys for both rows; their ratio matches
    assert sparse_tf / dense_tf == pytest.approx(rows["basa_w15x26_p4x4"]["tflops"] / rows["dense"]["tflops"], rel=2e-3)
    assert sparse_tf == pytest.approx(rows["basa_w15x26_p4x4"]["tflops"], rel=1e-2)
    assert dense_tf == pytest.approx(rows["dense"]["tflops"], rel=1e-2)
    # the same count from the video workload's own shape (synth table)
    from sparse_window_attention_b200 import synth
    c = A.workload_counts(synth.WORKLOADS["wan_video"])
    assert c["keys_per_query"] == keys == 24570 and c["N"] == N
    assert A.sparsity(c["keys_per_query"], c["N"]) == pytest.approx(rows["basa_w15x26_p4x4"]["sparsity"], abs=1e-12)
    for r in rows.values():  # MFU = TFLOPs / latency / 312 TFLOP/s
        assert r["tflops"] / (r["latency_ms"] * 1e-3) / 312.0 == pytest.approx(r["mfu"], abs=6e-5)


# ---------------------------------------------------------------- branch form (LSE)


@pytest.mark.parametrize("geo", TINY_GEOS)
def test_branches_merge_to_the_joint_softmax(geo):
    """BASA §A.1: local and text/global branches evaluated separately equal one
    softmax over the concatenated keys; two-way and three-way splits."""
    q, k, v = _qkv(geo, B=1, h=2, d=8, seed=21)
    route = O.route_windows(q, k, geo)[0] if geo.routed_k else None
    joint = O.basa_attention(q, k, v, geo, route_idx=route)
    out_all, lse_all = O.branch_attention(q, k, v, geo, O.KEYS_ALL, route_idx=route)
    np.testing.assert_allclose(out_all, joint, rtol=0, atol=1e-12)
    glob = (O.KEYS_POOLED if geo.has_pool else 0) | (O.KEYS_TEXT if geo.n_text else 0)
    if not glob:
        return
    splits = [[O.KEYS_WINDOWS, glob]]
    if geo.has_pool and geo.n_text:
        splits.append([O.KEYS_WINDOWS, O.KEYS_POOLED, O.KEYS_TEXT])
    for parts in splits:
        res = [O.branch_attention(q, k, v, geo, keys, route_idx=route) for keys in parts]
        out, lse = O.merge_branches([r[0] for r in res], [r[1] for r in res])
        np.testing.assert_allclose(out, joint, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_all, rtol=0, atol=1e-12)


def test_lse_of_zero_queries_is_log_of_key_count():
    """q = 0: every score is 0, so lse = log(number of keys) exactly."""
    geo = TINY_GEOS[0]
    q, k, v = _qkv(geo, B=1, h=1, d=8, seed=2)
    q[:] = 0.0
    route = O.route_windows(q, k, geo)[0]
    n_keys = geo.win_tokens * (1 + geo.routed_k) + geo.n_pool + geo.n_text
    _, lse = O.branch_attention(q, k, v, geo, O.KEYS_ALL, route_idx=route)
    np.testing.assert_allclose(lse, np.log(n_keys), rtol=0, atol=1e-12)
    _, lse_w = O.branch_attention(q, k, v, geo, O.KEYS_WINDOWS, route_idx=route)
    np.testing.assert_allclose(lse_w, np.log(geo.win_tokens * (1 + geo.routed_k)), rtol=0, atol=1e-12)


def test_lse_whole_grid_is_scipy_logsumexp():
    """window = grid, shift 0, nothing else: lse_i = logsumexp_j(q_i . k_j / sqrt(d))."""
    from scipy.special import logsumexp

    geo = O.Geometry(grid=(2, 4, 6), window=(2, 4, 6))
    q, k, v = _qkv(geo, B=1, h=2, d=16, seed=17)
    q *= 3.0  # spread the scores so the max term matters
    _, lse = O.branch_attention(q, k, v, geo, O.KEYS_ALL)
    for hh in range(2):
        ref = logsumexp(q[0, hh] @ k[0, hh].T / 4.0, axis=1)
        np.testing.assert_allclose(lse[0, hh], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- text-query rows


def test_text_queries_dense_sdpa():
    """Text queries attend to every visual and text key: torch SDPA in float64
    over the concatenated rows."""
    geo = O.Geometry(grid=(2, 4, 6), window=(1, 2, 3), shift=(1, 1, 2), pool=(1, 2, 3), n_text=5, routed_k=1)
    rng = np.random.default_rng(31)
    qt = rng.standard_normal((2, 3, 5, 16))
    k = rng.standard_normal((2, 3, geo.N + 5, 16))
    v = rng.standard_normal((2, 3, geo.N + 5, 16))
    out = O.text_query_attention(qt, k, v, geo)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(qt), torch.from_numpy(k),
                                                           torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_text_queries_zero_query_is_mean_of_all_values():
    geo = O.Geometry(grid=(1, 4, 4), window=(1, 2, 2), n_text=3)
    rng = np.random.default_rng(5)
    k = rng.standard_normal((1, 2, geo.N + 3, 8))
    v = rng.standard_normal((1, 2, geo.N + 3, 8))
    out = O.text_query_attention(np.zeros((1, 2, 3, 8)), k, v, geo)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=2, keepdims=True), out.shape), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- backward


BWD_GEOS = [
    O.Geometry(grid=(1, 8, 8), window=(1, 4, 4), shift=(0, 2, 2), pool=(1, 2, 2), n_text=3, routed_k=2),
    O.Geometry(grid=(4, 4, 6), window=(2, 2, 3), shift=(1, 1, 2), pool=(2, 2, 3), routed_k=1),
]


@pytest.mark.parametrize("geo", BWD_GEOS)
def test_backward_matches_finite_differences(geo):
    """Central differences of L = sum(dout * out) w.r.t. sampled entries of q, k, v
    (routing held fixed, pooling recomputed from k and v)."""
    q, k, v = _qkv(geo, B=1, h=1, d=4, seed=41)
    rng = np.random.default_rng(3)
    dout = rng.standard_normal(q.shape)
    route = O.route_windows(q, k, geo)[0] if geo.routed_k else None
    dq, dk, dv = O.basa_attention_backward(q, k, v, geo, dout, route_idx=route)

    def loss(qq, kk, vv):
        return float((dout * O.basa_attention(qq, kk, vv, geo, route_idx=route)).sum())

    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [tuple(rng.integers(0, s) for s in x.shape) for _ in range(12)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            lp = loss(*[xp if a is x else a for a in args])
            lm = loss(*[xm if a is x else a for a in args])
            num = (lp - lm) / (2 * eps)
            assert abs(num - g[idx]) <= 1e-7 + 1e-6 * abs(num), (name, idx, num, g[idx])


def test_backward_whole_grid_is_sdpa_autograd():
    """window = grid, shift 0, with text keys: float64 autograd through torch SDPA."""
    geo = O.Geometry(grid=(2, 4, 6), window=(2, 4, 6), n_text=4)
    q, k, v = _qkv(geo, B=1, h=2, d=8, seed=43)
    dout = np.random.default_rng(9).standard_normal(q.shape)
    dq, dk, dv = O.basa_attention_backward(q, k, v, geo, dout)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(torch.from_numpy(dout))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)

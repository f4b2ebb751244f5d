"""CPU oracle for the BASA forward hot path (float64, numpy).

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
CUDA library never calls it, and it shares no code with the CUDA library.

It states the operator the way the pages describe it, step by step, with no
blocking, fusion or reordering beyond what the definition needs:

  BASA = "Backend-Agnostic Sparse Attention for Fast High-Resolution Visual
  Generation" (arXiv 2610.08772); sections below are that paper's.

1. cyclic shift of the token grid (BASA §A.1: cyclic shift, reshape and
   permutation form non-overlapping windows folded into the batch);
2. non-overlapping windows of the shifted grid (BASA §3.1, §A.1);
3. average-pooled global K/V over patches of the unshifted grid (BASA §3.2
   "K/V-pooled global memory"; §A.1 "regular spatial reduction");
4. content-adaptive routing: each query window adds the K/V of the windows whose
   mean-pooled keys score highest against its mean-pooled query (BASA §3.3
   "content-adaptive true-window routing");
5. one softmax, scale 1/sqrt(d), over the concatenation own window | routed
   windows | pooled tokens | text tokens (BASA §A.1: the local and text/global
   branches are equivalent to one softmax over concatenated K/V);
6. inverse shift of the output.

The branch form (branch_attention, merge_branches) evaluates key groups separately
with their log-sum-exp and merges them (BASA §A.1). text_query_attention gives the
text queries' rows (dense over every key), and basa_attention_backward the
gradients of basa_attention with respect to q, k and v (routing held fixed).

Readings taken where the pages are silent:
  * shift convention Xr[t,y,x] = X[(t+st)%T, (y+sy)%H, (x+sx)%W] (roll by -s);
  * window ids are raster order over the window grid of the shifted frame;
  * routing score = dot product of float64 window means of Q and K, the window
    itself excluded, candidates = all other windows or, with a radius r, the
    windows within Chebyshev distance r on the window grid (no wrap-around),
    ties to the lower id, the chosen ids listed by descending score;
  * text tokens are keys only (rows N.. of k and v); only visual queries are output;
  * pooled tokens are listed in raster order of the pooled grid.

Layouts: q, out [B, h, N, d]; k, v [B, h, N + n_text, d] (visual rows in raster
(t, y, x) order, then text rows); kp, vp [B, h, Np, d]; route_idx [B, h, nWin, k].
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Geometry:
    """The arguments that fix the operator (besides the tensors themselves)."""

    grid: tuple  # (T, H, W)
    window: tuple  # (wt, wh, ww)
    shift: tuple = (0, 0, 0)  # (st, sy, sx)
    pool: tuple = (0, 0, 0)  # (pt, ph, pw); all zero = no pooled keys
    n_text: int = 0
    routed_k: int = 0
    route_radius: int = 0  # 0 = every other window is a routing candidate

    @property
    def N(self):
        T, H, W = self.grid
        return T * H * W

    @property
    def win_grid(self):
        return tuple(g // w for g, w in zip(self.grid, self.window))

    @property
    def n_win(self):
        a, b, c = self.win_grid
        return a * b * c

    @property
    def win_tokens(self):
        a, b, c = self.window
        return a * b * c

    @property
    def has_pool(self):
        return all(p > 0 for p in self.pool)

    @property
    def n_pool(self):
        if not self.has_pool:
            return 0
        return int(np.prod([g // p for g, p in zip(self.grid, self.pool)]))


def to_grid(x, grid):
    """[B, h, N, d] -> [B, h, T, H, W, d] (raster order t, y, x)."""
    B, h, N, d = x.shape
    return x.reshape(B, h, *grid, d)


def cyclic_shift(X, shift):
    """Xr[t, y, x] = X[(t+st)%T, (y+sy)%H, (x+sx)%W]  (BASA §A.1 cyclic shift)."""
    return np.roll(X, shift=tuple(-s for s in shift), axis=(2, 3, 4))


def inverse_cyclic_shift(Xr, shift):
    """Inverse of cyclic_shift: X[(t+st)%T, ...] = Xr[t, ...]."""
    return np.roll(Xr, shift=tuple(shift), axis=(2, 3, 4))


def window_partition(Xr, window):
    """[B,h,T,H,W,d] -> [B,h,nWin,wt*wh*ww,d]; windows in raster order (BASA §A.1)."""
    B, h, T, H, W, d = Xr.shape
    wt, wh, ww = window
    x = Xr.reshape(B, h, T // wt, wt, H // wh, wh, W // ww, ww, d)
    x = x.transpose(0, 1, 2, 4, 6, 3, 5, 7, 8)
    return x.reshape(B, h, (T // wt) * (H // wh) * (W // ww), wt * wh * ww, d)


def window_unpartition(Xw, grid, window):
    """Inverse of window_partition."""
    B, h, nw, wtok, d = Xw.shape
    T, H, W = grid
    wt, wh, ww = window
    x = Xw.reshape(B, h, T // wt, H // wh, W // ww, wt, wh, ww, d)
    x = x.transpose(0, 1, 2, 5, 3, 6, 4, 7, 8)
    return x.reshape(B, h, T, H, W, d)


def pool_kv(k, v, geo: Geometry):
    """Average of K and of V over each pt x ph x pw patch of the UNSHIFTED grid.

    BASA §3.2 (K/V-pooled global memory: spatially pooled K/V gives every window a
    cheap global context) and §A.1 (pooling is a regular spatial reduction). The
    pooled tokens are in raster order of the pooled grid. Returns float64
    [B, h, Np, d] twice.
    """
    T, H, W = geo.grid
    pt, ph, pw = geo.pool
    N = geo.N
    res = []
    for x in (k, v):
        X = to_grid(np.asarray(x[:, :, :N], dtype=np.float64), geo.grid)
        B, h, d = X.shape[0], X.shape[1], X.shape[-1]
        P = X.reshape(B, h, T // pt, pt, H // ph, ph, W // pw, pw, d).mean(axis=(3, 5, 7))
        res.append(P.reshape(B, h, -1, d))
    return res[0], res[1]


def window_means(q, k, geo: Geometry):
    """Mean over each shifted window of Q and of K: float64 [B, h, nWin, d] each."""
    N = geo.N
    out = []
    for x in (q, k):
        X = to_grid(np.asarray(x[:, :, :N], dtype=np.float64), geo.grid)
        Xw = window_partition(cyclic_shift(X, geo.shift), geo.window)
        out.append(Xw.mean(axis=3))
    return out[0], out[1]


def window_coords(geo: Geometry, w: int):
    """Window-grid coordinates (jt, jy, jx) of window id w (raster order)."""
    nt, ny, nx = geo.win_grid
    return w // (ny * nx), (w // nx) % ny, w % nx


def candidate_windows(geo: Geometry, w: int):
    """Windows that may be routed to query window w, in increasing id order.

    Every other window when geo.route_radius == 0. With a radius r >= 1, the other
    windows of the (2r+1)^3 block of the window grid centred on w, clipped at the
    grid's edges (BASA §A.2: candidate-window radius one in the video configuration;
    the distance is read as Chebyshev distance between window-grid coordinates,
    without wrap-around).
    """
    r = geo.route_radius
    nt, ny, nx = geo.win_grid
    if r == 0:
        return [u for u in range(geo.n_win) if u != w]
    jt, jy, jx = window_coords(geo, w)
    out = []
    for ut in range(max(0, jt - r), min(nt, jt + r + 1)):
        for uy in range(max(0, jy - r), min(ny, jy + r + 1)):
            for ux in range(max(0, jx - r), min(nx, jx + r + 1)):
                u = (ut * ny + uy) * nx + ux
                if u != w:
                    out.append(u)
    return out


def route_windows(q, k, geo: Geometry):
    """Top-k routed windows per query window (BASA §3.3, content-adaptive routing).

    score[w, u] = mean(Q over window w) . mean(K over window u) for the candidates u
    of w (candidate_windows). The k candidates with the largest scores are kept,
    ties going to the lower window id, listed by descending score. Returns
    (route_idx int32 [B,h,nWin,k], scores float64 [B,h,nWin,nWin] with every
    non-candidate entry, the diagonal included, set to -inf).
    """
    Qm, Km = window_means(q, k, geo)
    S = np.einsum("bhwd,bhud->bhwu", Qm, Km)
    nw = geo.n_win
    B, h = S.shape[:2]
    idx = np.zeros((B, h, nw, geo.routed_k), dtype=np.int32)
    for w in range(nw):
        cand = np.array(candidate_windows(geo, w), dtype=np.int64)
        keep = np.zeros(nw, dtype=bool)
        keep[cand] = True
        S[:, :, w, ~keep] = -np.inf
        for b in range(B):
            for hh in range(h):
                sc = S[b, hh, w, cand]
                order = np.lexsort((cand, -sc))  # primary: score descending, then id ascending
                idx[b, hh, w] = cand[order[: geo.routed_k]]
    return idx, S


def round_to_bf16(x):
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    Used to hand the oracle's pooled K/V to a bfloat16 kernel; done through float32
    (exact for the float32 path) with the bit arithmetic written out.
    """
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def basa_attention(q, k, v, geo: Geometry, kp=None, vp=None, route_idx=None, return_keys=False):
    """BASA forward: out [B, h, N, d] float64.

    For each query i of shifted window w: out_i = softmax_j(q_i . k_j / sqrt(d)) v_j
    over the keys [own window | routed windows (route order) | pooled | text]
    (BASA §3.1-§3.3, §A.1), then the output is shifted back to the original grid.
    ``kp``/``vp`` default to pool_kv(); ``route_idx`` defaults to route_windows().
    """
    q64 = np.asarray(q, dtype=np.float64)
    k64 = np.asarray(k, dtype=np.float64)
    v64 = np.asarray(v, dtype=np.float64)
    B, h, N, d = q64.shape
    assert N == geo.N
    if geo.has_pool and kp is None:
        kp, vp = pool_kv(k64, v64, geo)
    if geo.routed_k > 0 and route_idx is None:
        route_idx, _ = route_windows(q64, k64, geo)

    def windows(x):
        return window_partition(cyclic_shift(to_grid(x[:, :, :N], geo.grid), geo.shift), geo.window)

    Qw, Kw, Vw = windows(q64), windows(k64), windows(v64)
    Ow = np.empty_like(Qw)
    scale = 1.0 / np.sqrt(d)
    for b in range(B):
        for hh in range(h):
            for w in range(geo.n_win):
                kparts, vparts = [Kw[b, hh, w]], [Vw[b, hh, w]]
                for r in range(geo.routed_k):
                    u = int(route_idx[b, hh, w, r])
                    kparts.append(Kw[b, hh, u])
                    vparts.append(Vw[b, hh, u])
                if geo.has_pool:
                    kparts.append(np.asarray(kp[b, hh], dtype=np.float64))
                    vparts.append(np.asarray(vp[b, hh], dtype=np.float64))
                if geo.n_text > 0:
                    kparts.append(k64[b, hh, N:])
                    vparts.append(v64[b, hh, N:])
                Kc = np.concatenate(kparts, axis=0)
                Vc = np.concatenate(vparts, axis=0)
                s = (Qw[b, hh, w] @ Kc.T) * scale
                s = s - s.max(axis=1, keepdims=True)
                p = np.exp(s)
                p = p / p.sum(axis=1, keepdims=True)
                Ow[b, hh, w] = p @ Vc
    O = inverse_cyclic_shift(window_unpartition(Ow, geo.grid, geo.window), geo.shift)
    return O.reshape(B, h, N, d)


# Key groups of the branch form (BASA §A.1: the local-window and text/global-memory
# branches can be evaluated separately; the result equals one softmax over all keys).
KEYS_WINDOWS = 1  # own window and routed windows
KEYS_POOLED = 2
KEYS_TEXT = 4
KEYS_ALL = KEYS_WINDOWS | KEYS_POOLED | KEYS_TEXT


def branch_attention(q, k, v, geo: Geometry, keys, kp=None, vp=None, route_idx=None):
    """One branch of the decomposed form: attention of every query over the key
    groups in ``keys`` only, and the log-sum-exp of its scaled scores.

    out_i = sum_j softmax_j(s_ij) v_j and lse_i = log sum_j exp(s_ij), with
    s_ij = q_i . k_j / sqrt(d) over the selected groups (BASA §A.1). Returns
    (out [B, h, N, d], lse [B, h, N]) float64, both at original token positions.
    """
    q64 = np.asarray(q, dtype=np.float64)
    k64 = np.asarray(k, dtype=np.float64)
    v64 = np.asarray(v, dtype=np.float64)
    B, h, N, d = q64.shape
    if geo.has_pool and kp is None:
        kp, vp = pool_kv(k64, v64, geo)
    if geo.routed_k > 0 and route_idx is None:
        route_idx, _ = route_windows(q64, k64, geo)

    def windows(x):
        return window_partition(cyclic_shift(to_grid(x[:, :, :N], geo.grid), geo.shift), geo.window)

    Qw, Kw, Vw = windows(q64), windows(k64), windows(v64)
    Ow = np.empty_like(Qw)
    Lw = np.empty(Qw.shape[:-1])
    scale = 1.0 / np.sqrt(d)
    for b in range(B):
        for hh in range(h):
            for w in range(geo.n_win):
                kparts, vparts = [], []
                if keys & KEYS_WINDOWS:
                    for u in [w] + [int(route_idx[b, hh, w, r]) for r in range(geo.routed_k)]:
                        kparts.append(Kw[b, hh, u])
                        vparts.append(Vw[b, hh, u])
                if keys & KEYS_POOLED and geo.has_pool:
                    kparts.append(np.asarray(kp[b, hh], dtype=np.float64))
                    vparts.append(np.asarray(vp[b, hh], dtype=np.float64))
                if keys & KEYS_TEXT and geo.n_text > 0:
                    kparts.append(k64[b, hh, N:])
                    vparts.append(v64[b, hh, N:])
                Kc = np.concatenate(kparts, axis=0)
                Vc = np.concatenate(vparts, axis=0)
                s = (Qw[b, hh, w] @ Kc.T) * scale
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=1, keepdims=True)
                Ow[b, hh, w] = (e / l) @ Vc
                Lw[b, hh, w] = (m + np.log(l))[:, 0]
    O = inverse_cyclic_shift(window_unpartition(Ow, geo.grid, geo.window), geo.shift)
    L = inverse_cyclic_shift(window_unpartition(Lw[..., None], geo.grid, geo.window), geo.shift)
    return O.reshape(B, h, N, d), L.reshape(B, h, N)


def merge_branches(outs, lses):
    """Merge branch results into the joint softmax (BASA §A.1): with L = log sum_b
    exp(lse_b), out = sum_b exp(lse_b - L) out_b. Returns (out, L)."""
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])
    m = L.max(axis=0)
    wts = np.exp(L - m)
    tot = wts.sum(axis=0)
    out = sum(wts[i][..., None] * np.asarray(outs[i], dtype=np.float64) for i in range(len(outs))) / tot[..., None]
    return out, m + np.log(tot)


def text_query_attention(q_text, k, v, geo: Geometry):
    """Output rows of the text queries: dense attention over every key.

    The pages sparsify the image queries' keys only; a text query keeps the dense
    model's joint attention over all N visual keys and the n_text text keys (the
    text/global-memory branch of BASA §A.1 seen from the text side). out[i] =
    sum_j softmax_j(q_i . k_j / sqrt(d)) v_j over the N + n_text rows of k, v.
    q_text [B, h, n_text, d] -> [B, h, n_text, d] float64.
    """
    qt = np.asarray(q_text, dtype=np.float64)
    k64 = np.asarray(k, dtype=np.float64)
    v64 = np.asarray(v, dtype=np.float64)
    B, h, nt, d = qt.shape
    assert k64.shape[2] == geo.N + geo.n_text and nt == geo.n_text
    out = np.empty_like(qt)
    for b in range(B):
        for hh in range(h):
            s = (qt[b, hh] @ k64[b, hh].T) / np.sqrt(d)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            out[b, hh] = (p / p.sum(axis=1, keepdims=True)) @ v64[b, hh]
    return out


def basa_attention_backward(q, k, v, geo: Geometry, dout, route_idx=None):
    """Gradients of the BASA forward w.r.t. q, k and v for an output gradient dout.

    Differentiates basa_attention step by step (routing is a selection and is held
    fixed at route_idx; the pooled K/V are means of k, v and pass their gradient
    back to every token of the patch). Per query block of window w, with keys
    Kc = [own | routed | pooled | text] and P = softmax(Q Kc^T / sqrt(d)):
      dVc = P^T dO,  dP = dO Vc^T,  dS = P * (dP - rowsum(dP * P)),
      dQ = dS Kc / sqrt(d),  dKc = dS^T Q / sqrt(d);
    the rows of dKc, dVc are then added back to the tokens they came from.
    Returns (dq [B,h,N,d], dk, dv [B,h,N+n_text,d]) float64.
    """
    q64 = np.asarray(q, dtype=np.float64)
    k64 = np.asarray(k, dtype=np.float64)
    v64 = np.asarray(v, dtype=np.float64)
    do64 = np.asarray(dout, dtype=np.float64)
    B, h, N, d = q64.shape
    if geo.routed_k > 0 and route_idx is None:
        route_idx, _ = route_windows(q64, k64, geo)
    kp = vp = None
    if geo.has_pool:
        kp, vp = pool_kv(k64, v64, geo)

    def windows(x):
        return window_partition(cyclic_shift(to_grid(x[:, :, :N], geo.grid), geo.shift), geo.window)

    Qw, Kw, Vw, dOw = windows(q64), windows(k64), windows(v64), windows(do64)
    dQw = np.zeros_like(Qw)
    dKw = np.zeros_like(Kw)
    dVw = np.zeros_like(Vw)
    dkp = np.zeros((B, h, geo.n_pool, d))
    dvp = np.zeros((B, h, geo.n_pool, d))
    dk_text = np.zeros((B, h, geo.n_text, d))
    dv_text = np.zeros((B, h, geo.n_text, d))
    scale = 1.0 / np.sqrt(d)
    wt = geo.win_tokens
    for b in range(B):
        for hh in range(h):
            for w in range(geo.n_win):
                wins = [w] + [int(route_idx[b, hh, w, r]) for r in range(geo.routed_k)]
                kparts = [Kw[b, hh, u] for u in wins]
                vparts = [Vw[b, hh, u] for u in wins]
                if geo.has_pool:
                    kparts.append(kp[b, hh])
                    vparts.append(vp[b, hh])
                if geo.n_text > 0:
                    kparts.append(k64[b, hh, N:])
                    vparts.append(v64[b, hh, N:])
                Kc = np.concatenate(kparts, axis=0)
                Vc = np.concatenate(vparts, axis=0)
                Qb, dOb = Qw[b, hh, w], dOw[b, hh, w]
                s = (Qb @ Kc.T) * scale
                s = s - s.max(axis=1, keepdims=True)
                P = np.exp(s)
                P = P / P.sum(axis=1, keepdims=True)
                dVc = P.T @ dOb
                dP = dOb @ Vc.T
                dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
                dQw[b, hh, w] = (dS @ Kc) * scale
                dKc = (dS.T @ Qb) * scale
                for i, u in enumerate(wins):
                    dKw[b, hh, u] += dKc[i * wt:(i + 1) * wt]
                    dVw[b, hh, u] += dVc[i * wt:(i + 1) * wt]
                off = len(wins) * wt
                if geo.has_pool:
                    dkp[b, hh] += dKc[off:off + geo.n_pool]
                    dvp[b, hh] += dVc[off:off + geo.n_pool]
                    off += geo.n_pool
                if geo.n_text > 0:
                    dk_text[b, hh] += dKc[off:]
                    dv_text[b, hh] += dVc[off:]

    def unwindows(xw):
        X = inverse_cyclic_shift(window_unpartition(xw, geo.grid, geo.window), geo.shift)
        return X.reshape(B, h, N, d)

    dq = unwindows(dQw)
    dk_vis, dv_vis = unwindows(dKw), unwindows(dVw)
    if geo.has_pool:
        # kp = mean over the patch: each token of patch P receives dkp[P] / |P|
        T, H, W = geo.grid
        pt, ph, pw = geo.pool
        for g_vis, g_pool in ((dk_vis, dkp), (dv_vis, dvp)):
            G = g_pool.reshape(B, h, T // pt, H // ph, W // pw, d) / (pt * ph * pw)
            G = np.repeat(np.repeat(np.repeat(G, pt, axis=2), ph, axis=3), pw, axis=4)
            g_vis += G.reshape(B, h, N, d)
    dk = np.concatenate([dk_vis, dk_text], axis=2)
    dv = np.concatenate([dv_vis, dv_text], axis=2)
    return dq, dk, dv


def window_of_token(geo: Geometry):
    """Window id of every token of the ORIGINAL grid, computed without any roll.

    A token at original coordinate c (per axis) sits at shifted coordinate
    (c - s) mod G, hence in window ((c - s) mod G) // w along that axis.
    """
    T, H, W = geo.grid
    wt, wh, ww = geo.window
    st, sy, sx = geo.shift
    nWt, nWy, nWx = geo.win_grid
    t = ((np.arange(T) - st) % T) // wt
    y = ((np.arange(H) - sy) % H) // wh
    x = ((np.arange(W) - sx) % W) // ww
    return ((t[:, None, None] * nWy + y[None, :, None]) * nWx + x[None, None, :]).reshape(-1)


def dense_masked_attention(q, k, v, geo: Geometry, route_idx=None, kp=None, vp=None):
    """Independent formulation: dense attention in the original frame with a key mask.

    Keys are [all N visual tokens | pooled | text]; query i may see visual key j
    iff win(j) == win(i) or win(j) is one of win(i)'s routed windows; pooled and
    text keys are always visible. No roll, no window gather.
    """
    q64 = np.asarray(q, dtype=np.float64)
    k64 = np.asarray(k, dtype=np.float64)
    v64 = np.asarray(v, dtype=np.float64)
    B, h, N, d = q64.shape
    win = window_of_token(geo)
    if geo.has_pool and kp is None:
        kp, vp = pool_kv(k64, v64, geo)
    out = np.empty_like(q64)
    for b in range(B):
        for hh in range(h):
            allowed = win[:, None] == win[None, :]
            if geo.routed_k > 0:
                routed = np.zeros((geo.n_win, geo.n_win), dtype=bool)
                for w in range(geo.n_win):
                    routed[w, route_idx[b, hh, w]] = True
                allowed = allowed | routed[win[:, None], win[None, :]]
            keys = [k64[b, hh, :N]]
            vals = [v64[b, hh, :N]]
            extra = 0
            if geo.has_pool:
                keys.append(np.asarray(kp[b, hh], dtype=np.float64))
                vals.append(np.asarray(vp[b, hh], dtype=np.float64))
                extra += kp.shape[2]
            if geo.n_text > 0:
                keys.append(k64[b, hh, N:])
                vals.append(v64[b, hh, N:])
                extra += geo.n_text
            mask = np.concatenate([allowed, np.ones((N, extra), dtype=bool)], axis=1)
            Kc = np.concatenate(keys, axis=0)
            Vc = np.concatenate(vals, axis=0)
            s = (q64[b, hh] @ Kc.T) / np.sqrt(d)
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            out[b, hh] = p @ Vc
    return out


def attention_rows(q, k, v, geo: Geometry, b, hh, tokens, kp=None, vp=None, route_idx=None):
    """Output rows for a sample of ORIGINAL token indices of one (b, head), float64.

    Used to check large problems on a sample; it applies the same definition as
    basa_attention to just the listed queries, finding each query's window by
    window_of_token().
    """
    N = geo.N
    d = q.shape[-1]
    win = window_of_token(geo)
    k64 = np.asarray(k[b, hh], dtype=np.float64)
    v64 = np.asarray(v[b, hh], dtype=np.float64)
    q64 = np.asarray(q[b, hh], dtype=np.float64)
    members = {}
    res = np.empty((len(tokens), d))
    for n, i in enumerate(tokens):
        w = int(win[i])
        wins = [w] + ([int(u) for u in route_idx[b, hh, w]] if geo.routed_k > 0 else [])
        rows = []
        for u in wins:
            if u not in members:
                members[u] = np.nonzero(win == u)[0]
            rows.append(members[u])
        kparts = [k64[np.concatenate(rows)]]
        vparts = [v64[np.concatenate(rows)]]
        if geo.has_pool:
            kparts.append(np.asarray(kp[b, hh], dtype=np.float64))
            vparts.append(np.asarray(vp[b, hh], dtype=np.float64))
        if geo.n_text > 0:
            kparts.append(k64[N:])
            vparts.append(v64[N:])
        Kc = np.concatenate(kparts)
        Vc = np.concatenate(vparts)
        s = (Kc @ q64[i]) / np.sqrt(d)
        p = np.exp(s - s.max())
        res[n] = (p / p.sum()) @ Vc
    return res

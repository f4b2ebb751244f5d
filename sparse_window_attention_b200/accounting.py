"""Algorithmic work of one BASA layer call: FLOPs and compulsory bytes.

FLOPs follow the attention accounting of the BASA paper's Table 3 (Wan attention
efficiency: attention TFLOPs = 4 * d * heads * N * keys-per-query, i.e. 2 d for
Q K^T and 2 d for P V per query-key pair; softmax, padding and projections are
not counted). Bytes are the compulsory HBM traffic of each kernel: every input
read once and every output written once.
"""
from __future__ import annotations


def keys_per_query(win_tokens: int, routed_k: int, n_pool: int, n_text: int) -> int:
    return win_tokens * (1 + routed_k) + n_pool + n_text


def attn_flops(B: int, heads: int, N: int, d: int, keys: int) -> float:
    return 4.0 * d * B * heads * N * keys


def dense_attn_flops(B: int, heads: int, N: int, d: int, n_keys_total: int) -> float:
    return 4.0 * d * B * heads * N * n_keys_total


def sparsity(keys: int, n_keys_total: int) -> float:
    return 1.0 - keys / n_keys_total


def workload_counts(wl) -> dict:
    """Per-call counts for a synth.Workload."""
    T, H, W = wl.grid
    wt, wh, ww = wl.window
    N = T * H * W
    win_tokens = wt * wh * ww
    n_win = N // win_tokens
    if all(p > 0 for p in wl.pool):
        pt, ph, pw = wl.pool
        n_pool = (T // pt) * (H // ph) * (W // pw)
    else:
        n_pool = 0
    esz = 2 if wl.dtype == "bf16" else 4
    keys = keys_per_query(win_tokens, wl.routed_k, n_pool, wl.n_text)
    row = wl.d * esz
    bh = wl.B * wl.heads
    return {
        "N": N,
        "win_tokens": win_tokens,
        "n_win": n_win,
        "n_pool": n_pool,
        "keys_per_query": keys,
        "attn_flops": attn_flops(wl.B, wl.heads, N, wl.d, keys),
        # pool: read visual K and V, write Kp and Vp
        "pool_bytes": bh * (2 * N * row + 2 * n_pool * row) if n_pool else 0,
        # route: read visual Q and K (the window means and scores are negligible)
        "route_bytes": bh * 2 * N * row if wl.routed_k > 0 else 0,
        # fused pool + routing pass: read visual Q, K, V once, write Kp and Vp
        "pool_route_bytes": bh * (3 * N * row + 2 * n_pool * row) if (n_pool and wl.routed_k > 0) else 0,
        # attention: read Q, K, V (visual + text), Kp, Vp; write O
        "attn_bytes": bh * row * (N + 2 * (N + wl.n_text) + 2 * n_pool + N),
    }

"""Planted mistakes in a copy of the oracle must be caught by the pins.

Each case edits the oracle's source text (a wrong sign, a dropped term, a wrong
axis, a transposed order), builds a throw-away module from it, points the pin
tests at that module and expects at least one of them to fail. The real oracle
is never modified.
"""
import inspect
import sys
import types

import pytest

from oracle import basa_oracle
from tests import test_oracle as pins

MUTATIONS = [
    # (name, old text, new text, pins that must catch it)
    ("shift sign", "np.roll(X, shift=tuple(-s for s in shift)", "np.roll(X, shift=tuple(s for s in shift)", ["shift_membership"]),
    ("window order", "x.transpose(0, 1, 2, 4, 6, 3, 5, 7, 8)", "x.transpose(0, 1, 6, 4, 2, 3, 5, 7, 8)", ["shift_membership"]),
    ("mask sign", "t = ((np.arange(T) - st) % T) // wt", "t = ((np.arange(T) + st) % T) // wt", ["shift_membership"]),
    ("pool patch stride", "X.reshape(B, h, T // pt, pt, H // ph, ph, W // pw, pw, d)", "X.reshape(B, h, pt, T // pt, ph, H // ph, pw, W // pw, d)", ["pool_centre"]),
    ("route order", "np.lexsort((cand, -sc))", "np.lexsort((cand, sc))", ["route_planted", "route_brute"]),
    ("route self", "return [u for u in range(geo.n_win) if u != w]", "return list(range(geo.n_win))", ["route_planted", "route_brute"]),
    ("radius wraps", ["for ut in range(max(0, jt - r), min(nt, jt + r + 1)):", "for uy in range(max(0, jy - r), min(ny, jy + r + 1)):", "for ux in range(max(0, jx - r), min(nx, jx + r + 1)):", "u = (ut * ny + uy) * nx + ux"],
     ["for ut in range(jt - r, jt + r + 1):", "for uy in range(jy - r, jy + r + 1):", "for ux in range(jx - r, jx + r + 1):", "u = ((ut % nt) * ny + uy % ny) * nx + ux % nx"], ["radius_closed_form", "radius_brute"]),
    ("radius one-sided", "for ux in range(max(0, jx - r), min(nx, jx + r + 1)):", "for ux in range(max(0, jx - r), min(nx, jx + r)):", ["radius_closed_form", "radius_brute"]),
    ("radius ignores time", "for ut in range(max(0, jt - r), min(nt, jt + r + 1)):", "for ut in range(0, nt):", ["radius_brute"]),
    ("route tie", "np.lexsort((cand, -sc))", "np.lexsort((-cand, -sc))", ["route_ties"]),
    ("drop text keys", "                    kparts.append(k64[b, hh, N:])\n                    vparts.append(v64[b, hh, N:])\n                Kc", "                    pass\n                Kc", ["dense_masked", "constant_scores"]),
    ("drop pooled keys", "                    kparts.append(np.asarray(kp[b, hh], dtype=np.float64))\n                    vparts.append(np.asarray(vp[b, hh], dtype=np.float64))\n                if geo.n_text > 0:\n                    kparts.append(k64[b, hh, N:])", "                    pass\n                if geo.n_text > 0:\n                    kparts.append(k64[b, hh, N:])", ["dense_masked"]),
    ("scale", "scale = 1.0 / np.sqrt(d)", "scale = 1.0 / d", ["closed_form"]),
    ("softmax axis", "s = s - s.max(axis=1, keepdims=True)\n                p = np.exp(s)\n                p = p / p.sum(axis=1, keepdims=True)\n                Ow", "s = s - s.max(axis=0, keepdims=True)\n                p = np.exp(s)\n                p = p / p.sum(axis=0, keepdims=True)\n                Ow", ["closed_form", "rows_sum"]),
    ("routed window id", "u = int(route_idx[b, hh, w, r])", "u = int(route_idx[b, hh, (w + 1) % geo.n_win, r])", ["dense_masked"]),
    ("lse drops the max", "Lw[b, hh, w] = (m + np.log(l))[:, 0]", "Lw[b, hh, w] = np.log(l)[:, 0]", ["lse_scipy", "branch_merge"]),
    ("merge unnormalised", "out = sum(wts[i][..., None] * np.asarray(outs[i], dtype=np.float64) for i in range(len(outs))) / tot[..., None]", "out = sum(wts[i][..., None] * np.asarray(outs[i], dtype=np.float64) for i in range(len(outs)))", ["branch_merge"]),
    ("branch drops routed", "for u in [w] + [int(route_idx[b, hh, w, r]) for r in range(geo.routed_k)]:", "for u in [w]:", ["branch_merge", "lse_zero_q"]),
    ("text queries skip text keys", "            s = (qt[b, hh] @ k64[b, hh].T) / np.sqrt(d)", "            s = (qt[b, hh] @ k64[b, hh, : geo.N].T) / np.sqrt(d)", ["text_sdpa", "text_zero_q"]),
    ("text queries scale", "            s = (qt[b, hh] @ k64[b, hh].T) / np.sqrt(d)", "            s = (qt[b, hh] @ k64[b, hh].T) / d", ["text_sdpa"]),
    ("bwd softmax term", "dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))", "dS = P * dP", ["bwd_fd", "bwd_sdpa"]),
    ("bwd pool spread", "G = g_pool.reshape(B, h, T // pt, H // ph, W // pw, d) / (pt * ph * pw)", "G = g_pool.reshape(B, h, T // pt, H // ph, W // pw, d)", ["bwd_fd"]),
    ("bwd routed keys", "                    dKw[b, hh, u] += dKc[i * wt:(i + 1) * wt]", "                    dKw[b, hh, w] += dKc[i * wt:(i + 1) * wt]", ["bwd_fd"]),
    ("unshift output", "O = inverse_cyclic_shift(window_unpartition(Ow, geo.grid, geo.window), geo.shift)", "O = window_unpartition(Ow, geo.grid, geo.window)", ["dense_masked"]),
]

PINS = {
    "shift_membership": lambda: pins.test_shift_membership_golden(),
    "pool_centre": lambda: pins.test_pool_of_token_index_is_patch_centre(),
    "route_planted": lambda: pins.test_route_planted_winner_and_self_excluded(),
    "route_brute": lambda: [pins.test_route_matches_brute_force(g) for g in (pins.O.Geometry(grid=(1, 8, 12), window=(1, 4, 3), shift=(0, 1, 2), routed_k=3),)],
    "route_ties": lambda: pins.test_route_ties_go_to_lower_id(),
    "radius_closed_form": lambda: [pins.test_route_radius_picks_best_neighbour_in_closed_form(g) for g in (
        pins.O.Geometry(grid=(1, 16, 16), window=(1, 4, 4), shift=(0, 2, 3), routed_k=1, route_radius=1),
        pins.O.Geometry(grid=(6, 6, 9), window=(2, 2, 3), shift=(1, 1, 2), routed_k=1, route_radius=1))],
    "radius_brute": lambda: [pins.test_route_matches_brute_force(g) for g in (
        pins.O.Geometry(grid=(1, 12, 15), window=(1, 3, 3), shift=(0, 1, 2), routed_k=3, route_radius=1),
        pins.O.Geometry(grid=(6, 8, 8), window=(2, 2, 2), shift=(1, 1, 1), routed_k=7, route_radius=1))],
    "dense_masked": lambda: [pins.test_attention_matches_dense_masked_brute_force(g) for g in pins.TINY_GEOS],
    "constant_scores": lambda: [pins.test_constant_scores_give_mean_of_key_values(g) for g in pins.TINY_GEOS],
    "closed_form": lambda: pins.test_closed_form_whole_grid_is_dense_sdpa(),
    "rows_sum": lambda: [pins.test_softmax_rows_sum_to_one(g) for g in pins.TINY_GEOS],
    "lse_scipy": lambda: pins.test_lse_whole_grid_is_scipy_logsumexp(),
    "text_sdpa": lambda: pins.test_text_queries_dense_sdpa(),
    "bwd_fd": lambda: [pins.test_backward_matches_finite_differences(g) for g in pins.BWD_GEOS],
    "bwd_sdpa": lambda: pins.test_backward_whole_grid_is_sdpa_autograd(),
    "text_zero_q": lambda: pins.test_text_queries_zero_query_is_mean_of_all_values(),
    "lse_zero_q": lambda: pins.test_lse_of_zero_queries_is_log_of_key_count(),
    "branch_merge": lambda: [pins.test_branches_merge_to_the_joint_softmax(g) for g in pins.TINY_GEOS],
}


def _mutant(monkeypatch, old, new):
    src = inspect.getsource(basa_oracle)
    olds, news = (old, new) if isinstance(old, list) else ([old], [new])
    for o, n in zip(olds, news):
        assert src.count(o) >= 1, o
        src = src.replace(o, n, 1)
    mod = types.ModuleType("oracle_mutant")
    monkeypatch.setitem(sys.modules, "oracle_mutant", mod)
    exec(compile(src, "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, old, new, catchers):
    mutant = _mutant(monkeypatch, old, new)
    monkeypatch.setattr(pins, "O", mutant)
    for pin in catchers:
        with pytest.raises(Exception):
            PINS[pin]()

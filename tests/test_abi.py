"""Host-only checks of the C ABI: the library loads, exports what include/basa.h
declares, and rejects invalid calls with the documented status before any CUDA
call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from sparse_window_attention_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "basa.h")).read()
    return sorted(set(re.findall(r"^\w[\w\s\*]*?\b(basa_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert set(names) == set(B.EXPORTED), names
    lib = ctypes.CDLL(os.path.join(ROOT, "sparse_window_attention_b200", "libbasa.so"))
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code, name in B.STATUS_NAMES.items():
        assert B.basa_status_string(code) == name
    assert B.basa_device_error_status(0) == B.BASA_OK
    assert B.basa_device_error_status(2) == 5
    assert B.basa_device_error_status(B.BASA_DEVERR_BAD_ROUTE) == 6
    assert B.basa_device_error_status(B.BASA_DEVERR_BAD_ROUTE | 1) == 6


def test_params_struct_layout_matches_header():
    # 18 ints, a pointer, two uint32, an int -> 72 + 8 + 8 + 4 (+4 padding) bytes on LP64
    assert ctypes.sizeof(B.basa_params) == 96
    assert B.basa_params.dev_err.offset == 72
    assert B.basa_params.route_radius.offset == 88


def _p(**kw):
    base = dict(B=1, heads=2, head_dim=128, grid=(1, 64, 64), window=(1, 16, 16), shift=(0, 8, 8), pool=(1, 8, 8),
                n_text=16, routed_k=0, dtype="bf16", route_radius=0)
    base.update(kw)
    return B.make_params(base["B"], base["heads"], base["head_dim"], base["grid"], base["window"], base["shift"],
                         base["pool"], base["n_text"], base["routed_k"], base["dtype"], route_radius=base["route_radius"])


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: every case fails its checks first


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(head_dim=96), 3),
        (dict(grid=(1, 60, 64)), 2),
        (dict(window=(1, 16, 20)), 2),
        (dict(shift=(0, 64, 0)), 2),
        (dict(shift=(0, -1, 0)), 2),
        (dict(pool=(1, 8, 0)), 2),
        (dict(pool=(1, 7, 8)), 2),
        (dict(n_text=-1), 1),
        (dict(routed_k=16), 1),  # nWin - 1 = 15
        (dict(routed_k=17, grid=(1, 128, 128)), 1),
        (dict(B=-1), 1),
        (dict(dtype=7), 1),
        (dict(route_radius=-1), 1),
        # a corner window of the 1x4x4 window grid has 3 neighbours within radius 1
        (dict(routed_k=4, route_radius=1), 1),
        (dict(routed_k=9, route_radius=2, grid=(1, 128, 128)), 1),
    ],
)
def test_invalid_params_rejected_before_launch(kw, status):
    p = _p(**kw)
    if kw.get("dtype") == 7:
        p.dtype = 7
    got = B.basa_window_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE if p.routed_k > 0 else None, FAKE, p,
                                 stream=0, check=False)
    assert got == status


def test_pointer_rules():
    p = _p()
    # pooled pointers must be given iff a pool patch is set
    assert B.basa_window_attn_fwd(FAKE, FAKE, FAKE, None, None, None, FAKE, p, stream=0, check=False) == 1
    # misaligned
    assert B.basa_window_attn_fwd(FAKE + 8, FAKE, FAKE, FAKE, FAKE, None, FAKE, p, stream=0, check=False) == 1
    # null output
    assert B.basa_window_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, p, stream=0, check=False) == 1
    # route ids must be given iff routed_k > 0
    pr = _p(routed_k=2)
    assert B.basa_window_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, pr, stream=0, check=False) == 1
    assert B.basa_window_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, p, stream=0, check=False) == 1
    # bfloat16 attention is built for head_dim 128 only
    assert B.basa_window_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, _p(head_dim=64), stream=0, check=False) == 3
    # pooling needs a patch; routing needs routed_k >= 1
    assert B.basa_pool_kv(FAKE, FAKE, FAKE, FAKE, _p(pool=(0, 0, 0)), stream=0, check=False) == 1
    assert B.basa_route_windows(FAKE, FAKE, FAKE, None, FAKE, p, stream=0, check=False) == 1
    assert B.basa_route_windows(FAKE, FAKE, FAKE + 2, None, FAKE, pr, stream=0, check=False) == 1


def test_empty_batch_is_a_no_op():
    for kw in (dict(B=0), dict(heads=0)):
        p = _p(**kw)
        assert B.basa_window_attn_fwd(None, None, None, None, None, None, None, p, stream=0, check=False) == 0
        assert B.basa_pool_kv(None, None, None, None, p, stream=0, check=False) == 0


def test_route_radius_limits_routed_k():
    """routed_k may reach the fewest candidates any window has under the radius."""
    assert B.basa_route_workspace_bytes(_p(routed_k=3, route_radius=1)) > 0
    assert B.basa_route_workspace_bytes(_p(routed_k=4, route_radius=1)) == 0
    # 8x8 window grid, radius 2: a corner sees 3 x 3 positions, itself included
    assert B.basa_route_workspace_bytes(_p(routed_k=8, route_radius=2, grid=(1, 128, 128))) > 0
    assert B.basa_route_workspace_bytes(_p(routed_k=9, route_radius=2, grid=(1, 128, 128))) == 0
    # the full video configuration: 4x4 spatial window grid, one routed window
    p = B.make_params(1, 12, 128, (21, 60, 104), (21, 15, 26), (0, 7, 13), (1, 4, 4), 0, 1, "bf16", route_radius=1)
    assert B.basa_route_workspace_bytes(p) == 2 * 12 * 16 * 128 * 4


def test_fused_pool_route_checks():
    """basa_pool_route: needs pooling and routing; shapes whose boxes would hold too
    many pieces (pool patch ∩ window) are refused before any launch."""
    pr = _p(routed_k=2)
    n = B.basa_pool_route_workspace_bytes(pr)
    # window means (2 x heads x 16 windows x 128 floats) + at least one partial slot each
    assert n >= 2 * (2 * 2 * 16 * 128 * 4)
    assert B.basa_pool_route_workspace_bytes(_p()) == 0  # no routing
    assert B.basa_pool_route_workspace_bytes(_p(routed_k=2, pool=(0, 0, 0))) == 0
    assert B.basa_pool_route(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, _p(), stream=0, check=False) == 1
    # a 32x32 patch cut by 2x2 windows into 256 cells: more than one CTA may hold
    big = _p(routed_k=2, pool=(1, 32, 32), window=(1, 2, 2), shift=(0, 1, 1))
    assert B.basa_pool_route_workspace_bytes(big) == 0
    assert B.basa_pool_route(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, big, stream=0, check=False) == 3
    # null and misaligned pointers
    assert B.basa_pool_route(FAKE, FAKE, None, FAKE, FAKE, FAKE, None, FAKE, pr, stream=0, check=False) == 1
    assert B.basa_pool_route(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE + 4, pr, stream=0, check=False) == 1
    # the video configuration fits
    p = B.make_params(1, 12, 128, (21, 60, 104), (21, 15, 26), (0, 7, 13), (1, 4, 4), 0, 1, "bf16", route_radius=1)
    assert B.basa_pool_route_workspace_bytes(p) > 2 * 12 * 16 * 128 * 4


def test_branch_form_checks():
    p = _p()  # pool and 16 text rows, no routing
    call = lambda keys, pp=p: B.basa_window_attn_fwd_lse(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, keys, pp,
                                                         stream=0, check=False)
    assert call(0) == 1 and call(8) == 1
    nop = _p(pool=(0, 0, 0))
    assert B.basa_window_attn_fwd_lse(FAKE, FAKE, FAKE, None, None, None, FAKE, None, B.BASA_KEYS_POOLED, nop,
                                      stream=0, check=False) == 1
    assert call(B.BASA_KEYS_TEXT, _p(n_text=0)) == 1
    assert B.basa_window_attn_fwd_lse(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE + 2, B.BASA_KEYS_ALL, p,
                                      stream=0, check=False) == 1  # misaligned lse
    merge = lambda outs, lses, out=FAKE: B.basa_merge_branches(outs, lses, out, None, p, stream=0, check=False)
    assert merge([], []) == 1
    assert merge([FAKE] * 5, [FAKE] * 5) == 1
    assert merge([FAKE, None], [FAKE, FAKE]) == 1
    assert merge([FAKE, FAKE + 8], [FAKE, FAKE]) == 1
    assert merge([FAKE], [FAKE], out=None) == 1


def test_text_attn_checks():
    p = _p()
    assert B.basa_text_attn_fwd(FAKE, FAKE, FAKE, FAKE, None, _p(n_text=0), stream=0, check=False) == 1
    assert B.basa_text_attn_fwd(FAKE + 8, FAKE, FAKE, FAKE, None, p, stream=0, check=False) == 1
    assert B.basa_text_attn_fwd(FAKE, FAKE, FAKE, None, None, p, stream=0, check=False) == 1
    assert B.basa_text_attn_fwd(FAKE, FAKE, FAKE, FAKE, None, _p(head_dim=64), stream=0, check=False) == 3
    assert B.basa_text_attn_workspace_bytes(_p(n_text=0)) == 0


def test_backward_checks():
    pf = _p(dtype="f32")
    args = [FAKE] * 5 + [None] + [FAKE] * 7
    assert B.basa_window_attn_bwd(*args, _p(dtype="f32", head_dim=64), stream=0, check=False) == 3
    assert B.basa_window_attn_bwd(*args, _p(head_dim=64), stream=0, check=False) == 3  # bfloat16 needs 128
    bad = list(args)
    bad[12] = FAKE + 16  # bfloat16: the workspace must be 256-byte aligned
    assert B.basa_window_attn_bwd(*bad, _p(), stream=0, check=False) == 1
    bad[12] = None
    assert B.basa_window_attn_bwd(*bad, _p(), stream=0, check=False) == 1
    bad = list(args)
    bad[8] = None  # no dout
    assert B.basa_window_attn_bwd(*bad, pf, stream=0, check=False) == 1
    bad = list(args)
    bad[9] = FAKE + 4  # misaligned dq
    assert B.basa_window_attn_bwd(*bad, pf, stream=0, check=False) == 1
    # pooled gradients: 2 x heads x 64 patches x 128 floats
    assert B.basa_window_attn_bwd_workspace_bytes(pf) == 2 * 2 * 64 * 128 * 4
    # bfloat16 (computed on the host, the same on every device): per-token records
    # (2 heads x 4096 tokens x 16 B), chunk partials of the pooled and text key tiles
    # (2 heads x 2 tiles x 8 chunks of the 32 query tiles x [dK | dV] x 128 x 128 floats),
    # pooled-key gradients (2 x 2 heads x 64 x 128 floats)
    rec, part, pooled = 2 * 4096 * 16, 2 * 2 * 8 * 2 * 128 * 128 * 4, 2 * 2 * 64 * 128 * 4
    assert B.basa_window_attn_bwd_workspace_bytes(_p()) == rec + part + pooled


def test_route_workspace_bytes():
    p = _p(routed_k=2)
    assert B.basa_route_workspace_bytes(p) == 2 * 1 * 2 * 16 * 128 * 4
    assert B.basa_route_workspace_bytes(_p(head_dim=100)) == 0


def _bwd_chunks(wl, shift):
    """Chunk count of the bfloat16 backward's pooled/text key pass, read back from
    the workspace size (records + chunk partials + pooled-key gradients)."""
    p = B.make_params(wl.B, wl.heads, wl.d, wl.grid, wl.window, shift, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                      route_radius=wl.route_radius)
    bh = wl.B * wl.heads
    n = wl.grid[0] * wl.grid[1] * wl.grid[2]
    pt, ph, pw = wl.pool
    n_pool = (wl.grid[0] // pt) * (wl.grid[1] // ph) * (wl.grid[2] // pw)
    n_long = -(-n_pool // 128) + -(-wl.n_text // 128)
    up = lambda x: (x + 255) // 256 * 256
    part = B.basa_window_attn_bwd_workspace_bytes(p) - up(bh * n * 16) - up(bh * n_pool * 128 * 4 * 2)
    assert part % (bh * n_long * 2 * 128 * 128 * 4) == 0
    return part // (bh * n_long * 2 * 128 * 128 * 4), bh * n_long


def test_backward_chunking_fills_whole_waves():
    """The pooled/text pass splits each head's query tiles into the chunk count that
    minimises waves x (tiles per chunk + a CTA's fixed cost) on 148 SMs: one chunk
    (144 CTAs, one wave) at FLUX 2048^2 and 1024^2, six on Wan (144 CTAs), where
    the earlier rule of about two waves gave 2.9 and 2.1 waves."""
    from sparse_window_attention_b200 import synth

    for name, want in (("flux2k", 1), ("flux1k", 1), ("wan", 6)):
        wl = synth.WORKLOADS[name]
        chunks, units = _bwd_chunks(wl, synth.SHIFT_CYCLES[name][-1])
        assert chunks == want, (name, chunks)
        assert units * chunks <= 148, (name, units * chunks)  # one wave

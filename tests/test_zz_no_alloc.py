"""basa_route_windows_noalloc: routing for callers that cannot allocate a device
workspace (a plain C host without an allocator, a plugin inside a framework that
owns the device memory pool, a path where cudaMalloc's implicit synchronisation
is not allowed). It must give the same routed windows and scores as
basa_route_windows with a caller workspace, call after call, although every call
reuses the library's one fixed scratch array.

This file is collected last on purpose, so a failure here does not hide any
other test in a run that stops at the first failure.
"""
import numpy as np
import pytest
import torch

from sparse_window_attention_b200 import synth
from tests import parity as PT


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from sparse_window_attention_b200 import binding as B

    # 64 heads x 1024 windows x 128 x 4 B x 2 = 64 MiB > 4 MiB: rejected before any launch
    p = B.make_params(1, 64, 128, (1, 256, 256), (1, 8, 8), (0, 4, 4), (1, 8, 8), 0, 2, "bf16")
    assert B.basa_route_workspace_bytes(p) > 4 << 20
    fake = 0x7F0000000000
    assert B.basa_route_windows_noalloc(fake, fake, fake, None, p, stream=0, check=False) == 3


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    """Calls in a row: the Wan shape (1.7 MiB of window means), then 24 heads of the
    same grid (3.4 MiB, most of the scratch array), then the Wan shape again with
    other inputs, so the last call runs over stale means left past its own extent."""
    from sparse_window_attention_b200 import binding as B

    wan = synth.WORKLOADS["wan"]
    wide = synth.Workload(**{**wan.__dict__, "name": "wan_24_heads", "heads": 24})
    nwin = 140
    for call, (wl, seed) in enumerate(((wan, 0), (wide, 2), (wan, 1))):
        _, (qd, kd, _) = PT.gpu_inputs(wl, seed=seed)
        p = B.make_params(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.shift, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
        assert B.basa_route_workspace_bytes(p) <= 4 << 20
        shape = (wl.B, wl.heads, nwin, wl.routed_k)
        idx_ws = torch.full(shape, -1, dtype=torch.int32, device="cuda")
        sc_ws = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        ws = torch.empty(B.basa_route_workspace_bytes(p), dtype=torch.uint8, device="cuda")
        B.basa_route_windows(qd, kd, idx_ws, sc_ws, ws, p)
        idx_na = torch.full(shape, -1, dtype=torch.int32, device="cuda")
        sc_na = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        B.basa_route_windows_noalloc(qd, kd, idx_na, sc_na, p)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx_na.cpu().numpy(), idx_ws.cpu().numpy(), err_msg=f"call {call}")
        a = sc_na.cpu().numpy().astype(np.float64)
        b = sc_ws.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(a - b) <= PT.ROUTE_SCORE_TOL * np.maximum(1.0, np.abs(b))), f"call {call}"

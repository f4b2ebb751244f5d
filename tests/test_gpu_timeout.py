"""Failure detection without a GPU fault: a test hook makes the attention
kernel's loader (forward, and each pass of the bfloat16 backward) skip the first
key or query tile, so every wait on it runs into its (short) time limit; the
kernel records the expiry in the device error word, frees its resources and
returns. The context must stay usable."""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives():
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    wl = synth.Workload("timeout", "bf16", 1, 2, 128, (1, 32, 32), (1, 16, 16), (0, 8, 8), (1, 8, 8), 0, 0, "iid")
    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl)
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype, route_radius=wl.route_radius)
    out = torch.zeros_like(qd)
    layer.pool_kv(kd, vd, wl.shift)
    layer.attention(qd, kd, vd, out, wl.shift, flags=B.BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD, wait_timeout_us=20000)
    torch.cuda.synchronize()
    err = layer.device_error()
    # whichever role's wait expires first records its bit (loader 0x1, MMA 0x2, softmax 0x4)
    assert err != 0 and (err & ~0x7) == 0, f"expected timeout bits in the device error word, got {err:#x}"
    assert B.basa_device_error_status(err) == 5
    assert B.basa_status_string(B.basa_device_error_status(err)) == "BASA_ERR_DEVICE_TIMEOUT"
    # no output was stored
    assert torch.count_nonzero(out).item() == 0
    # the context is still usable: a normal call matches the oracle
    layer.dev_err.zero_()
    out2 = layer.forward(qd, kd, vd, wl.shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    geo = PT.geometry(wl)
    ref = O.basa_attention(PT.to64(q), PT.to64(k), PT.to64(v), geo)
    PT.assert_outputs_close(PT.to64(out2), ref, "bf16", "after timeout")


def test_backward_bounded_wait_expires_and_context_survives():
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    wl = synth.Workload("timeout_bwd", "bf16", 1, 2, 128, (1, 32, 32), (1, 16, 16), (0, 8, 8), (1, 8, 8), 256, 0, "iid")
    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl)
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
    layer.pool_kv(kd, vd, wl.shift)
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out, lse, wl.shift, B.BASA_KEYS_ALL)
    dout = torch.from_numpy(np.random.default_rng(3).standard_normal(q.shape, dtype=np.float32)).to(torch.bfloat16)
    doutd = dout.to(qd.device)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    # every pass (dq, pooled/text dK/dV, window dK/dV) skips its first ring load
    layer.backward(qd, kd, vd, out, lse, doutd, wl.shift, flags=B.BASA_FLAG_TEST_SKIP_FIRST_KEY_LOAD,
                   wait_timeout_us=20000)
    torch.cuda.synchronize()
    err = layer.device_error()
    assert err != 0 and (err & ~0x7) == 0, f"expected timeout bits in the device error word, got {err:#x}"
    assert B.basa_device_error_status(err) == 5
    # the context is still usable: a normal backward matches the oracle
    layer.dev_err.zero_()
    dq, dk, dv = layer.backward(qd, kd, vd, out, lse, doutd, wl.shift)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    geo = PT.geometry(wl)
    refs = O.basa_attention_backward(PT.to64(q), PT.to64(k), PT.to64(v), geo, PT.to64(dout))
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        g64 = PT.to64(g)
        rel = np.linalg.norm(g64 - r) / np.linalg.norm(r)
        assert np.isfinite(g64).all() and rel <= 1e-2, (name, rel)

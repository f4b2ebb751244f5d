"""GPU parity of the text-query rows: dense attention of the text queries over
every visual and text key (basa_text_attn_fwd), against the oracle."""
import numpy as np
import pytest
import torch

from oracle import basa_oracle as O
from sparse_window_attention_b200 import synth
from tests import parity as PT

pytestmark = pytest.mark.gpu

W = synth.Workload

CASES = [
    synth.WORKLOADS["flux2k"],
    synth.WORKLOADS["flux1k"],
    # ragged text rows (77) and a key count that is not a multiple of 128
    W("text77", "bf16", 2, 2, 128, (1, 48, 48), (1, 16, 16), (0, 8, 8), (1, 4, 4), 77, 0, "sinusoid"),
    # one text row
    W("text1", "bf16", 1, 3, 128, (2, 16, 24), (1, 8, 8), (1, 4, 4), (0, 0, 0), 1, 0, "iid"),
    W("f32_d128", "f32", 1, 2, 128, (2, 16, 16), (1, 8, 8), (1, 4, 2), (2, 4, 4), 9, 2, "block_mean"),
    W("f32_d64", "f32", 2, 3, 64, (1, 24, 16), (1, 8, 8), (0, 5, 3), (1, 4, 4), 33, 1, "iid"),
]


def _q_text(wl, seed=7):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((wl.B, wl.heads, wl.n_text, wl.d), dtype=np.float32)
    t = torch.from_numpy(x)
    return t.to(torch.bfloat16) if wl.dtype == "bf16" else t


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_text_queries_match_oracle(wl):
    from sparse_window_attention_b200.layer import BasaLayer

    (q, k, v), (qd, kd, vd) = PT.gpu_inputs(wl)
    qt = _q_text(wl)
    qtd = qt.cuda()
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
    out = torch.full_like(qtd, float("nan"))
    layer.text_attention(qtd, kd, vd, out)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    hs = list(range(wl.heads)) if wl.heads <= 4 else [0, wl.heads // 2, wl.heads - 1]
    geo = PT.geometry(wl)
    ref = O.text_query_attention(PT.to64(qt[:, hs]), PT.to64(k[:, hs]), PT.to64(v[:, hs]), geo)
    PT.assert_outputs_close(PT.to64(out[:, hs]), ref, wl.dtype, f"{wl.name} text queries")
    assert not torch.isnan(out).any()
    # deterministic
    out2 = torch.empty_like(out)
    layer.text_attention(qtd, kd, vd, out2)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)

"""One BASA layer call on device tensors: pool -> (route) -> attention.

``BasaLayer`` owns the intermediate device buffers of one layer shape (pooled
K/V, routed window ids and scores, the routing workspace and the device error
word), allocated once with torch, and calls the three C entry points on the
current CUDA stream. It computes nothing itself.
"""
from __future__ import annotations

import torch

from . import binding as B
from . import sharding


class BasaLayer:
    def __init__(self, batch, heads, head_dim, grid, window, pool=(0, 0, 0), n_text=0, routed_k=0, dtype="bf16",
                 device="cuda", route_radius=0):
        self.batch, self.heads, self.head_dim = batch, heads, head_dim
        self.grid, self.window, self.pool = tuple(grid), tuple(window), tuple(pool)
        self.n_text, self.routed_k, self.dtype = n_text, routed_k, dtype
        self.route_radius = route_radius
        self.device = torch.device(device)
        T, H, W = self.grid
        self.N = T * H * W
        self.n_win = (T // window[0]) * (H // window[1]) * (W // window[2])
        self.has_pool = all(p > 0 for p in self.pool)
        self.n_pool = (T // pool[0]) * (H // pool[1]) * (W // pool[2]) if self.has_pool else 0
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        self._params = {}
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.kp = self.vp = None
        if self.has_pool:
            self.kp = torch.empty(batch, heads, self.n_pool, head_dim, dtype=tdt, device=self.device)
            self.vp = torch.empty_like(self.kp)
        self.route_idx = self.route_score = self.workspace = None
        if routed_k > 0:
            self.route_idx = torch.empty(batch, heads, self.n_win, routed_k, dtype=torch.int32, device=self.device)
            self.route_score = torch.empty(batch, heads, self.n_win, routed_k, dtype=torch.float32, device=self.device)
            nbytes = B.basa_route_workspace_bytes(self.params((0, 0, 0)))
            self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=self.device)
        # fused pooling + routing pass (one read of q, k, v) where the shape allows it;
        # its workspace size depends on the shift and grows on first use
        self.fused = self.has_pool and routed_k > 0
        self.fused_workspace = None
        self.text_workspace = None  # text-query rows: per-split partial results
        self._branch_bufs = []      # branch form: (out, lse) per branch

    @classmethod
    def for_shard(cls, batch, heads, head_dim, grid, window, world, rank, **kw):
        """The layer for rank `rank` of `world` GPUs splitting the (batch, head) units
        (sharding.unit_shard): it runs B = 1 and its own units as heads, on the views
        `layer.shard_of(x)` of the full tensors. Pooling, routing and attention have no
        term across heads, so the shards need no exchange."""
        start, stop = sharding.unit_shard(batch, heads, world, rank)
        layer = cls(1, stop - start, head_dim, grid, window, **kw)
        layer.units = (start, stop)
        return layer

    def shard_of(self, x):
        """This layer's units of a full [B, heads, rows, d] tensor (a view, no copy)."""
        start, stop = getattr(self, "units", (0, self.batch * self.heads))
        return sharding.shard_view(x, start, stop)

    def params(self, shift, **extra) -> B.basa_params:
        key = (tuple(shift), tuple(sorted(extra.items())))
        if key not in self._params:
            self._params[key] = B.make_params(self.batch, self.heads, self.head_dim, self.grid, self.window, shift,
                                              self.pool, self.n_text, self.routed_k, self.dtype,
                                              dev_err=self.dev_err, route_radius=self.route_radius, **extra)
        return self._params[key]

    def pool_kv(self, k, v, shift=(0, 0, 0), stream=None):
        B.basa_pool_kv(k, v, self.kp, self.vp, self.params(shift), stream)

    def route(self, q, k, shift, stream=None):
        B.basa_route_windows(q, k, self.route_idx, self.route_score, self.workspace, self.params(shift), stream)

    def fused_bytes(self, shift) -> int:
        return B.basa_pool_route_workspace_bytes(self.params(shift))

    def pool_route(self, q, k, v, shift, stream=None):
        """Pooled K/V and routed windows in one pass (basa_pool_route)."""
        nbytes = self.fused_bytes(shift)
        if self.fused_workspace is None or self.fused_workspace.numel() < nbytes:
            self.fused_workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=self.device)
        B.basa_pool_route(q, k, v, self.kp, self.vp, self.route_idx, self.route_score, self.fused_workspace,
                          self.params(shift), stream)

    def attention(self, q, k, v, out, shift, kp=None, vp=None, route_idx=None, stream=None, **extra):
        kp = self.kp if kp is None else kp
        vp = self.vp if vp is None else vp
        route_idx = self.route_idx if route_idx is None else route_idx
        B.basa_window_attn_fwd(q, k, v, kp, vp, route_idx, out, self.params(shift, **extra), stream)

    def attention_lse(self, q, k, v, out, lse, shift, keys, kp=None, vp=None, route_idx=None, stream=None):
        """One branch: attention over the key groups in ``keys`` and its log-sum-exp."""
        kp = self.kp if kp is None else kp
        vp = self.vp if vp is None else vp
        route_idx = self.route_idx if route_idx is None else route_idx
        B.basa_window_attn_fwd_lse(q, k, v, kp, vp, route_idx, out, lse, keys, self.params(shift), stream)

    def merge(self, outs, lses, out, lse=None, stream=None):
        """Joint softmax from branch results (basa_merge_branches)."""
        B.basa_merge_branches(outs, lses, out, lse, self.params((0, 0, 0)), stream)

    def forward_branches(self, q, k, v, shift, splits, out=None, stream=None):
        """The layer in branch form: pooled K/V and routing as in forward(), then one
        attention call per key-group set in ``splits`` (e.g. [WINDOWS, POOLED | TEXT])
        and their merge."""
        if out is None:
            out = torch.empty_like(q)
        if self.fused and self.fused_bytes(shift) > 0:
            self.pool_route(q, k, v, shift, stream)
        else:
            if self.has_pool:
                self.pool_kv(k, v, shift, stream)
            if self.routed_k > 0:
                self.route(q, k, shift, stream)
        if len(self._branch_bufs) < len(splits):
            self._branch_bufs = [(torch.empty_like(q), torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device))
                                 for _ in splits]
        for (o, l), keys in zip(self._branch_bufs, splits):
            self.attention_lse(q, k, v, o, l, shift, keys, stream=stream)
        bufs = self._branch_bufs[: len(splits)]
        self.merge([o for o, _ in bufs], [l for _, l in bufs], out, None, stream)
        return out

    def text_attention(self, q_text, k, v, out_text, stream=None):
        """Output rows of the text queries (dense over all keys; basa_text_attn_fwd)."""
        nbytes = B.basa_text_attn_workspace_bytes(self.params((0, 0, 0)))
        ws = None
        if nbytes > 0:
            if self.text_workspace is None or self.text_workspace.numel() < nbytes:
                self.text_workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            ws = self.text_workspace
        B.basa_text_attn_fwd(q_text, k, v, out_text, ws, self.params((0, 0, 0)), stream)

    def backward(self, q, k, v, out, lse, dout, shift, stream=None, **extra):
        """dq, dk, dv of the attention (basa_window_attn_bwd: bfloat16 on the tensor
        cores, or float32) for the pooled K/V and routed windows currently held by
        the layer; `lse` is the forward's log-sum-exp over all keys. ``extra`` goes
        into the parameters (e.g. ``wait_timeout_us``, ``flags``)."""
        dq = torch.empty_like(q)
        dk = torch.empty_like(k)
        dv = torch.empty_like(v)
        params = self.params(shift, **extra)
        nbytes = B.basa_window_attn_bwd_workspace_bytes(params)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device) if nbytes else None
        B.basa_window_attn_bwd(q, k, v, self.kp, self.vp, self.route_idx, out, lse, dout, dq, dk, dv, ws, params,
                               stream)
        return dq, dk, dv

    def forward(self, q, k, v, shift, out=None, stream=None):
        """Full layer: pooled K/V, routed windows (if routed_k > 0), attention."""
        if out is None:
            out = torch.empty_like(q)
        if self.fused and self.fused_bytes(shift) > 0:
            self.pool_route(q, k, v, shift, stream)
        else:
            if self.has_pool:
                self.pool_kv(k, v, shift, stream)
            if self.routed_k > 0:
                self.route(q, k, shift, stream)
        self.attention(q, k, v, out, shift, stream=stream)
        return out

    def launches_per_forward(self) -> int:
        # fused: pool + partial sums, reduction, top-k; else pool, means + top-k
        return (1 if self.has_pool else 0) + (2 if self.routed_k > 0 else 0) + 1

    def device_error(self) -> int:
        return int(self.dev_err.item())

"""Multi-rank host logic on CPU (gloo, world size 2): the (batch, head) shards of
each rank, computed independently, reassemble the full layer, and the timing
reduction returns the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_window_attention_b200.sharding import max_over_ranks, shard_view, unit_shard


@pytest.mark.parametrize("B,heads,world", [(1, 24, 2), (2, 3, 4), (1, 5, 8), (3, 1, 2)])
def test_unit_shards_partition_all_units(B, heads, world):
    seen = []
    for r in range(world):
        a, b = unit_shard(B, heads, world, r)
        assert 0 <= a <= b <= B * heads
        seen.extend(range(a, b))
    assert seen == list(range(B * heads))
    sizes = [unit_shard(B, heads, world, r)[1] - unit_shard(B, heads, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import basa_oracle as O

        geo = O.Geometry(grid=(2, 8, 12), window=(1, 4, 4), shift=(1, 2, 3), pool=(2, 4, 4), n_text=3, routed_k=2)
        B, heads, d = 2, 3, 8
        rng = np.random.default_rng(0)  # same full inputs on every rank
        q = rng.standard_normal((B, heads, geo.N, d))
        k = rng.standard_normal((B, heads, geo.N + geo.n_text, d))
        v = rng.standard_normal((B, heads, geo.N + geo.n_text, d))
        a, b = unit_shard(B, heads, world, rank)
        # the rank's units as the product takes them: flat [1, units, rows, d] views
        qv, kv, vv = (shard_view(torch.from_numpy(x), a, b).numpy() for x in (q, k, v))
        part = O.basa_attention(qv, kv, vv, geo)  # [1, this rank's units, N, d]
        gathered = [None] * world
        dist.all_gather_object(gathered, (a, b, part))
        t = max_over_ranks(float(rank + 1) * 0.5)
        if rank == 0:
            full = O.basa_attention(q, k, v, geo)
            got = np.zeros_like(full).reshape(1, B * heads, geo.N, d)
            for a_, b_, p_ in gathered:
                got[:, a_:b_] = p_.reshape(1, -1, geo.N, d)
            got = got.reshape(full.shape)
            np.save(os.path.join(out_dir, "err.npy"), np.array([np.abs(got - full).max(), t]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shards_reassemble_layer_and_max_timing(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    err, t = np.load(tmp_path / "err.npy")
    assert err < 1e-12
    assert t == 1.0  # max of 0.5, 1.0


def test_shard_view_is_a_view_of_the_units():
    x = torch.arange(2 * 3 * 5 * 4, dtype=torch.float32).reshape(2, 3, 5, 4)
    for world in (1, 2, 4):
        parts = []
        for r in range(world):
            a, b = unit_shard(2, 3, world, r)
            v = shard_view(x, a, b)
            assert v.shape == (1, b - a, 5, 4) and v.is_contiguous()
            assert v.data_ptr() == x.data_ptr() + a * 5 * 4 * x.element_size()
            parts.append(v)
        assert torch.equal(torch.cat(parts, dim=1).reshape(x.shape), x)

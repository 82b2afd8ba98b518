"""The N > 1 path on CPU: world size 2 with the gloo backend.

Each rank owns a contiguous slice of a global batch (batch_shard), computes
it (here with the fp64 oracle, standing in for the device), and the slices
put together equal the whole batch computed at once; the timing reduction
takes the maximum over ranks.  No data-path collective is involved: results
are gathered only to check them.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from blockwise_exact_attention_attn_b200.shard import batch_shard, max_over_ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, S, H, D, N = 5, 48, 2, 8, 4
        g = torch.Generator().manual_seed(99)
        q, k, v = (torch.randn(B, S, H, D, generator=g, dtype=torch.float64) for _ in range(3))
        b0, b1 = batch_shard(B, rank, world)
        mine = slice(b0, b1)
        nb = b1 - b0
        p = oracle.Problem(q=q[mine].reshape(-1, H, D).numpy(), k=k[mine].reshape(-1, H, D).numpy(),
                           v=v[mine].reshape(-1, H, D).numpy(), seq_start=np.arange(nb) * S,
                           seq_len=np.full(nb, S), n_ring=N, layout=1, causal=True, passes=3,
                           scale=0.35)
        o, lse = oracle.attention_full(p)
        # gather (checking only) -- pad to the largest shard
        cap = (B + world - 1) // world
        buf = torch.zeros(cap * S, H, D, dtype=torch.float64)
        buf[:nb * S] = torch.from_numpy(o)
        parts = [torch.zeros_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf)
        t_max = max_over_ranks(float(rank + 1))
        if rank == 0:
            full = oracle.Problem(q=q.reshape(-1, H, D).numpy(), k=k.reshape(-1, H, D).numpy(),
                                  v=v.reshape(-1, H, D).numpy(), seq_start=np.arange(B) * S,
                                  seq_len=np.full(B, S), n_ring=N, layout=1, causal=True,
                                  passes=3, scale=0.35)
            o_full, _ = oracle.attention_full(full)
            pieces = []
            for r in range(world):
                a, b = batch_shard(B, r, world)
                pieces.append(parts[r][:(b - a) * S].numpy())
            got = np.concatenate(pieces)
            result["err"] = float(np.abs(got - o_full).max())
            result["tmax"] = t_max
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_batch_shard_partitions():
    for B in range(0, 20):
        for W in range(1, 6):
            seen = []
            for r in range(W):
                a, b = batch_shard(B, r, W)
                seen.extend(range(a, b))
                assert 0 <= b - a <= -(-B // W)
            assert seen == list(range(B))
    with pytest.raises(ValueError):
        batch_shard(4, 2, 2)


def test_two_rank_gloo_shards_equal_whole():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    result = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), result), nprocs=world,
                       join=True, start_method="spawn")
    assert result["err"] < 1e-12
    assert result["tmax"] == float(world)

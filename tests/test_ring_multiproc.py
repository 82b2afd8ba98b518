"""The sequence-parallel ring (ring.ring_attention_forward) with 2 and 4
gloo ranks on CPU.

Each rank holds one ring block of q, k, v; the key/value blocks travel
around the ring by point-to-point messages and each step is folded with the
fp64 oracle's ring step, standing in for the device kernel
(ring_attn_fwd_step, which the GPU tests check against the same oracle
fold).  The blocks' results put together equal full attention over the whole
sequence, for contiguous and striped layouts, causal or not, and with a pass
limit below the ring size.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from blockwise_exact_attention_attn_b200.ring import ring_attention_forward


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_fold(q, k, v, out, lse, q_block, kv_block, accumulate, seqlen, n_ring, layout,
                causal, scale):
    import oracle
    for bi in range(q.shape[0]):
        prev_o = out[bi].numpy() if accumulate else np.zeros(tuple(q[bi].shape))
        prev_l = lse[bi].numpy() if accumulate else np.full(tuple(lse[bi].shape), -np.inf)
        o, l = oracle.ring_step(q[bi].numpy(), k[bi].numpy(), v[bi].numpy(), prev_o, prev_l,
                                seqlen, n_ring, layout, causal, scale, q_block, kv_block)
        out[bi] = torch.from_numpy(o)
        lse[bi] = torch.from_numpy(l)


def _worker(rank, world, port, case, result):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layout, causal, P = case
        B, b, H, D = 1, 6, 2, 4
        L = b * world
        g = torch.Generator().manual_seed(123)
        q, k, v = (torch.randn(B, L, H, D, generator=g, dtype=torch.float64) for _ in range(3))
        rows = oracle.block_rows(L, world, layout, rank)
        out, lse = ring_attention_forward(q[:, rows], k[:, rows].contiguous(),
                                          v[:, rows].contiguous(), causal=causal, layout=layout,
                                          softmax_scale=0.4, max_ring_passes=P,
                                          fold=oracle_fold)
        outs = [torch.zeros_like(out) for _ in range(world)]
        lses = [torch.zeros_like(lse) for _ in range(world)]
        dist.all_gather(outs, out.contiguous())
        dist.all_gather(lses, lse.contiguous())
        if rank == 0:
            p = oracle.Problem(q=q[0].numpy(), k=k[0].numpy(), v=v[0].numpy(),
                               seq_start=np.array([0]), seq_len=np.array([L]), n_ring=world,
                               layout=layout, causal=causal, passes=P, scale=0.4)
            o_ref, l_ref = oracle.attention_full(p)
            err_o = err_l = 0.0
            for r in range(world):
                rr = oracle.block_rows(L, world, layout, r)
                err_o = max(err_o, float(np.abs(outs[r][0].numpy() - o_ref[rr]).max()))
                err_l = max(err_l, float(np.abs(lses[r][0].numpy() - l_ref[:, rr]).max()))
            result.put((err_o, err_l))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", [(0, True, None), (1, True, 2), (0, False, None),
                                  (1, False, 3)])
def test_ring_across_ranks_equals_full_attention(world, case):
    layout, causal, P = case
    P = world if P is None else min(P, world)
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, (layout, causal, P), result))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    err_o, err_l = result.get(timeout=10)
    assert err_o < 1e-12 and err_l < 1e-12


@pytest.mark.parametrize("dtype,shape,scale", [
    (torch.float32, (1, 128, 2, 128), 0.1),      # fp32 has no device ring step
    (torch.bfloat16, (1, 128, 2, 32), 0.1),      # d_head 32
    (torch.bfloat16, (1, 100, 2, 128), 0.1),     # block not whole 128-row tiles
    (torch.bfloat16, (1, 128, 2, 128), 0.0),     # zero scale
])
def test_device_fold_arguments_are_refused_before_any_exchange(dtype, shape, scale):
    # the check needs no process group: every rank refuses before communicating
    from blockwise_exact_attention_attn_b200.ring import check_device_fold
    with pytest.raises(ValueError):
        check_device_fold(torch.zeros(*shape, dtype=dtype), scale)


def test_device_fold_arguments_accepted():
    from blockwise_exact_attention_attn_b200.ring import check_device_fold
    for dt, D in ((torch.bfloat16, 128), (torch.float16, 64)):
        check_device_fold(torch.zeros(2, 256, 3, D, dtype=dt), -0.5)

"""The ring driver on the GPU with the device fold (ring_attn_fwd_step), one
NCCL rank: the whole sequence is one ring block, so the ring is a single
step.  The multi-rank exchange runs with gloo ranks on CPU
(test_ring_multiproc.py); one GPU per test run gives no second device.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from blockwise_exact_attention_attn_b200.ring import ring_attention_forward
from gpu_util import TOL

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("causal,layout", [(True, 0), (False, 1)])
def test_single_rank_ring_matches_the_oracle(causal, layout):
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=dev)
    try:
        B, L, H, D = 1, 512, 2, 128
        g = torch.Generator().manual_seed(91)
        q, k, v = (torch.randn(B, L, H, D, generator=g).to(torch.bfloat16) for _ in range(3))
        out, lse = ring_attention_forward(q.to(dev), k.to(dev), v.to(dev), causal=causal,
                                          layout=layout, softmax_scale=0.08,
                                          out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert out.dtype == torch.bfloat16 and lse.dtype == torch.float32
        p = oracle.Problem(q=q[0].float().numpy(), k=k[0].float().numpy(),
                           v=v[0].float().numpy(), seq_start=np.array([0]),
                           seq_len=np.array([L]), n_ring=1, layout=layout, causal=causal,
                           passes=1, scale=0.08)
        o_ref, l_ref = oracle.attention_full(p)
        assert float(np.abs(out[0].float().cpu().numpy() - o_ref).max()) <= TOL["bf16"][0]
        assert float(np.abs(lse[0].cpu().numpy() - l_ref).max()) <= TOL["bf16"][1]
    finally:
        dist.destroy_process_group()

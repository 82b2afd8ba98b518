"""ring_attn_func_host: the forward from pinned host tensors, with copies
and kernels of different chunks of sequences overlapped on three streams,
returns exactly what the device call returns."""

import pytest
import torch

import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,chunk,Hkv", [(3, 1, 2), (4, 2, 1), (1, 1, 2)])
def test_host_call_equals_device_call(B, chunk, Hkv):
    w = gen.Workload("host", "bf16", B, 2, 1024, 128, True, 4, 1, 3, seed=55, heads_kv=Hkv)
    inp = gen.make_inputs(w)
    host = [inp[n].pin_memory() for n in ("q", "k", "v")]
    out_h, lse_h = ra.ring_attn_func_host(*host, w.n_ring, w.causal, w.layout, None, w.passes,
                                          chunk=chunk)
    dev = [t.cuda() for t in host]
    out_d, lse_d = ra.ring_attn_func(*dev, w.n_ring, w.causal, w.layout, None, w.passes)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    assert out_h.is_pinned() and not out_h.is_cuda
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(lse_h, lse_d.cpu())


def test_host_call_refuses_pageable_inputs():
    x = torch.zeros(1, 256, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ra.ring_attn_func_host(x, x, x, 2)

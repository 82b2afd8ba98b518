"""ring_attn_fwd_host: the forward from page-locked host tensors through the
C ABI, with chunks of heads copied in, computed and copied out on three
streams.  It must return exactly what the device call returns, for every
chunking (one head per chunk, a ragged last chunk, a single chunk), and
leave the caller's stream ordered after its last copy."""

import pytest
import torch

import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,B,H,head_chunk", [
    ("bf16", 1, 4, 1), ("bf16", 2, 5, 2), ("bf16", 3, 3, 0), ("bf16", 1, 2, 8),
    ("f16", 2, 4, 3), ("f32", 1, 3, 1)])
def test_host_call_equals_device_call(dtype, B, H, head_chunk):
    d = 16 if dtype == "f32" else 128
    w = gen.Workload("host", dtype, B, H, 1024, d, True, 4, gen.STRIPED, 3, seed=55)
    inp = gen.make_inputs(w)
    host = [inp[n].pin_memory() for n in ("q", "k", "v")]
    S = w.seqlen
    out_h = torch.full((B, S, H, d), float("nan"), dtype=w.torch_dtype).pin_memory()
    lse_h = torch.full((B, H, S), float("nan")).pin_memory()
    code = {"bf16": ra.BF16, "f16": ra.F16, "f32": ra.F32}[dtype]
    nbytes = ra.ring_attn_fwd_host_workspace(B, H, S, d, code, head_chunk)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    for _ in range(2):   # the second call reuses the workspace and the library streams
        ra.ring_attn_fwd_host(*host, out_h, lse_h, B, H, S, d, w.n_ring, w.layout, w.causal,
                              w.softmax_scale, w.passes, ws, head_chunk)
        torch.cuda.current_stream().synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    out_d, lse_d = ra.ring_attn_func(*(t.cuda() for t in host), w.n_ring, w.causal, w.layout,
                                     w.softmax_scale, w.passes)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(lse_h, lse_d.cpu())


def test_func_host_wrapper_allocates_its_workspace():
    w = gen.Workload("host", "bf16", 2, 3, 512, 64, False, 2, gen.CONTIGUOUS, 2, seed=56)
    inp = gen.make_inputs(w)
    host = [inp[n].pin_memory() for n in ("q", "k", "v")]
    out_h, lse_h = ra.ring_attn_func_host(*host, w.n_ring, w.causal, w.layout, None, w.passes)
    out_d, lse_d = ra.ring_attn_func(*(t.cuda() for t in host), w.n_ring, w.causal, w.layout,
                                     None, w.passes)
    torch.cuda.synchronize()
    assert out_h.is_pinned() and not out_h.is_cuda
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


def test_host_call_refuses_pageable_inputs_and_small_workspaces():
    x = torch.zeros(1, 256, 1, 128, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 256)
    xp, lp = x.pin_memory(), lse.pin_memory()
    need = ra.ring_attn_fwd_host_workspace(1, 1, 256, 128, ra.BF16, 0)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(ra.RingAttnError):       # pageable q
        ra.ring_attn_fwd_host(x, xp, xp, xp, lp, 1, 1, 256, 128, 2, workspace=ws)
    with pytest.raises(ra.RingAttnError):       # workspace one byte short
        ra.ring_attn_fwd_host(xp, xp, xp, xp, lp, 1, 1, 256, 128, 2, workspace=ws[:need - 1])
    ra.ring_attn_fwd_host(xp, xp, xp, xp, lp, 1, 1, 256, 128, 2, workspace=ws)
    torch.cuda.current_stream().synchronize()
    assert ra.ring_attn_status() == ra.RA_OK

"""Grouped-query and multi-query attention on the GPU (ring_attn_gqa_fwd)
against the fp64 oracle, whose key/value head map is pinned against torch's
grouped-query attention.

Query head h reads key/value head h // (heads / heads_kv).  Same tolerances
as the other parity tests; the GPU result must also equal, bit for bit, the
ordinary multi-head call on key/value heads repeated to one per query head
(the kernels read the same values in the same order).
"""

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
from gpu_util import TOL, compare_full, compare_rows, run_gpu, sample_rows

pytestmark = pytest.mark.gpu

GQA_SMALL = [
    # (dtype, B, H, H_kv, S, D, causal, N, layout, P)
    ("bf16", 1, 4, 2, 1024, 128, True, 8, 0, 8),
    ("bf16", 2, 4, 1, 768, 128, False, 4, 1, 2),     # multi-query
    ("bf16", 1, 6, 3, 640, 64, True, 5, 0, 5),
    ("bf16", 1, 8, 2, 1000, 128, True, 8, 1, 3),
    ("f32", 1, 4, 2, 512, 64, True, 4, 0, 4),        # CUDA-core kernel
]


def check(w, err_o, err_l):
    to, tl = TOL[w.dtype]
    assert err_o <= to and err_l <= tl, (w.name, err_o, err_l)


@pytest.mark.parametrize("case", GQA_SMALL, ids=lambda c: "-".join(map(str, c)))
def test_gqa_small_all_rows(case):
    dt, B, H, Hkv, S, D, causal, N, layout, P = case
    w = gen.Workload("gqa", dt, B, H, S, D, causal, N, layout, P, seed=300 + S, heads_kv=Hkv)
    inp = gen.make_inputs(w)
    assert inp["k"].shape[2] == Hkv
    out, lse = run_gpu(w, inp)
    check(w, *compare_full(w, inp, out, lse))


@pytest.mark.parametrize("dt,D", [("bf16", 128), ("bf16", 64), ("f32", 32)])
def test_gqa_equals_multi_head_on_repeated_heads_bitwise(dt, D):
    H, Hkv = 8, 2
    w = gen.Workload("gqa", dt, 1, H, 1024, D, True, 4, 1, 3, seed=41, heads_kv=Hkv)
    inp = gen.make_inputs(w)
    out_g, lse_g = run_gpu(w, inp)
    rep = dict(inp)
    rep["k"] = inp["k"].repeat_interleave(H // Hkv, dim=2).contiguous()
    rep["v"] = inp["v"].repeat_interleave(H // Hkv, dim=2).contiguous()
    out_m, lse_m = run_gpu(gen.Workload("mha", dt, 1, H, 1024, D, True, 4, 1, 3, seed=41), rep)
    assert torch.equal(out_g, out_m)
    assert torch.equal(lse_g, lse_m)


def test_gqa_varlen_all_rows():
    dev = torch.device("cuda", 0)
    lens = [700, 129, 1500, 64]
    H, Hkv, D, N, P = 4, 2, 128, 4, 4
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(12)
    q = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    out = torch.empty(T, H, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(H, T, device=dev)
    scale = 1.0 / np.sqrt(D)
    ra.ring_attn_gqa_fwd(q.to(dev), k.to(dev), v.to(dev), out, lse, len(lens), H, Hkv, T, D, N,
                         0, True, scale, P, cu.to(dev))
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    p = oracle.Problem(q=q.float().numpy(), k=k.float().numpy(), v=v.float().numpy(),
                       seq_start=cu[:-1].numpy(), seq_len=np.array(lens), n_ring=N, layout=0,
                       causal=True, passes=P, scale=scale)
    o_ref, l_ref = oracle.attention_full(p)
    assert float(np.abs(out.cpu().float().numpy() - o_ref).max()) <= TOL["bf16"][0]
    assert float(np.abs(lse.cpu().numpy() - l_ref).max()) <= TOL["bf16"][1]


def test_gqa_full_size_sampled_rows():
    w = gen.WORKLOADS["bf16_b1_h32_kv4_s32768_d128_causal_n8_contiguous"]
    inp = gen.make_inputs(w)
    out, lse = run_gpu(w, inp)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    heads = (0, 7, 8, w.heads - 1)     # both ends of two key/value groups
    rng = np.random.default_rng(2)
    seqs, hs, rows = sample_rows(w, inp, rng, n_random=128, max_tiles=32, heads=heads)
    check(w, *compare_rows(w, inp, out, lse, seqs, hs, rows, heads))

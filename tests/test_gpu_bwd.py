"""The backward (ring_attn_bwd, CUDA cores, fp32 arithmetic) against the
fp64 oracle's gradients (pinned against torch autograd).

The GPU forward produces out and lse; ring_attn_bwd takes them with a seeded
dout.  Tolerance: max |d grad| <= tol * (1 + max |grad|) with tol 1e-4
(fp32), 2e-2 (bf16), 4e-3 (fp16): the gradients are rounded once to the
input type, and D = <dout, out> inherits the rounding of the 16-bit forward
output, both relative to the gradients' own size.
"""

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
from gpu_util import problem_for

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
BWD_TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 4e-3}

CASES = [
    # (dtype, B, H, H_kv, S, D, causal, N, layout, P)
    ("f32", 1, 2, 2, 256, 64, True, 4, 0, 4),
    ("f32", 1, 2, 1, 200, 32, False, 5, 1, 2),
    ("f32", 1, 1, 1, 128, 16, True, 2, 1, 2),
    ("bf16", 1, 2, 2, 512, 128, True, 4, 1, 4),
    ("bf16", 2, 4, 2, 384, 64, True, 3, 0, 2),
    ("f16", 1, 2, 2, 512, 128, False, 4, 0, 4),
]


def run_bwd(w, inp, dout):
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    B, S, H, D = q.shape
    Hkv = k.shape[2]
    out = torch.empty_like(q)
    lse = torch.empty(B, H, S, device=DEV)
    ra.ring_attn_gqa_fwd(q, k, v, out, lse, B, H, Hkv, S, D, w.n_ring, w.layout, w.causal,
                         w.softmax_scale, w.passes)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ra.ring_attn_bwd(q, k, v, out, lse, dout.to(DEV), dq, dk, dv, B, H, Hkv, S, D, w.n_ring,
                     w.layout, w.causal, w.softmax_scale, w.passes)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    return (dq.cpu().reshape(B * S, H, D), dk.cpu().reshape(B * S, Hkv, D),
            dv.cpu().reshape(B * S, Hkv, D))


def check_grads(w, got, ref):
    tol = BWD_TOL[w.dtype]
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        err = float(np.abs(g.float().numpy() - r).max())
        assert err <= tol * (1.0 + float(np.abs(r).max())), (name, err, float(np.abs(r).max()))


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_oracle(case):
    dt, B, H, Hkv, S, D, causal, N, layout, P = case
    w = gen.Workload("bwd", dt, B, H, S, D, causal, N, layout, P, seed=900 + S, heads_kv=Hkv)
    inp = gen.make_inputs(w)
    g = torch.Generator().manual_seed(901 + S)
    dout = torch.randn(B, S, H, D, generator=g).to(w.torch_dtype)
    got = run_bwd(w, inp, dout)
    ref = oracle.attention_backward(problem_for(w, inp), dout.reshape(B * S, H, D).double().numpy())
    check_grads(w, got, ref)


def test_backward_varlen_matches_oracle():
    lens = [300, 129, 611]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    T, H, Hkv, D, N = int(cu[-1]), 4, 2, 64, 4
    g = torch.Generator().manual_seed(907)
    q = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    dout = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    scale = 1.0 / np.sqrt(D)
    qd, kd, vd, cud = q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV)
    out = torch.empty_like(qd)
    lse = torch.empty(H, T, device=DEV)
    ra.ring_attn_gqa_fwd(qd, kd, vd, out, lse, len(lens), H, Hkv, T, D, N, 0, True, scale, N, cud)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ra.ring_attn_bwd(qd, kd, vd, out, lse, dout.to(DEV), dq, dk, dv, len(lens), H, Hkv, T, D, N,
                     0, True, scale, N, cud)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    p = oracle.Problem(q=q.float().numpy(), k=k.float().numpy(), v=v.float().numpy(),
                       seq_start=cu[:-1].numpy(), seq_len=np.array(lens), n_ring=N, layout=0,
                       causal=True, passes=N, scale=scale)
    ref = oracle.attention_backward(p, dout.double().numpy())
    w = gen.Workload("bwdvl", "bf16", 1, H, T, D, True, N, 0, N, seed=0)
    check_grads(w, (dq.cpu(), dk.cpu(), dv.cpu()), ref)


# The 16-bit cases with d_head 64 or 128 above run on the tensor cores; the
# tests below add a larger case, the CUDA-core cross-check and the masked-key
# invariance of dq.

def test_tensor_core_backward_on_a_multi_tile_case():
    # 4096 tokens: 32 query tiles of 128 rows and 64 key tiles of 64 keys per
    # head, 8 ring blocks, causal striped with a pass cap
    w = gen.Workload("bwd_big", "bf16", 1, 2, 4096, 128, True, 8, 1, 5, seed=930)
    inp = gen.make_inputs(w)
    g = torch.Generator().manual_seed(931)
    dout = torch.randn(1, 4096, 2, 128, generator=g).to(torch.bfloat16)
    got = run_bwd(w, inp, dout)
    ref = oracle.attention_backward(problem_for(w, inp),
                                    dout.reshape(4096, 2, 128).double().numpy())
    check_grads(w, got, ref)


@pytest.mark.parametrize("dt,D,causal,layout,P,Hkv", [
    ("bf16", 128, True, 0, 8, 2), ("f16", 64, False, 1, 3, 1), ("bf16", 64, True, 1, 8, 4)])
def test_tensor_core_backward_agrees_with_cuda_core_kernels(dt, D, causal, layout, P, Hkv):
    w = gen.Workload("bwd_x", dt, 2, 4, 1024, D, causal, 8, layout, P, seed=940 + D,
                     heads_kv=Hkv)
    inp = gen.make_inputs(w)
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    B, S, H, _ = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, H, S, device=DEV)
    ra.ring_attn_gqa_fwd(q, k, v, out, lse, B, H, Hkv, S, D, w.n_ring, w.layout, w.causal,
                         w.softmax_scale, w.passes)
    dout = torch.randn(B, S, H, D, generator=torch.Generator().manual_seed(941)).to(q.dtype)
    dout = dout.to(DEV)
    res = []
    for fn in (ra.ring_attn_bwd, ra.ring_attn_bwd_simt):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fn(q, k, v, out, lse, dout, dq, dk, dv, B, H, Hkv, S, D, w.n_ring, w.layout, w.causal,
           w.softmax_scale, w.passes)
        torch.cuda.synchronize()
        assert ra.ring_attn_status() == ra.RA_OK
        res.append((dq.float(), dk.float(), dv.float()))
    tol = BWD_TOL[dt]
    for a, b in zip(*res):
        assert float((a - b).abs().max()) <= tol * (1.0 + float(b.abs().max()))


def test_dq_of_rows_that_never_see_a_key_block_is_bitwise_unchanged():
    # causal contiguous: rows before the last ring block never see its keys,
    # so overwriting that block's k and v (large finite values) must leave
    # their dq bitwise as it was
    B, H, S, D, N = 1, 2, 2048, 128, 4
    w = gen.Workload("bwd_mask", "bf16", B, H, S, D, True, N, 0, N, seed=950)
    inp = gen.make_inputs(w)
    dout = torch.randn(B, S, H, D, generator=torch.Generator().manual_seed(951))
    dout = dout.to(torch.bfloat16)
    dqs = []
    for poison in (False, True):
        k, v = inp["k"].clone(), inp["v"].clone()
        if poison:
            k[:, 3 * S // 4:] = 1e4
            v[:, 3 * S // 4:] = -1e4
        w_inp = dict(q=inp["q"], k=k, v=v)
        dq, _, _ = run_bwd(w, w_inp, dout)
        dqs.append(dq)
    rows = 3 * S // 4
    assert torch.equal(dqs[0][:rows], dqs[1][:rows])


def test_backward_at_the_benchmark_size_on_two_heads():
    # the benchmark's backward workload (bf16 1x8x8192x128 causal, 8 ring
    # blocks) in the launch configuration bench.py times; the oracle's
    # gradients of the first and last head (a whole head: dk and dv need
    # every query row that sees a key)
    B, H, S, D, N = 1, 8, 8192, 128, 8
    w = gen.Workload("bwd_bench", "bf16", B, H, S, D, True, N, 0, N, seed=960)
    inp = gen.make_inputs(w)
    dout = torch.randn(B, S, H, D, generator=torch.Generator().manual_seed(961))
    dout = dout.to(torch.bfloat16)
    got = run_bwd(w, inp, dout)
    heads = [0, H - 1]
    ref = oracle.attention_backward(problem_for(w, inp, heads=heads),
                                    dout.reshape(S, H, D)[:, heads].double().numpy())
    check_grads(w, tuple(g[:, heads] for g in got), ref)

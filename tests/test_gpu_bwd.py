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

"""The e4m3 (fp8) forward, ring_attn_fwd_fp8, against the fp64 oracle on the
same (dequantised) values.

The inputs are N(0, 1) draws divided by their descale factor and rounded to
e4m3; the oracle receives descale * e4m3 value, exactly.  The kernel rounds P
to e4m3 before P V, which no page fixes a tolerance for, so the bound is
derived per output element from that rounding (tests/test_fp8_rounding.py
pins the rounding model): with p_ij = exp(s_ij - m_i), l_i = sum_j p_ij over
the allowed keys and v the dequantised values,

    |dO_id| <= (2^-4 sum_j p_ij |v_jd| + 2^-10 sum_j |v_jd|) / l_i
               + 2^-8 |O_id| + 1e-4

(relative error <= 2^-4 for P >= 2^-6 and absolute <= 2^-10 below, in units
of the kernel's running reference, which is within 8 log2 units below the
row max so the absolute term only shrinks in units of the max; then the bf16
rounding of the output and fp32 accumulation).  lse uses the unrounded P in
fp32: 1e-3, as for bf16.
"""

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
E4M3 = torch.float8_e4m3fn


def quantize(x, descale):
    return (x / descale).to(E4M3)


def dense_case(B, H, Hkv, S, causal, N, layout, P, scale, dq, dk, dv, seed):
    g = torch.Generator().manual_seed(seed)
    q = quantize(torch.randn(B, S, H, 128, generator=g), dq)
    k = quantize(torch.randn(B, S, Hkv, 128, generator=g), dk)
    v = quantize(torch.randn(B, S, Hkv, 128, generator=g), dv)
    out = torch.empty(B, S, H, 128, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, H, S, device=DEV)
    ra.ring_attn_fwd_fp8(q.to(DEV), k.to(DEV), v.to(DEV), out, lse, B, H, Hkv, S, 128, N,
                         layout, causal, scale, P, None, dq, dk, dv)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    deq = lambda t, d, h: (t.float() * d).numpy().astype(np.float64).reshape(B * S, h, 128)
    prob = oracle.Problem(q=deq(q, dq, H), k=deq(k, dk, Hkv), v=deq(v, dv, Hkv),
                          seq_start=np.arange(B) * S, seq_len=np.full(B, S), n_ring=N,
                          layout=layout, causal=causal, passes=P, scale=scale)
    o = out.cpu().float().numpy().reshape(B * S, H, 128)
    l = lse.cpu().permute(1, 0, 2).reshape(H, B * S).numpy()
    return prob, o, l


def check(prob, o, l):
    o_ref, l_ref = oracle.attention_full(prob)
    assert float(np.abs(l - l_ref).max()) <= 1e-3
    H = prob.q.shape[1]
    Hk = prob.k.shape[1]
    for b in range(len(prob.seq_len)):
        s0, L = int(prob.seq_start[b]), int(prob.seq_len[b])
        if L == 0:
            continue
        mask = oracle.allowed_matrix(L, prob.n_ring, prob.layout, prob.causal, prob.passes)
        for h in range(H):
            hk = oracle.kv_head(h, H, Hk)
            Q, K, V = (prob.q[s0:s0 + L, h], prob.k[s0:s0 + L, hk], prob.v[s0:s0 + L, hk])
            s = np.where(mask, prob.scale * (Q @ K.T), -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            lrow = p.sum(axis=1, keepdims=True)
            av = np.abs(V)
            bound = (2.0 ** -4 * (p @ av) + 2.0 ** -10 * (mask.astype(np.float64) @ av)) / lrow
            ref = o_ref[s0:s0 + L, h]
            bound = bound + 2.0 ** -8 * np.abs(ref) + 1e-4
            err = np.abs(o[s0:s0 + L, h] - ref)
            assert (err <= bound).all(), (b, h, float(err.max()), float((err - bound).max()))


@pytest.mark.parametrize("case", [
    # (B, H, Hkv, S, causal, N, layout, P, scale, dq, dk, dv)
    (1, 2, 2, 1024, False, 4, 0, 4, 128 ** -0.5, 1.0, 1.0, 1.0),
    (1, 2, 2, 2048, True, 8, 1, 3, 128 ** -0.5, 0.5, 2.0, 0.25),
    (2, 4, 2, 640, True, 5, 0, 5, 128 ** -0.5, 1.0, 1.0, 1.0),
    (1, 2, 1, 1000, True, 8, 1, 8, -0.09, 1.0, 1.0, 1.0),
], ids=lambda c: "-".join(map(str, c)))
def test_fp8_forward_within_the_e4m3_bound(case):
    B, H, Hkv, S, causal, N, layout, P, scale, dq, dk, dv = case
    prob, o, l = dense_case(B, H, Hkv, S, causal, N, layout, P, scale, dq, dk, dv, seed=S + H)
    check(prob, o, l)


def test_fp8_varlen_within_the_e4m3_bound():
    lens = [300, 1, 0, 777, 1500]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    T, H, N = int(cu[-1]), 2, 4
    g = torch.Generator().manual_seed(81)
    q, k, v = (quantize(torch.randn(T, H, 128, generator=g), 1.0) for _ in range(3))
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(H, T, device=DEV)
    scale = 128 ** -0.5
    ra.ring_attn_fwd_fp8(q.to(DEV), k.to(DEV), v.to(DEV), out, lse, len(lens), H, H, T, 128, N,
                         0, True, scale, N, cu.to(DEV))
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    f = lambda t: t.float().numpy().astype(np.float64)
    prob = oracle.Problem(q=f(q), k=f(k), v=f(v), seq_start=cu[:-1].numpy(),
                          seq_len=np.array(lens), n_ring=N, layout=0, causal=True, passes=N,
                          scale=scale)
    check(prob, out.cpu().float().numpy(), lse.cpu().numpy())


def test_fp8_rejects_what_it_has_no_kernel_for():
    x = torch.zeros(1, 256, 1, 64, dtype=torch.uint8, device=DEV)
    o = torch.empty(1, 256, 1, 64, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(1, 1, 256, device=DEV)
    with pytest.raises(ra.RingAttnError):           # d_head 64
        ra.ring_attn_fwd_fp8(x, x, x, o, lse, 1, 1, 1, 256, 64, 2)
    x = torch.zeros(1, 256, 1, 128, dtype=torch.uint8, device=DEV)
    o = torch.empty(1, 256, 1, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ra.RingAttnError):           # non-finite descale
        ra.ring_attn_fwd_fp8(x, x, x, o, lse, 1, 1, 1, 256, 128, 2, descale_v=float("inf"))

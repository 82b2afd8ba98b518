"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (max abs error): fp32 inputs 1e-4 on O, 1e-5 on lse; bf16 inputs
2e-2 on O, 1e-3 on lse (fp32 accumulation).  Small cases compare every row;
the full-size workloads, in the launch configuration the benchmark uses,
compare sampled rows (ring-block and tile edges plus random rows).
"""

import itertools

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
from gpu_util import TOL, compare_full, compare_rows, problem_for, run_gpu, sample_rows

pytestmark = pytest.mark.gpu


def check(w, err_o, err_l):
    to, tl = TOL[w.dtype]
    assert err_o <= to and err_l <= tl, (w.name, err_o, err_l)


# ---------------------------------------------------------------- small cases

SMALL = [
    # (dtype, B, H, S, D, causal, N, layout, P)
    ("bf16", 2, 2, 1024, 128, False, 8, 0, 8),
    ("bf16", 1, 3, 1000, 128, True, 8, 0, 8),      # ragged tail, blocks of 125
    ("bf16", 1, 2, 1024, 128, True, 8, 1, 8),
    ("bf16", 1, 2, 1024, 128, True, 8, 1, 3),
    ("bf16", 2, 1, 768, 128, False, 4, 0, 2),
    ("bf16", 1, 2, 1536, 128, True, 16, 1, 4),
    ("bf16", 1, 2, 640, 64, True, 5, 0, 5),
    ("bf16", 1, 1, 384, 64, False, 3, 1, 1),
    ("bf16", 1, 1, 130, 128, True, 2, 0, 2),       # one full tile + 2 rows
    ("bf16", 1, 1, 64, 128, False, 1, 0, 1),       # shorter than a tile
    ("bf16", 1, 2, 512, 128, True, 4, 1, 4, -0.3),  # negative scale
    ("bf16", 1, 1, 256, 64, True, 2, 0, 2, 0.0),    # zero scale: plain average
    ("f32", 1, 2, 1024, 16, False, 16, 0, 16),
    ("f32", 1, 2, 500, 32, True, 5, 1, 2),
    ("f32", 2, 1, 384, 64, True, 3, 0, 3),
    ("f32", 1, 1, 256, 128, True, 4, 1, 4),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_small_all_rows(case):
    dt, B, H, S, D, causal, N, layout, P = case[:9]
    scale = case[9] if len(case) > 9 else None
    w = gen.Workload("small", dt, B, H, S, D, causal, N, layout, P, seed=100 + S, scale=scale)
    inp = gen.make_inputs(w)
    out, lse = run_gpu(w, inp)
    check(w, *compare_full(w, inp, out, lse))


def test_fp32_workload_full():
    w = gen.WORKLOADS["fp32_b1_h1_s1024_d16_noncausal_n16"]
    inp = gen.make_inputs(w)
    out, lse = run_gpu(w, inp)
    check(w, *compare_full(w, inp, out, lse))


@pytest.mark.parametrize("packed", [True, False])
@pytest.mark.parametrize("causal,layout,N,P", [(True, 0, 4, 4), (False, 0, 3, 3),
                                               (True, 1, 4, 2)])
def test_small_varlen_all_rows(packed, causal, layout, N, P):
    lens = [1, 127, 128, 129, 300, 1000, 2, 511]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    T = int(cu[-1])
    w = gen.Workload("varlen_small", "bf16", len(lens), 2, T, 128, causal, N, layout, P,
                     seed=77, varlen=True, packed=packed, n_seqs=len(lens))
    g = torch.Generator().manual_seed(77)
    qkv = torch.randn(T, 3, 2, 128, generator=g).to(torch.bfloat16)
    inp = dict(qkv=qkv, cu_seqlens=cu, q=qkv[:, 0], k=qkv[:, 1], v=qkv[:, 2])
    out, lse = run_gpu(w, inp)
    check(w, *compare_full(w, inp, out, lse))


def test_tensor_core_matches_simt_kernel():
    w = gen.Workload("cross", "bf16", 1, 4, 4096, 128, True, 8, 1, 5, seed=9)
    inp = gen.make_inputs(w)
    o1, l1 = run_gpu(w, inp, "tc")
    o2, l2 = run_gpu(w, inp, "simt")
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2
    assert float((l1 - l2).abs().max()) <= 1e-3


# ---------------------------------------------------------------- full sizes

FULL = [
    "bf16_b2_h16_s8192_d128_noncausal_n8",
    "bf16_b1_h32_s32768_d128_causal_n8_contiguous",
    "bf16_b1_h32_s32768_d128_causal_n8_striped",
    "bf16_varlen_t65536_s16_h16_d128_causal_n4_packed",
    "bf16_b1_h8_s262144_d128_causal_striped_n16_p16",
    "bf16_b1_h8_s262144_d128_causal_striped_n16_p4",
]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w)
    out, lse = run_gpu(w, inp)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    heads = (0, w.heads - 1)
    rng = np.random.default_rng(1)
    seqs, hs, rows = sample_rows(w, inp, rng, n_random=128, max_tiles=32, heads=heads)
    check(w, *compare_rows(w, inp, out, lse, seqs, hs, rows, heads))


def test_striped_equals_contiguous_after_unpermute():
    # the 32K causal workload run in both layouts (inputs permuted into the
    # striped order), compared after un-permuting; sizes reduced to 4 heads
    w = gen.small("bf16_b1_h32_s32768_d128_causal_n8_contiguous", heads=4)
    ws = gen.small("bf16_b1_h32_s32768_d128_causal_n8_striped", heads=4)
    inp = gen.make_inputs(w)
    S, N = w.seqlen, w.n_ring
    pos = np.concatenate([np.arange(r, S, N) for r in range(N)])   # stored -> token
    inp_s = {n: inp[n][:, pos].contiguous() for n in ("q", "k", "v")}
    oc, lc = run_gpu(w, inp)
    os_, ls = run_gpu(ws, inp_s)
    back = torch.empty_like(os_)
    back[pos] = os_
    lback = torch.empty_like(ls)
    lback[:, pos] = ls
    assert float((back.float() - oc.float()).abs().max()) <= 2e-2
    assert float((lback - lc).abs().max()) <= 1e-3


# ---------------------------------------------------------------- bit-exact

def test_masked_keys_do_not_change_results_bitwise():
    """Keys/values a row may not see are overwritten with large finite
    values; that row's O and lse stay bitwise identical."""
    for layout, P in ((0, 8), (1, 8), (1, 3), (0, 2)):
        w = gen.Workload("mask", "bf16", 1, 2, 2048, 128, True, 8, layout, P, seed=5)
        inp = gen.make_inputs(w)
        o1, l1 = run_gpu(w, inp)
        L = w.seqlen
        blk = oracle.ring_block(np.arange(L), L, w.n_ring, layout)
        # rows of query ring block 5 (stored), keys they never see
        rows = np.flatnonzero(blk == 5)
        mask = oracle.allowed(rows[:, None], np.arange(L)[None, :], L, w.n_ring, layout, True, P)
        never = np.flatnonzero(~mask.any(axis=0))
        assert never.size > 0
        inp2 = {n: inp[n].clone() for n in ("q", "k", "v")}
        inp2["k"][:, never] = 1e4
        inp2["v"][:, never] = -1e4
        o2, l2 = run_gpu(w, inp2)
        assert torch.equal(o1[rows], o2[rows])
        assert torch.equal(l1[:, rows], l2[:, rows])


def test_varlen_sequence_alone_is_bitwise_identical():
    lens = [700, 129, 1500, 64]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(T, 3, 2, 128, generator=g).to(torch.bfloat16)
    w = gen.Workload("vl", "bf16", len(lens), 2, T, 128, True, 4, 0, 4, seed=3, varlen=True,
                     packed=True, n_seqs=len(lens))
    out, lse = run_gpu(w, dict(qkv=qkv, cu_seqlens=cu))
    for b, L in enumerate(lens):
        s0 = int(cu[b])
        w1 = gen.Workload("vl1", "bf16", 1, 2, L, 128, True, 4, 0, 4, seed=3, varlen=True,
                          packed=True, n_seqs=1)
        cu1 = torch.tensor([0, L], dtype=torch.int32)
        o1, l1 = run_gpu(w1, dict(qkv=qkv[s0:s0 + L].contiguous(), cu_seqlens=cu1))
        assert torch.equal(out[s0:s0 + L], o1)
        assert torch.equal(lse[:, s0:s0 + L], l1)


@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_varlen_empty_sequences(impl):
    """Zero-length sequences (allowed: cu_seqlens only has to be
    non-decreasing) at the start, in the middle and at the end contribute no
    work: every row matches the oracle, and the result is bit for bit the
    one of the same tokens without the empty sequences."""
    lens = [0, 300, 0, 0, 129, 1, 0]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(12)
    qkv = torch.randn(T, 3, 2, 128, generator=g).to(torch.bfloat16)
    mk = lambda n, c: (gen.Workload("vl_empty", "bf16", n, 2, T, 128, True, 4, 1, 3, seed=12,
                                    varlen=True, packed=impl == "tc", n_seqs=n),
                       dict(qkv=qkv, cu_seqlens=c, q=qkv[:, 0], k=qkv[:, 1], v=qkv[:, 2]))
    w, inp = mk(len(lens), cu)
    out, lse = run_gpu(w, inp, impl=impl)
    check(w, *compare_full(w, inp, out, lse))
    kept = [L for L in lens if L > 0]
    cu2 = torch.zeros(len(kept) + 1, dtype=torch.int32)
    cu2[1:] = torch.cumsum(torch.tensor(kept), 0)
    w2, inp2 = mk(len(kept), cu2)
    out2, lse2 = run_gpu(w2, inp2, impl=impl)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_rows_outside_the_sequences_stay_untouched():
    dev = torch.device("cuda", 0)
    lens = [300, 200]
    T = sum(lens)
    cu = torch.tensor([0, 300, 500], dtype=torch.int32, device=dev)
    g = torch.Generator().manual_seed(4)
    qkv = torch.randn(T, 3, 1, 128, generator=g).to(torch.bfloat16).to(dev)
    pad = 64
    out_big = torch.full((T + pad, 1, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, T, device=dev)
    ra.ring_attn_qkvpacked_fwd(qkv, out_big, lse, 2, 1, T, 128, 4, 0, True, None, 4, cu)
    torch.cuda.synchronize()
    assert torch.isnan(out_big[T:].float()).all()
    assert torch.isfinite(out_big[:T].float()).all()


def test_zero_queries_count_allowed_keys():
    """q = 0: every allowed score is 0 and every P is exactly 1, so lse =
    ln(#allowed keys) up to fp32 rounding, whatever the mask."""
    for layout, causal, P in ((0, True, 8), (1, True, 3), (0, False, 2), (1, False, 8)):
        w = gen.Workload("zero", "bf16", 1, 1, 2048, 128, causal, 8, layout, P, seed=6)
        inp = gen.make_inputs(w)
        inp["q"].zero_()
        _, lse = run_gpu(w, inp)
        L = w.seqlen
        cnt = np.array([oracle.allowed(np.int64(i), np.arange(L), L, 8, layout, causal,
                                       P).sum() for i in range(L)])
        assert np.abs(lse[0].numpy() - np.log(cnt)).max() < 2e-6 * np.log(L) + 1e-6


# ---------------------------------------------------------------- merge

@pytest.mark.parametrize("dtype,D", [(torch.float32, 128), (torch.bfloat16, 128),
                                     (torch.float32, 16), (torch.bfloat16, 64),
                                     (torch.float16, 128), (torch.float16, 32)])
def test_merge_matches_oracle(dtype, D):
    dev = torch.device("cuda", 0)
    B, S, H = 2, 257, 3
    g = torch.Generator().manual_seed(D)
    oa = torch.randn(B, S, H, D, generator=g).to(dtype)
    ob = torch.randn(B, S, H, D, generator=g).to(dtype)
    la = torch.randn(B, H, S, generator=g) * 3
    lb = torch.randn(B, H, S, generator=g) * 3
    la[0, 0, :7] = float("-inf")
    lb[0, 0, 3:9] = float("-inf")
    ref_o, ref_l = oracle.merge(oa.float().numpy().transpose(0, 2, 1, 3), la.numpy(),
                                ob.float().numpy().transpose(0, 2, 1, 3), lb.numpy())
    a_o, a_l = oa.to(dev), la.to(dev)
    ra.ring_attn_merge(a_o, a_l, ob.to(dev), lb.to(dev), B, H, S, D)
    torch.cuda.synchronize()
    got_o = a_o.cpu().float().numpy().transpose(0, 2, 1, 3)
    got_l = a_l.cpu().numpy()
    tol_o = {torch.float32: 1e-5, torch.bfloat16: 2e-2, torch.float16: 4e-3}[dtype]
    assert np.abs(got_o - ref_o).max() <= tol_o
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert np.abs(got_l[fin] - ref_l[fin]).max() <= 1e-5
    # one side empty: the other side comes through bit for bit
    only_b = (la[0, 0] == float("-inf")) & (lb[0, 0] != float("-inf"))
    assert only_b.any()
    assert torch.equal(a_o.cpu()[0, only_b, 0], ob[0, only_b, 0])


def test_merge_of_two_ring_halves_equals_full_ring():
    """Split the key blocks of a non-causal problem into two halves (each half
    computed with the forward on its own keys), merge, compare with the full
    forward and the oracle."""
    dev = torch.device("cuda", 0)
    B, S, H, D, N = 1, 2048, 2, 128, 8
    g = torch.Generator().manual_seed(12)
    q, k, v = (torch.randn(B, S, H, D, generator=g).to(torch.bfloat16) for _ in range(3))
    # forward over each key half: queries attend a key sequence of the same
    # length made of the half's keys repeated twice; the repeat leaves the
    # softmax over the half unchanged and lse shifted by ln 2
    halves = []
    for hsl in (slice(0, S // 2), slice(S // 2, S)):
        kk = torch.cat([k[:, hsl], k[:, hsl]], 1).to(dev)
        vv = torch.cat([v[:, hsl], v[:, hsl]], 1).to(dev)
        o, l = ra.ring_attn_func(q.to(dev), kk, vv, N)
        halves.append((o, l - float(np.log(2.0))))
    (oa, la), (ob, lb) = halves
    oa = oa.float()
    ra.ring_attn_merge(oa, la, ob.float(), lb, B, H, S, D)
    of, lf = ra.ring_attn_func(q.to(dev), k.to(dev), v.to(dev), N)
    torch.cuda.synchronize()
    assert float((oa - of.float()).abs().max()) <= 2e-2
    assert float((la - lf).abs().max()) <= 1e-3


# ---------------------------------------------------------------- status word

def test_bad_cu_seqlens_latch_invalid():
    dev = torch.device("cuda", 0)
    qkv = torch.zeros(256, 3, 1, 128, dtype=torch.bfloat16, device=dev)
    out = torch.empty(256, 1, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, 256, device=dev)
    cu = torch.tensor([0, 200, 100], dtype=torch.int32, device=dev)   # decreasing + wrong total
    ra.ring_attn_qkvpacked_fwd(qkv, out, lse, 2, 1, 256, 128, 2, 0, True, None, 2, cu)
    assert ra.ring_attn_status() == ra.RA_ERR_INVALID
    assert ra.ring_attn_status() == ra.RA_OK        # reading clears it

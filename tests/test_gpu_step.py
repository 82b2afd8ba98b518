"""The key/value-outer ring step (ring_attn_fwd_step) on the GPU against the
fp64 oracle.

A step folds one ring block's keys into the running fp32 (out, lse) of one
ring block's queries.  Folding every block in ring order must reach full
attention (the blockwise result is exact); one step from a given state must
equal the oracle's fold.  Tolerances as for the forward of the input dtype.
"""

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from gpu_util import TOL

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def blocks(x, L, N, layout):
    """[B, L, H, D] -> list of the N ring blocks' rows, each [B, b, H, D]."""
    return [x[:, oracle.block_rows(L, N, layout, r)].contiguous() for r in range(N)]


def draw(B, L, H, D, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, L, H, D, generator=g).to(dtype) for _ in range(3)]


@pytest.mark.parametrize("layout,causal,L,N,D,dt", [
    (0, True, 1024, 4, 128, torch.bfloat16),
    (1, True, 1024, 4, 128, torch.bfloat16),
    (0, False, 1536, 4, 64, torch.bfloat16),     # blocks of 384: a partial second item
    (1, False, 1024, 8, 128, torch.float16),
])
def test_ring_of_steps_reaches_full_attention(layout, causal, L, N, D, dt):
    B, H = 1, 2
    q, k, v = draw(B, L, H, D, 60 + L + D, dt)
    scale = 1.0 / np.sqrt(D)
    qb, kb, vb = (blocks(t, L, N, layout) for t in (q, k, v))
    p = oracle.Problem(q=q[0].float().numpy(), k=k[0].float().numpy(), v=v[0].float().numpy(),
                       seq_start=np.array([0]), seq_len=np.array([L]), n_ring=N, layout=layout,
                       causal=causal, passes=N, scale=scale)
    full_o, full_l = oracle.attention_full(p)
    b = L // N
    tol_o, tol_l = TOL["bf16" if dt == torch.bfloat16 else "f16"]
    for i in range(N):
        out = torch.empty(B, b, H, D, device=DEV)
        lse = torch.empty(B, H, b, device=DEV)
        qi = qb[i].to(DEV)
        for s in range(N):
            j = (i - s) % N
            ra.ring_attn_fwd_step(qi, kb[j].to(DEV), vb[j].to(DEV), out, lse, B, H, L, D, N,
                                  i, j, s > 0, layout, causal, scale)
        torch.cuda.synchronize()
        assert ra.ring_attn_status() == ra.RA_OK
        rows = oracle.block_rows(L, N, layout, i)
        assert float(np.abs(out[0].cpu().numpy() - full_o[rows]).max()) <= tol_o
        assert float(np.abs(lse[0].cpu().numpy() - full_l[:, rows]).max()) <= tol_l


def test_one_step_from_a_running_state_matches_the_oracle_fold():
    B, H, L, N, D, layout = 1, 2, 1024, 4, 128, 1
    q, k, v = draw(B, L, H, D, 71, torch.bfloat16)
    scale = 0.09
    i, j = 2, 3
    qi, kj, vj = (t[:, oracle.block_rows(L, N, layout, r)].contiguous()
                  for t, r in ((q, i), (k, j), (v, j)))
    b = L // N
    g = torch.Generator().manual_seed(72)
    out0 = torch.randn(B, b, H, D, generator=g)
    lse0 = torch.randn(B, H, b, generator=g) * 2
    lse0[0, 0, :17] = float("-inf")          # rows with nothing folded yet
    out0[0, :17, 0] = float("nan")           # their out is not read
    out, lse = out0.clone().to(DEV), lse0.clone().to(DEV)
    ra.ring_attn_fwd_step(qi.to(DEV), kj.to(DEV), vj.to(DEV), out, lse, B, H, L, D, N, i, j,
                          True, layout, True, scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    prev_o = np.nan_to_num(out0[0].numpy(), nan=0.0)
    ref_o, ref_l = oracle.ring_step(qi[0].float().numpy(), kj[0].float().numpy(),
                                    vj[0].float().numpy(), prev_o, lse0[0].numpy(), L, N,
                                    layout, True, scale, i, j)
    got_o, got_l = out[0].cpu().numpy(), lse[0].cpu().numpy()
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert float(np.abs(got_l[fin] - ref_l[fin]).max()) <= TOL["bf16"][1]
    seen = fin.T
    assert float(np.abs(got_o[seen] - ref_o[seen]).max()) <= TOL["bf16"][0]


def test_invisible_block_gives_the_empty_state_or_leaves_it():
    """Causal contiguous: the queries of block 0 see no key of block 2.  A
    fresh step writes the empty state; an accumulating one leaves the
    running state bit for bit."""
    B, H, L, N, D = 1, 2, 1024, 4, 128
    q, k, v = draw(B, L, H, D, 73, torch.bfloat16)
    b = L // N
    qi, kj, vj = q[:, :b].contiguous(), k[:, 2 * b:3 * b].contiguous(), v[:, 2 * b:3 * b].contiguous()
    out = torch.full((B, b, H, D), 7.0, device=DEV)
    lse = torch.full((B, H, b), 3.0, device=DEV)
    ra.ring_attn_fwd_step(qi.to(DEV), kj.to(DEV), vj.to(DEV), out, lse, B, H, L, D, N, 0, 2,
                          False, 0, True, 0.1)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    out2 = torch.randn(B, b, H, D, device=DEV)
    lse2 = torch.randn(B, H, b, device=DEV)
    o_keep, l_keep = out2.clone(), lse2.clone()
    ra.ring_attn_fwd_step(qi.to(DEV), kj.to(DEV), vj.to(DEV), out2, lse2, B, H, L, D, N, 0, 2,
                          True, 0, True, 0.1)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    assert torch.equal(out2, o_keep) and torch.equal(lse2, l_keep)


@pytest.mark.parametrize("i,j,accumulate", [(3, 1, True), (2, 2, False)])
def test_step_whose_last_wave_is_split_matches_the_oracle_fold(i, j, accumulate):
    """A step launch whose items leave the last wave of CTAs at most half
    full splits those items in halves of their key tiles and merges the
    second halves afterwards.  The head count is chosen from the SM count so
    that the launch has whole items and split ones (8 items of 256 query rows
    per head: 2048 rows per ring block)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = -(-(sms + sms // 8) // 8)        # items = 8 H in (sms, 1.5 sms]
    assert 0 < (8 * H) % sms <= sms // 2
    B, N, D, layout = 1, 4, 128, 0
    L = 2048 * N
    q, k, v = draw(B, L, H, D, 74 + i + j, torch.bfloat16)
    scale = 1.0 / np.sqrt(D)
    qi, kj, vj = (t[:, oracle.block_rows(L, N, layout, r)].contiguous()
                  for t, r in ((q, i), (k, j), (v, j)))
    b = L // N
    g = torch.Generator().manual_seed(75)
    out0 = torch.randn(B, b, H, D, generator=g)
    lse0 = torch.randn(B, H, b, generator=g) * 2
    out, lse = out0.clone().to(DEV), lse0.clone().to(DEV)
    ra.ring_attn_fwd_step(qi.to(DEV), kj.to(DEV), vj.to(DEV), out, lse, B, H, L, D, N, i, j,
                          accumulate, layout, True, scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    if accumulate:
        prev_o, prev_l = out0[0].numpy(), lse0[0].numpy()
    else:
        prev_o = np.zeros((b, H, D))
        prev_l = np.full((H, b), -np.inf)
    ref_o, ref_l = oracle.ring_step(qi[0].float().numpy(), kj[0].float().numpy(),
                                    vj[0].float().numpy(), prev_o, prev_l, L, N, layout, True,
                                    scale, i, j)
    got_o, got_l = out[0].cpu().numpy(), lse[0].cpu().numpy()
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert float(np.abs(got_l[fin] - ref_l[fin]).max()) <= TOL["bf16"][1]
    seen = fin.T
    assert float(np.abs(got_o[seen] - ref_o[seen]).max()) <= TOL["bf16"][0]

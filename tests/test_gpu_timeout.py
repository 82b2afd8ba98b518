"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The library's test hook makes the tensor-core forward load no query tile, a
barrier phase that nothing completes.  The MMA warps' wait for Q is bounded
(about one second of SM clock), so the launch must end by itself: every role
unwinds, copies already issued are drained and tensor memory is freed, and
RA_ERR_TIMEOUT is latched in the status word.  The context must stay usable:
the next call, with the hook off, runs on the same SMs (its tensor-memory
allocation succeeds only if the aborted launch freed its own) and matches the
oracle.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
from gpu_util import TOL, compare_full, run_gpu

pytestmark = pytest.mark.gpu

# (dtype, B, H, S, D, causal, N, layout, P): a persistent launch with dynamic
# claiming (non-causal) and a one-CTA-per-item launch (dense causal); both
# have fewer work items than SMs, so every CTA waits at the same time.
CASES = [
    ("bf16", 1, 2, 512, 128, False, 4, 0, 4),
    ("f16", 1, 2, 512, 64, True, 4, 1, 4),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_expired_wait_latches_timeout_and_context_recovers(case):
    dt, B, H, S, D, causal, N, layout, P = case
    w = gen.Workload("timeout", dt, B, H, S, D, causal, N, layout, P, seed=500 + S)
    inp = gen.make_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    out = torch.zeros_like(q)
    lse = torch.zeros(B, H, S, dtype=torch.float32, device=dev)
    assert ra.ring_attn_status() == ra.RA_OK

    prev = ra.ring_attn_test_withhold_q(True)
    try:
        t0 = time.monotonic()
        ra.ring_attn_fwd(q, k, v, out, lse, B, H, S, D, N, layout, causal, w.softmax_scale, P)
        st = ra.ring_attn_status()
        elapsed = time.monotonic() - t0
    finally:
        ra.ring_attn_test_withhold_q(prev)
    assert st == ra.RA_ERR_TIMEOUT, ra.ring_attn_status_string(st)
    # one bound (~1 s at full clock) per CTA, all CTAs resident at once
    assert elapsed < 20.0, elapsed
    # the status word was cleared by the read
    assert ra.ring_attn_status() == ra.RA_OK

    # the same call with the hook off: correct, status clean
    out2, lse2 = run_gpu(w, inp)
    err_o, err_l = compare_full(w, inp, out2, lse2)
    to, tl = TOL[w.dtype]
    assert err_o <= to and err_l <= tl, (err_o, err_l)


def test_cuda_core_kernel_ignores_the_hook():
    # fp32 runs on the CUDA-core kernel, which has no query-load pipeline:
    # the hook changes nothing there
    w = gen.Workload("timeout_f32", "f32", 1, 2, 256, 64, True, 4, 0, 4, seed=31)
    inp = gen.make_inputs(w)
    prev = ra.ring_attn_test_withhold_q(True)
    try:
        out, lse = run_gpu(w, inp)  # asserts RA_OK
    finally:
        ra.ring_attn_test_withhold_q(prev)
    err_o, err_l = compare_full(w, inp, out, lse)
    to, tl = TOL[w.dtype]
    assert err_o <= to and err_l <= tl, (err_o, err_l)


def test_ring_step_unwinds_from_a_loaded_state():
    """An accumulating ring step loads the running state into tensor memory
    before its first wait; with the hook on it must unwind the same way, and
    a whole ring of steps with the hook off must then reach full attention."""
    dev = torch.device("cuda", 0)
    B, H, L, N, D, layout = 1, 2, 1024, 4, 128, 0
    scale = 1.0 / np.sqrt(D)
    g = torch.Generator().manual_seed(41)
    q, k, v = (torch.randn(B, L, H, D, generator=g).to(torch.bfloat16) for _ in range(3))
    blk = [[t[:, oracle.block_rows(L, N, layout, r)].contiguous().to(dev) for r in range(N)]
           for t in (q, k, v)]
    b = L // N
    i = 2
    out = torch.zeros(B, b, H, D, device=dev)
    lse = torch.zeros(B, H, b, device=dev)  # a running state: one unit of weight, O = 0
    prev = ra.ring_attn_test_withhold_q(True)
    try:
        ra.ring_attn_fwd_step(blk[0][i], blk[1][1], blk[2][1], out, lse, B, H, L, D, N, i, 1,
                              True, layout, True, scale)
        st = ra.ring_attn_status()
    finally:
        ra.ring_attn_test_withhold_q(prev)
    assert st == ra.RA_ERR_TIMEOUT, ra.ring_attn_status_string(st)

    for s in range(N):
        j = (i - s) % N
        ra.ring_attn_fwd_step(blk[0][i], blk[1][j], blk[2][j], out, lse, B, H, L, D, N, i, j,
                              s > 0, layout, True, scale)
    assert ra.ring_attn_status() == ra.RA_OK
    p = oracle.Problem(q=q[0].float().numpy(), k=k[0].float().numpy(), v=v[0].float().numpy(),
                       seq_start=np.array([0]), seq_len=np.array([L]), n_ring=N, layout=layout,
                       causal=True, passes=N, scale=scale)
    full_o, full_l = oracle.attention_full(p)
    rows = oracle.block_rows(L, N, layout, i)
    to, tl = TOL["bf16"]
    assert float(np.abs(out[0].cpu().numpy() - full_o[rows]).max()) <= to
    assert float(np.abs(lse[0].cpu().numpy() - full_l[:, rows]).max()) <= tl

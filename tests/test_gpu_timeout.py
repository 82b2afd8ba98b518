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

import pytest
import torch

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

"""Ring-step scheduler (host view of the code the kernels run) against brute
force: the visited (q-tile, kv-tile) pairs are exactly the non-empty ones,
FULL pairs have every element allowed, PARTIAL pairs are mixed, and the
visit order follows the ring (step (r_q - r_k) mod N non-decreasing)."""

import itertools

import numpy as np
import pytest

import oracle
from blockwise_exact_attention_attn_b200 import ring_attn_schedule


def brute(L, N, layout, causal, P, tq, tk):
    mask = oracle.allowed_matrix(L, N, layout, causal, P)
    res = {}
    for a in range(0, L, tq):
        for b in range(0, L, tk):
            sub = mask[a:a + tq, b:b + tk]
            if sub.any():
                res[(a // tq, b // tk)] = 1 if sub.all() else 2
    return res


CASES = [
    # (L, N, tq, tk)
    (512, 4, 128, 128), (1024, 8, 128, 128), (1024, 8, 64, 64), (640, 5, 128, 128),
    (1000, 8, 128, 128), (1000, 4, 256, 128), (300, 3, 128, 64), (96, 16, 32, 32),
    (257, 1, 128, 128), (130, 4, 128, 128),
]


@pytest.mark.parametrize("L,N,tq,tk", CASES)
@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.STRIPED])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_equals_brute_force(L, N, tq, tk, layout, causal):
    for P in sorted({1, 2, max(1, N // 2), N}):
        qt, kt, cl = ring_attn_schedule(L, N, layout, causal, P, tq, tk)
        got = {}
        for a, b, c in zip(qt.tolist(), kt.tolist(), cl.tolist()):
            assert (a, b) not in got, "a kv tile was visited twice"
            got[(a, b)] = c
        assert got == brute(L, N, layout, causal, P, tq, tk)


@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.STRIPED])
@pytest.mark.parametrize("causal", [False, True])
def test_visit_order_is_ring_order(layout, causal):
    # blocks a multiple of both tiles: every tile lies in one ring block
    L, N, T = 2048, 8, 128
    for P in (1, 3, 8):
        qt, kt, _ = ring_attn_schedule(L, N, layout, causal, P, T, T)
        blk = oracle.ring_block(np.arange(L), L, N, layout)
        for q in np.unique(qt):
            ks = kt[qt == q]
            rq = blk[q * T]
            steps = [(rq - blk[k * T]) % N for k in ks]
            assert steps == sorted(steps)
            assert steps[0] == 0          # the own block comes first
            assert max(steps) < P         # never beyond the pass limit


def test_tiny_blocks_are_conservative():
    # 128 ring blocks of 1-2 tokens: beyond the exact regime the scheduler may
    # call an empty/full pair PARTIAL, but never the reverse
    L, N, T = 256, 128, 128
    for layout, causal, P in itertools.product((0, 1), (False, True), (1, 5, 128)):
        qt, kt, cl = ring_attn_schedule(L, N, layout, causal, P, T, T)
        ref = brute(L, N, layout, causal, P, T, T)
        got = {(a, b): c for a, b, c in zip(qt.tolist(), kt.tolist(), cl.tolist())}
        for key, c in ref.items():
            assert key in got                    # no non-empty pair skipped
            if got[key] == 1:
                assert c == 1                    # FULL only when really full


def test_causal_contiguous_skips_future_blocks():
    # causal + contiguous: q-tile i visits exactly kv-tiles 0..i
    L, N, T = 4096, 8, 128
    qt, kt, cl = ring_attn_schedule(L, N, 0, True, N, T, T)
    for q in range(L // T):
        ks = sorted(kt[qt == q].tolist())
        assert ks == list(range(q + 1))
        diag = cl[(qt == q) & (kt == q)]
        assert diag.tolist() == [2]


def test_schedule_rejects_bad_arguments():
    from blockwise_exact_attention_attn_b200 import RingAttnError
    with pytest.raises(RingAttnError):
        ring_attn_schedule(0, 4)
    with pytest.raises(RingAttnError):
        ring_attn_schedule(128, 0)

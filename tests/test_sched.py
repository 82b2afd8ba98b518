"""Ring-step scheduler (host view of the code the kernels run) against brute
force: the visited (q-tile, kv-tile) pairs are exactly the non-empty ones,
FULL pairs have every element allowed, PARTIAL pairs are mixed, and the
visit order follows the ring (step (r_q - r_k) mod N non-decreasing)."""

import itertools

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

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


@pytest.mark.parametrize("per_item", [1, 2])
@pytest.mark.parametrize("L,N,tq,tk", CASES)
@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.STRIPED])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_equals_brute_force(L, N, tq, tk, layout, causal, per_item):
    # per_item 2 is the tensor-core kernel's walk: two q-tiles, one stream
    for P in sorted({1, 2, max(1, N // 2), N}):
        qt, kt, cl = ring_attn_schedule(L, N, layout, causal, P, tq, tk, per_item)
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


def block_pairs(blk, L, a, tq, b, tk):
    """Product of the ring-block index ranges q-tile a and kv-tile b span
    (stored rows are in block order in both layouts; empty blocks inside a
    range, which exist when a sequence is shorter than N, count)."""
    qa, qb = blk[a * tq], blk[min(L, (a + 1) * tq) - 1]
    ka, kb = blk[b * tk], blk[min(L, (b + 1) * tk) - 1]
    return (qb - qa + 1) * (kb - ka + 1)


@settings(max_examples=300, deadline=None)
@given(L=st.integers(1, 600), N=st.integers(1, 20), layout=st.sampled_from([0, 1]),
       causal=st.booleans(), p_extra=st.integers(0, 20),
       tq=st.sampled_from([16, 32, 64, 128]), tk=st.sampled_from([16, 32, 64, 128]),
       per_item=st.sampled_from([1, 2]))
def test_schedule_properties_on_random_geometry(L, N, layout, causal, p_extra, tq, tk,
                                                per_item):
    P = 1 + p_extra % (N + 1)          # 1 .. N+1 (values above N clamp to N)
    qt, kt, cl = ring_attn_schedule(L, N, layout, causal, P, tq, tk, per_item)
    ref = brute(L, N, layout, causal, P, tq, tk)
    mask = oracle.allowed_matrix(L, N, layout, causal, P)
    blk = oracle.ring_block(np.arange(L), L, N, layout)
    got = {}
    for a, b, c in zip(qt.tolist(), kt.tolist(), cl.tolist()):
        assert (a, b) not in got, "a kv tile was visited twice"
        assert c in (1, 2)
        got[(a, b)] = c
    for key in ref:
        assert key in got, ("non-empty pair skipped", key)
    for (a, b), c in got.items():
        sub = mask[a * tq:(a + 1) * tq, b * tk:(b + 1) * tk]
        if c == 1:
            assert sub.all(), ("false FULL", a, b)
        if block_pairs(blk, L, a, tq, b, tk) <= 64:
            assert ref.get((a, b)) == c, ("inexact class in the exact regime", a, b)
    # ring order: per q-tile, the step of each visited kv tile (block of its
    # first key, relative to the block of the item's first row) never falls
    for a in np.unique(qt):
        item0 = (a // per_item) * per_item * tq
        steps = [(blk[item0] - blk[b * tk]) % N for b in kt[qt == a]]
        assert steps == sorted(steps)

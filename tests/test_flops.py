"""FLOP accounting of the benchmark (closed forms per ring-block pair) against
the oracle's enumeration of allowed pairs."""

import itertools

import pytest

import oracle
from blockwise_exact_attention_attn_b200.flops import allowed_pairs, forward_flops


@pytest.mark.parametrize("L,N", [(64, 4), (100, 8), (37, 5), (256, 16), (12, 12), (5, 8)])
def test_pairs_match_enumeration(L, N):
    for layout, causal in itertools.product((0, 1), (False, True)):
        for P in sorted({1, 2, N // 2 or 1, N}):
            assert allowed_pairs(L, N, layout, causal, P) == \
                oracle.unmasked_pairs(L, N, layout, causal, P)


def test_workload_flops_closed_forms():
    # non-causal 2x16x8192x128: 4 * S^2 * D * H * B
    assert forward_flops([8192] * 2, 16, 128, 8, 0, False, 8) == 4.0 * 8192**2 * 128 * 16 * 2
    # causal 32K, any layout: S(S+1)/2 pairs per head
    for layout in (0, 1):
        assert forward_flops([32768], 32, 128, 8, layout, True, 8) == \
            4.0 * 32768 * 32769 // 2 * 128 * 32
    # striped causal N=16, P=4, b=16384: 32 b^2 + 26 b pairs per head
    b = 16384
    assert forward_flops([16 * b], 8, 128, 16, 1, True, 4) == 4.0 * (32 * b * b + 26 * b) * 128 * 8


@pytest.mark.parametrize("L,N,layout,causal,P", [
    (64, 4, 0, False, 4), (100, 8, 1, True, 3), (37, 5, 0, True, 5), (96, 16, 1, True, 4)])
def test_oracle_row_flops_sum_to_the_workload_flops(L, N, layout, causal, P):
    # the CPU baseline's FLOP count (oracle.row_flops over every row) equals
    # the benchmark's closed form for the whole sequence
    import numpy as np
    D = 16
    p = oracle.Problem(q=np.zeros((L, 1, D)), k=np.zeros((L, 1, D)), v=np.zeros((L, 1, D)),
                       seq_start=np.array([0]), seq_len=np.array([L]), n_ring=N, layout=layout,
                       causal=causal, passes=P, scale=1.0)
    rows = np.arange(L)
    got = oracle.row_flops(p, np.zeros(L, dtype=np.int64), np.zeros(L, dtype=np.int64), rows)
    assert got == forward_flops([L], 1, D, N, layout, causal, P)

"""Algorithmic work of one forward call, for throughput reporting.

FLOPs = 4 * (allowed query/key pairs) * d_head * heads, summed over the
sequences (2 for Q K^T and 2 for P V per pair), counting only the pairs the
mask allows.  Pairs are counted per (query block, key block) of the ring with
closed forms over token ranges.
"""

from __future__ import annotations

import numpy as np


def _blocks(L: int, N: int, layout: int):
    """Per ring block: (first token, token stride, count)."""
    out = []
    if layout == 0:
        for r in range(N):
            a = -(-r * L // N)
            b = -(-(r + 1) * L // N)
            out.append((a, 1, max(0, b - a)))
    else:
        for r in range(N):
            out.append((r, N, max(0, (L - r + N - 1) // N)))
    return out


def allowed_pairs(L: int, N: int, layout: int, causal: bool, P: int) -> int:
    """Allowed (query, key) pairs of one sequence of length L."""
    P = min(P, N)
    blocks = _blocks(L, N, layout)
    total = 0
    for rq in range(N):
        t0q, sq, nq = blocks[rq]
        if nq == 0:
            continue
        for step in range(P):
            rk = (rq - step) % N
            t0k, sk, nk = blocks[rk]
            if nk == 0:
                continue
            if not causal:
                total += nq * nk
                continue
            # keys of block rk with token <= token of each query of block rq
            qt = t0q + sq * np.arange(nq, dtype=np.int64)
            cnt = np.floor_divide(qt - t0k, sk) + 1
            total += int(np.clip(cnt, 0, nk).sum())
    return total


def forward_flops(seq_lens, heads: int, d_head: int, N: int, layout: int, causal: bool,
                  P: int) -> float:
    pairs = sum(allowed_pairs(int(L), N, layout, causal, P) for L in seq_lens)
    return 4.0 * pairs * d_head * heads

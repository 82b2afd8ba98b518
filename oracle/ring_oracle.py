"""fp64 CPU oracle for blockwise exact ("ring") attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  It shares no
code with the CUDA library (it does not import the package, and the package
does not import it).  Inputs reach both sides from the seeded generators only.

What it computes is the plain definition, not the blockwise method: the pages
state that the ring/blockwise evaluation reaches exactly full softmax attention
("Ring Attention" glossary, "Come funziona la ring attention": the four-device
simulation shows the result is exact; "Ring Attention simulation" gist: the
ring output is compared with softmax(q k^T) v).  So, for one query row i with
allowed key set A(i):

    s_j   = scale * <q_i, k_j>            (fp64, j in A(i))
    m     = max_j s_j
    l     = sum_j exp(s_j - m)
    O_i   = sum_j exp(s_j - m) v_j / l
    lse_i = m + ln(l)

The subtraction of the row maximum is the shift invariance of softmax
("Attention的分块计算" blog, "局部softmax和全局softmax之间的关系": subtracting the
maximum leaves softmax unchanged and keeps exp in range).

The allowed set A(i) follows the ring geometry.  Where the pages leave a step
open, the plainest reading consistent with them is taken:
  * contiguous layout: token t sits in ring block floor(t*N/L);
  * striped layout: ring block r holds tokens r, r+N, r+2N, ... ("Ring
    Attention" glossary: Striped Attention spreads each device's tokens evenly
    over the sequence), stored block after block;
  * causal compares ORIGINAL token positions;
  * max ring passes P: query block r sees key blocks r, r-1, ..., r-P+1
    (mod N) -- its own block and the P-1 blocks that reach it first in the
    ring ("Ring Attention" glossary ring step: the block held at step s came
    from the previous device, j = (i - step) mod N; issue thread "A ring
    attention with flash attention kernel implementation": the maximum number
    of ring passes).

Merge of two partial results (issue thread above: the returned lse is what
lets blockwise results be combined) is the log-add-exp of the two lse values
with each output weighted by exp(lse_side - lse).

Every function here is pinned by tests in ``tests/test_oracle.py`` against
facts the pages and mathematics fix (worked examples, closed-form counts,
brute force, library special cases).
"""

from __future__ import annotations

import os
import time
from dataclasses import dataclass

import numpy as np

CONTIGUOUS = 0
STRIPED = 1


# --------------------------------------------------------------------------
# Ring geometry of one sequence (stored index -> ring block, original token)
# --------------------------------------------------------------------------

def striped_block_sizes(L: int, N: int) -> np.ndarray:
    """Tokens per ring block in the striped layout: block r holds the tokens
    t < L with t mod N == r, so it has ceil((L - r) / N) of them (0 when
    r >= L)."""
    r = np.arange(N, dtype=np.int64)
    return np.maximum(0, (L - r + N - 1) // N)


def ring_block(t, L: int, N: int, layout: int) -> np.ndarray:
    """Ring block of stored row(s) t of a sequence of length L."""
    t = np.asarray(t, dtype=np.int64)
    if layout == CONTIGUOUS:
        return (t * N) // L
    sizes = striped_block_sizes(L, N)
    starts = np.concatenate([[0], np.cumsum(sizes)])
    # the block whose stored range [starts[r], starts[r+1]) contains t
    return np.searchsorted(starts, t, side="right") - 1


def token_pos(t, L: int, N: int, layout: int) -> np.ndarray:
    """Original token index of stored row(s) t."""
    t = np.asarray(t, dtype=np.int64)
    if layout == CONTIGUOUS:
        return t.copy()
    sizes = striped_block_sizes(L, N)
    starts = np.concatenate([[0], np.cumsum(sizes)])
    r = np.searchsorted(starts, t, side="right") - 1
    local = t - starts[r]
    return local * N + r


def allowed(tq, tk, L: int, N: int, layout: int, causal: bool, P: int) -> np.ndarray:
    """A(i) membership for stored query rows tq and stored key rows tk of the
    same sequence (broadcasting)."""
    tq = np.asarray(tq, dtype=np.int64)
    tk = np.asarray(tk, dtype=np.int64)
    ok = np.ones(np.broadcast(tq, tk).shape, dtype=bool)
    if causal:
        ok &= token_pos(tk, L, N, layout) <= token_pos(tq, L, N, layout)
    passes = min(P, N)
    if passes < N:
        d = (ring_block(tq, L, N, layout) - ring_block(tk, L, N, layout)) % N
        ok &= d < passes
    return ok


def allowed_matrix(L: int, N: int, layout: int, causal: bool, P: int) -> np.ndarray:
    """Dense [L, L] boolean A(i) for small L."""
    t = np.arange(L, dtype=np.int64)
    return allowed(t[:, None], t[None, :], L, N, layout, causal, P)


# --------------------------------------------------------------------------
# The definition: masked softmax attention in fp64
# --------------------------------------------------------------------------

def masked_attention(q, k, v, mask, scale: float):
    """softmax(scale * q k^T restricted to mask) v and lse, fp64, two-pass.

    q: [Sq, D], k, v: [Sk, D], mask: [Sq, Sk] bool.  Rows with an empty mask
    get O = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe[:, None])            # exp(-inf) = 0 on masked keys
    l = e.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        o = (e @ v) / l[:, None]
        lse = m_safe + np.log(l)
    o[empty] = 0.0
    lse[empty] = -np.inf
    return o, lse


def kv_head(h, heads: int, heads_kv: int):
    """Key/value head read by query head h.

    Grouped-query and multi-query attention ("Tensorflow flash attention"
    page: several query heads attend to one key/value head) -- the page does
    not say which query heads share; the reading taken is consecutive groups
    of heads / heads_kv query heads per key/value head (heads_kv == heads is
    ordinary multi-head attention, heads_kv == 1 multi-query)."""
    if heads_kv < 1 or heads % heads_kv != 0:
        raise ValueError("heads must be a multiple of heads_kv")
    return h // (heads // heads_kv)


@dataclass
class Problem:
    """One forward call: q is a float array [T, H, D] over all tokens of all
    sequences, k and v are [T, H_kv, D] with H a multiple of H_kv (bf16 inputs
    are passed upcast, exactly)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    seq_start: np.ndarray   # [B] first stored row of each sequence
    seq_len: np.ndarray     # [B]
    n_ring: int
    layout: int
    causal: bool
    passes: int
    scale: float


def attention_rows(p: Problem, seq, head, row, chunk: int = 64):
    """O and lse (fp64) for the listed (sequence, head, stored row) triples.

    Rows are grouped by (sequence, head); each group multiplies its rows
    against that sequence's keys (a library matmul) and applies the
    definition above.
    """
    seq = np.asarray(seq, dtype=np.int64)
    head = np.asarray(head, dtype=np.int64)
    row = np.asarray(row, dtype=np.int64)
    n = seq.shape[0]
    D = p.q.shape[2]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    keys = seq * (p.q.shape[1] + 1) + head
    order = np.argsort(keys, kind="stable")
    bounds = np.flatnonzero(np.diff(keys[order])) + 1
    for grp in np.split(order, bounds):
        if grp.size == 0:
            continue
        b, h = int(seq[grp[0]]), int(head[grp[0]])
        s0, L = int(p.seq_start[b]), int(p.seq_len[b])
        hk = kv_head(h, p.q.shape[1], p.k.shape[1])
        K = p.k[s0:s0 + L, hk, :].astype(np.float64)
        V = p.v[s0:s0 + L, hk, :].astype(np.float64)
        tk = np.arange(L, dtype=np.int64)
        for c in range(0, grp.size, chunk):
            idx = grp[c:c + chunk]
            tq = row[idx]
            Q = p.q[s0 + tq, h, :].astype(np.float64)
            mask = allowed(tq[:, None], tk[None, :], L, p.n_ring, p.layout,
                           p.causal, p.passes)
            o, ls = masked_attention(Q, K, V, mask, p.scale)
            out[idx] = o
            lse[idx] = ls
    return out, lse


def attention_full(p: Problem):
    """Every row: returns O [T, H, D] and lse [H, T] (token-major rows)."""
    T, H, D = p.q.shape
    out = np.zeros((T, H, D), dtype=np.float64)
    lse = np.zeros((H, T), dtype=np.float64)
    for b in range(len(p.seq_len)):
        s0, L = int(p.seq_start[b]), int(p.seq_len[b])
        for h in range(H):
            rows = np.arange(L, dtype=np.int64)
            o, ls = attention_rows(p, np.full(L, b), np.full(L, h), rows, chunk=256)
            out[s0:s0 + L, h, :] = o
            lse[h, s0:s0 + L] = ls
    return out, lse


# --------------------------------------------------------------------------
# Merge of partial results
# --------------------------------------------------------------------------

def merge(out_a, lse_a, out_b, lse_b):
    """(out, lse) of the union of two disjoint key sets, fp64.

    lse = max + log1p(exp(min - max)); each side weighted by exp(lse_side -
    lse).  Both sides empty (-inf) give lse = -inf, out = 0; one side empty
    returns the other side unchanged.
    """
    oa = np.asarray(out_a, dtype=np.float64)
    ob = np.asarray(out_b, dtype=np.float64)
    la = np.asarray(lse_a, dtype=np.float64)
    lb = np.asarray(lse_b, dtype=np.float64)
    hi = np.maximum(la, lb)
    lo = np.minimum(la, lb)
    both_empty = ~np.isfinite(hi)
    a_empty = ~np.isfinite(la)
    b_empty = ~np.isfinite(lb)
    with np.errstate(invalid="ignore", over="ignore"):
        lse = hi + np.log1p(np.exp(lo - hi))
        wa = np.exp(la - lse)
        wb = np.exp(lb - lse)
    out = wa[..., None] * oa + wb[..., None] * ob
    out = np.where(a_empty[..., None], ob, out)
    out = np.where(b_empty[..., None], oa, out)
    lse = np.where(a_empty, lb, np.where(b_empty, la, lse))
    out = np.where(both_empty[..., None], 0.0, out)
    lse = np.where(both_empty, -np.inf, lse)
    return out, lse


def block_rows(L: int, N: int, layout: int, r: int) -> np.ndarray:
    """Stored indices of ring block r of a sequence of length L."""
    t = np.arange(L, dtype=np.int64)
    return np.flatnonzero(ring_block(t, L, N, layout) == r)


def ring_step(q, k, v, out_prev, lse_prev, L: int, N: int, layout: int, causal: bool,
              scale: float, q_block: int, kv_block: int):
    """One key/value-outer ring step, fp64: the queries of ring block q_block
    fold the keys of ring block kv_block into their running result.

    The issue thread "A ring attention with flash attention kernel
    implementation" notes that with keys and values on the outer loop the
    reduced outputs and lse of the queries are stored and passed back in on
    the next ring pass; the fold is the merge above of the running result
    with attention over the new block's keys.

    q: [nq, H, D] rows of block q_block in stored order; k, v: [nk, H, D]
    rows of block kv_block; out_prev [nq, H, D] and lse_prev [H, nq] the
    running normalised output and lse (lse = -inf: nothing folded yet).  The
    mask is the sequence's (causal in original positions); no pass limit
    applies, the caller chooses the blocks.  Returns (out, lse) in the same
    shapes.
    """
    tq = block_rows(L, N, layout, q_block)
    tk = block_rows(L, N, layout, kv_block)
    mask = allowed(tq[:, None], tk[None, :], L, N, layout, causal, N)
    H = q.shape[1]
    o_new = np.zeros(np.shape(q), dtype=np.float64)
    l_new = np.zeros((H, tq.size), dtype=np.float64)
    for h in range(H):
        o_new[:, h, :], l_new[h] = masked_attention(q[:, h, :], k[:, h, :], v[:, h, :], mask,
                                                    scale)
    out, lse = merge(np.transpose(out_prev, (1, 0, 2)), lse_prev,
                     np.transpose(o_new, (1, 0, 2)), l_new)
    return np.transpose(out, (1, 0, 2)), lse


def attention_backward(p: Problem, dout):
    """Gradients (dq, dk, dv) of sum(dout * O) for the forward of p, fp64,
    from the plain definition, one (sequence, head) at a time.

    The pages stop at the forward; the issue thread "A ring attention with
    flash attention kernel implementation" notes that the backward is where
    an implementation went wrong and that the returned lse is what the
    blockwise method keeps.  The gradient itself is plain calculus on
    O_i = sum_j P_ij v_j with P_ij = exp(s_ij - lse_i), s_ij = scale <q_i, k_j>
    over the allowed keys:
        dV_j = sum_i P_ij dO_i
        dP_ij = <dO_i, v_j>,   D_i = <dO_i, O_i> = sum_j P_ij dP_ij
        dS_ij = P_ij (dP_ij - D_i)
        dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
    dout has q's shape [T, H, D]; k and v may have fewer heads (grouped
    queries), their gradients summing over the query heads that share them.
    """
    q = np.asarray(p.q, dtype=np.float64)
    k = np.asarray(p.k, dtype=np.float64)
    v = np.asarray(p.v, dtype=np.float64)
    do = np.asarray(dout, dtype=np.float64)
    T, H, D = q.shape
    Hk = k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(len(p.seq_len)):
        s0, L = int(p.seq_start[b]), int(p.seq_len[b])
        mask = allowed_matrix(L, p.n_ring, p.layout, p.causal, p.passes)
        for h in range(H):
            hk = kv_head(h, H, Hk)
            Q, K, V = q[s0:s0 + L, h], k[s0:s0 + L, hk], v[s0:s0 + L, hk]
            dO = do[s0:s0 + L, h]
            s = np.where(mask, p.scale * (Q @ K.T), -np.inf)
            m = s.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            e = np.exp(s - m)
            P = e / e.sum(axis=1, keepdims=True)
            O = P @ V
            dP = dO @ V.T
            Dd = (dO * O).sum(axis=1, keepdims=True)
            dS = P * (dP - Dd)
            dq[s0:s0 + L, h] = p.scale * (dS @ K)
            dk[s0:s0 + L, hk] += p.scale * (dS.T @ Q)
            dv[s0:s0 + L, hk] += P.T @ dO
    return dq, dk, dv


# --------------------------------------------------------------------------
# Helpers for tests and the CPU baseline
# --------------------------------------------------------------------------

def unmasked_pairs(L: int, N: int, layout: int, causal: bool, P: int,
                   chunk: int = 4096) -> int:
    """Number of allowed (query, key) pairs of one sequence, by enumeration
    (chunked rows, so it works for long sequences)."""
    tk = np.arange(L, dtype=np.int64)
    total = 0
    for r0 in range(0, L, chunk):
        tq = np.arange(r0, min(L, r0 + chunk), dtype=np.int64)
        total += int(allowed(tq[:, None], tk[None, :], L, N, layout, causal, P).sum())
    return total


def blas_threads() -> int:
    """Threads the BLAS behind numpy uses (reported as the CPU baseline's
    core count)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info()
             if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def timed_rows(p: Problem, seq, head, row):
    """attention_rows with wall time (seconds) -- used by the CPU baseline."""
    t0 = time.perf_counter()
    o, lse = attention_rows(p, seq, head, row)
    return o, lse, time.perf_counter() - t0


def row_flops(p: Problem, seq, head, row) -> float:
    """Unmasked FLOPs (4 * D per allowed pair) of the listed rows."""
    D = p.q.shape[2]
    total = 0
    for b, r in zip(np.asarray(seq), np.asarray(row)):
        L = int(p.seq_len[int(b)])
        tk = np.arange(L, dtype=np.int64)
        total += int(allowed(np.int64(r), tk, L, p.n_ring, p.layout,
                             p.causal, p.passes).sum())
    return 4.0 * D * total


__all__ = [
    "CONTIGUOUS", "STRIPED", "Problem", "allowed", "allowed_matrix", "attention_backward",
    "block_rows",
    "attention_full", "attention_rows", "blas_threads", "masked_attention",
    "merge", "ring_block", "ring_step", "row_flops", "striped_block_sizes", "timed_rows",
    "kv_head", "token_pos", "unmasked_pairs",
]

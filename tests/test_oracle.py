"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: the pages'
worked examples (re-enacted from their description, fixtures in
tests/golden/), a library routine on a special case (torch SDPA / logsumexp
in fp64), brute force with an independently built mask, closed-form counts,
and algebraic invariants of the blockwise method (ring order, permutation,
merge).
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from blockwise_exact_attention_attn_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TIGHT = 1e-12


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# Independent geometry: stored order built by explicit enumeration
# ----------------------------------------------------------------------------

def explicit_geometry(L, N, layout):
    """(pos, blk) per stored row, built from first principles:
    contiguous -- blocks are consecutive runs, block r holding the tokens t
    with r*L <= t*N < (r+1)*L; striped -- ring block r collects the tokens
    t with t % N == r in increasing order, blocks concatenated 0..N-1."""
    if layout == oracle.CONTIGUOUS:
        pos = list(range(L))
        blk = []
        for t in range(L):
            r = 0
            while not (r * L <= t * N < (r + 1) * L):
                r += 1
            blk.append(r)
        return np.array(pos), np.array(blk)
    pos, blk = [], []
    for r in range(N):
        for t in range(L):
            if t % N == r:
                pos.append(t)
                blk.append(r)
    return np.array(pos), np.array(blk)


def explicit_mask(L, N, layout, causal, P):
    pos, blk = explicit_geometry(L, N, layout)
    m = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for j in range(L):
            ok = True
            if causal and pos[j] > pos[i]:
                ok = False
            if (blk[i] - blk[j]) % N >= min(P, N):
                ok = False
            m[i, j] = ok
    return m


def problem(q, k, v, N, layout, causal, P, scale, starts=None, lens=None):
    T = q.shape[0]
    return oracle.Problem(q=q, k=k, v=v,
                          seq_start=np.array(starts if starts is not None else [0]),
                          seq_len=np.array(lens if lens is not None else [T]),
                          n_ring=N, layout=layout, causal=causal, passes=P, scale=scale)


# ----------------------------------------------------------------------------
# Geometry and mask
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("L,N", [(8, 4), (12, 3), (10, 4), (7, 3), (5, 8), (64, 16)])
@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.STRIPED])
def test_geometry_matches_explicit_construction(L, N, layout):
    pos, blk = explicit_geometry(L, N, layout)
    t = np.arange(L)
    assert np.array_equal(oracle.token_pos(t, L, N, layout), pos)
    assert np.array_equal(oracle.ring_block(t, L, N, layout), blk)


@pytest.mark.parametrize("L,N", [(32, 4), (1024, 16), (64, 8)])
def test_contiguous_blocks_are_the_pages_chunks(L, N):
    # divisible case: the pages split the sequence into N equal consecutive
    # chunks (glossary demo: q.chunk(n_devices); gist: [i*chunk:(i+1)*chunk])
    blk = oracle.ring_block(np.arange(L), L, N, oracle.CONTIGUOUS)
    assert np.array_equal(blk, np.repeat(np.arange(N), L // N))


@pytest.mark.parametrize("L,N", [(10, 4), (1000, 7), (4097, 4), (3, 5)])
def test_contiguous_blocks_balanced_when_not_divisible(L, N):
    blk = oracle.ring_block(np.arange(L), L, N, oracle.CONTIGUOUS)
    assert np.all(np.diff(blk) >= 0)                     # consecutive runs
    sizes = np.bincount(blk, minlength=N)
    assert sizes.sum() == L and sizes.max() - sizes.min() <= 1


def test_striped_token_t_in_block_t_mod_n():
    L, N = 37, 5
    pos = oracle.token_pos(np.arange(L), L, N, oracle.STRIPED)
    blk = oracle.ring_block(np.arange(L), L, N, oracle.STRIPED)
    assert sorted(pos.tolist()) == list(range(L))
    assert np.array_equal(blk, pos % N)


@pytest.mark.parametrize("L,N", [(12, 4), (12, 3), (10, 4), (9, 2), (11, 1)])
@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.STRIPED])
@pytest.mark.parametrize("causal", [False, True])
def test_mask_matches_explicit(L, N, layout, causal):
    for P in range(1, N + 1):
        assert np.array_equal(oracle.allowed_matrix(L, N, layout, causal, P),
                              explicit_mask(L, N, layout, causal, P))


# ----------------------------------------------------------------------------
# Closed-form counts of allowed pairs
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("L,N", [(64, 4), (96, 8), (100, 5)])
@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.STRIPED])
def test_counts_noncausal_and_causal(L, N, layout):
    assert oracle.unmasked_pairs(L, N, layout, False, N) == L * L
    # causal over original positions: L(L+1)/2 whatever the stored order
    assert oracle.unmasked_pairs(L, N, layout, True, N) == L * (L + 1) // 2


@pytest.mark.parametrize("b", [4, 8, 16])
def test_counts_striped_causal_pass_limited(b):
    # N = 16, P = 4, striped, causal: own block plus three preceding ring
    # blocks; block pairs (r_q, r_q - s) with r_q - s >= 0 hold b(b+1)/2
    # allowed pairs, wrapped ones b(b-1)/2 -> 58*b(b+1)/2 + 6*b(b-1)/2
    N, P = 16, 4
    assert oracle.unmasked_pairs(N * b, N, oracle.STRIPED, True, P) == 32 * b * b + 26 * b


@pytest.mark.parametrize("N,P", [(4, 1), (4, 2), (8, 3)])
def test_counts_contiguous_pass_limited(N, P):
    # non-causal contiguous with P < N: every query sees exactly P blocks
    b = 6
    L = N * b
    assert oracle.unmasked_pairs(L, N, oracle.CONTIGUOUS, False, P) == L * P * b


def test_zero_queries_give_log_count_and_mean():
    # q = 0: every allowed score is 0, so lse = ln|A(i)| and O = mean of v_j
    rng = np.random.default_rng(7)
    L, N, D = 48, 6, 5
    q = np.zeros((L, 1, D), dtype=np.float32)
    k = rng.standard_normal((L, 1, D)).astype(np.float32)
    v = rng.standard_normal((L, 1, D)).astype(np.float32)
    for layout, causal, P in itertools.product((0, 1), (False, True), (1, 3, 6)):
        p = problem(q, k, v, N, layout, causal, P, 0.3)
        o, lse = oracle.attention_full(p)
        mask = explicit_mask(L, N, layout, causal, P)
        cnt = mask.sum(axis=1)
        assert np.allclose(lse[0], np.log(cnt), atol=TIGHT, rtol=0)
        mean = (mask.astype(np.float64) @ v[:, 0, :].astype(np.float64)) / cnt[:, None]
        assert np.allclose(o[:, 0, :], mean, atol=TIGHT, rtol=0)


# ----------------------------------------------------------------------------
# Library special case: torch SDPA / logsumexp in fp64
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P", [1, 2, 4])
def test_core_definition_vs_torch_sdpa(layout, causal, P):
    L, N, H, D = 24, 4, 2, 8
    g = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(L, H, D, generator=g, dtype=torch.float64) for _ in range(3))
    scale = 0.37
    p = problem(q.numpy(), k.numpy(), v.numpy(), N, layout, causal, P, scale)
    o, lse = oracle.attention_full(p)
    mask = torch.from_numpy(explicit_mask(L, N, layout, causal, P))
    for h in range(H):
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, h][None], k[:, h][None], v[:, h][None], attn_mask=mask[None], scale=scale)[0]
        s = scale * (q[:, h] @ k[:, h].T)
        s = s.masked_fill(~mask, float("-inf"))
        ref_lse = torch.logsumexp(s, dim=-1)
        assert np.abs(o[:, h] - ref.numpy()).max() < TIGHT
        assert np.abs(lse[h] - ref_lse.numpy()).max() < TIGHT


@pytest.mark.parametrize("H,Hkv", [(4, 2), (4, 1), (6, 3), (3, 3)])
@pytest.mark.parametrize("layout,causal,P", [(0, True, 4), (1, True, 2), (0, False, 3)])
def test_grouped_query_heads_vs_torch_sdpa(H, Hkv, layout, causal, P):
    """Grouped-query / multi-query attention: query head h reads key/value
    head h // (H / Hkv).  Pinned against torch's own grouped-query SDPA
    (enable_gqa), fp64."""
    L, N, D = 20, 4, 6
    g = torch.Generator().manual_seed(17)
    q = torch.randn(L, H, D, generator=g, dtype=torch.float64)
    k = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64)
    scale = 0.41
    p = problem(q.numpy(), k.numpy(), v.numpy(), N, layout, causal, P, scale)
    o, _ = oracle.attention_full(p)
    mask = torch.from_numpy(explicit_mask(L, N, layout, causal, P))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None],
        attn_mask=mask[None, None], scale=scale, enable_gqa=True)[0].permute(1, 0, 2)
    assert np.abs(o - ref.numpy()).max() < TIGHT


def test_grouped_query_zero_queries_give_group_means():
    # q = 0 with 2 key/value heads for 4 query heads: lse = ln|A(i)| and O is
    # the mean of the allowed values of the shared head
    rng = np.random.default_rng(9)
    L, N, D, H, Hkv = 30, 5, 3, 4, 2
    q = np.zeros((L, H, D))
    k = rng.standard_normal((L, Hkv, D))
    v = rng.standard_normal((L, Hkv, D))
    p = problem(q, k, v, N, 1, True, 3, 0.5)
    o, lse = oracle.attention_full(p)
    mask = explicit_mask(L, N, 1, True, 3)
    cnt = mask.sum(axis=1)
    for h in range(H):
        assert np.allclose(lse[h], np.log(cnt), atol=TIGHT, rtol=0)
        mean = (mask.astype(np.float64) @ v[:, h // 2, :]) / cnt[:, None]
        assert np.allclose(o[:, h, :], mean, atol=TIGHT, rtol=0)
    with pytest.raises(ValueError):
        oracle.kv_head(0, 4, 3)


# ----------------------------------------------------------------------------
# Backward: gradients against torch autograd (fp64)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout,causal,P,H,Hkv", [(0, True, 4, 2, 2), (1, True, 2, 2, 2),
                                                   (0, False, 3, 4, 2), (1, False, 4, 3, 1)])
def test_backward_matches_torch_autograd(layout, causal, P, H, Hkv):
    L, N, D = 20, 4, 6
    g = torch.Generator().manual_seed(31)
    q = torch.randn(L, H, D, generator=g, dtype=torch.float64, requires_grad=True)
    k = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64, requires_grad=True)
    v = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64, requires_grad=True)
    do = torch.randn(L, H, D, generator=g, dtype=torch.float64)
    scale = 0.43
    mask = torch.from_numpy(explicit_mask(L, N, layout, causal, P))
    o = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None],
        attn_mask=mask[None, None], scale=scale, enable_gqa=True)[0].permute(1, 0, 2)
    (o * do).sum().backward()
    p = problem(q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), N, layout, causal,
                P, scale)
    dq, dk, dv = oracle.attention_backward(p, do.numpy())
    assert np.abs(dq - q.grad.numpy()).max() < TIGHT
    assert np.abs(dk - k.grad.numpy()).max() < TIGHT
    assert np.abs(dv - v.grad.numpy()).max() < TIGHT


def test_backward_of_varlen_equals_each_sequence_alone():
    rng = np.random.default_rng(33)
    lens = [7, 12, 5]
    T, H, D, N = sum(lens), 2, 3, 3
    q, k, v, do = (rng.standard_normal((T, H, D)) for _ in range(4))
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    p = problem(q, k, v, N, 0, True, N, 0.7, starts=starts, lens=lens)
    grads = oracle.attention_backward(p, do)
    for s0, L in zip(starts, lens):
        sl = slice(s0, s0 + L)
        one = problem(q[sl], k[sl], v[sl], N, 0, True, N, 0.7)
        for g_all, g_one in zip(grads, oracle.attention_backward(one, do[sl])):
            assert np.array_equal(g_all[sl], g_one)


# ----------------------------------------------------------------------------
# Key/value-outer ring step
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout,causal", [(0, True), (1, True), (0, False), (1, False)])
def test_ring_steps_in_ring_order_reach_full_attention(layout, causal):
    """Folding every key/value block into the queries of each block, in ring
    order from an empty state, reaches full attention (the blockwise result
    is exact)."""
    L, N, H, D = 24, 4, 2, 5
    rng = np.random.default_rng(21)
    q, k, v = (rng.standard_normal((L, H, D)) for _ in range(3))
    scale = 0.45
    full_o, full_l = oracle.attention_full(problem(q, k, v, N, layout, causal, N, scale))
    for i in range(N):
        tq = oracle.block_rows(L, N, layout, i)
        out = np.zeros((tq.size, H, D))
        lse = np.full((H, tq.size), -np.inf)
        for s in range(N):
            j = (i - s) % N
            tk = oracle.block_rows(L, N, layout, j)
            out, lse = oracle.ring_step(q[tq], k[tk], v[tk], out, lse, L, N, layout, causal,
                                        scale, i, j)
        assert np.abs(out - full_o[tq]).max() < TIGHT
        assert np.abs(lse - full_l[:, tq]).max() < TIGHT


def test_ring_step_order_does_not_matter_and_one_step_is_block_attention():
    L, N, H, D, layout = 30, 5, 1, 4, 1
    rng = np.random.default_rng(22)
    q, k, v = (rng.standard_normal((L, H, D)) for _ in range(3))
    scale = 0.6
    i = 3
    tq = oracle.block_rows(L, N, layout, i)
    results = []
    for order in ([0, 1, 2, 3, 4], [4, 2, 0, 3, 1]):
        out = np.zeros((tq.size, H, D))
        lse = np.full((H, tq.size), -np.inf)
        for j in order:
            tk = oracle.block_rows(L, N, layout, j)
            out, lse = oracle.ring_step(q[tq], k[tk], v[tk], out, lse, L, N, layout, True,
                                        scale, i, j)
        results.append((out, lse))
    assert np.abs(results[0][0] - results[1][0]).max() < TIGHT
    assert np.abs(results[0][1] - results[1][1]).max() < TIGHT
    # one step from the empty state: attention over that block's keys, against
    # torch SDPA with the explicit mask restricted to the block
    j = 1
    tk = oracle.block_rows(L, N, layout, j)
    out, lse = oracle.ring_step(q[tq], k[tk], v[tk], np.zeros((tq.size, H, D)),
                                np.full((H, tq.size), -np.inf), L, N, layout, True, scale, i, j)
    mask = torch.from_numpy(explicit_mask(L, N, layout, True, N)[np.ix_(tq, tk)])
    has = mask.any(dim=1).numpy()
    qt, kt, vt = (torch.from_numpy(x[:, 0]) for x in (q[tq], k[tk], v[tk]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt[has][None], kt[None], vt[None], attn_mask=mask[has][None], scale=scale)[0]
    assert np.abs(out[has, 0] - ref.numpy()).max() < TIGHT
    # rows without an allowed key in the block keep the empty state
    assert np.all(out[~has] == 0.0) and np.all(np.isneginf(lse[0, ~has]))


# ----------------------------------------------------------------------------
# Brute force on tiny inputs (pure Python exp / normalise)
# ----------------------------------------------------------------------------

def brute_force(q, k, v, mask, scale):
    L, D = q.shape
    out = np.zeros((L, D))
    lse = np.zeros(L)
    for i in range(L):
        js = [j for j in range(L) if mask[i, j]]
        s = {j: scale * sum(float(q[i, d]) * float(k[j, d]) for d in range(D)) for j in js}
        m = max(s.values())
        w = {j: math.exp(s[j] - m) for j in js}
        tot = sum(w.values())
        for d in range(D):
            out[i, d] = sum(w[j] * float(v[j, d]) for j in js) / tot
        lse[i] = m + math.log(tot)
    return out, lse


def test_brute_force_tiny():
    rng = np.random.default_rng(3)
    for L in (1, 5, 8, 12):
        for N in (1, 2, 3, 4):
            if N > L:
                continue
            q = rng.standard_normal((L, 1, 3))
            k = rng.standard_normal((L, 1, 3))
            v = rng.standard_normal((L, 1, 3))
            for layout, causal in itertools.product((0, 1), (False, True)):
                for P in range(1, N + 1):
                    p = problem(q, k, v, N, layout, causal, P, 0.8)
                    o, lse = oracle.attention_full(p)
                    mask = explicit_mask(L, N, layout, causal, P)
                    bo, bl = brute_force(q[:, 0], k[:, 0], v[:, 0], mask, 0.8)
                    assert np.abs(o[:, 0] - bo).max() < 1e-12
                    assert np.abs(lse[0] - bl).max() < 1e-12


# ----------------------------------------------------------------------------
# The pages' worked examples
# ----------------------------------------------------------------------------

def test_glossary_four_device_ring_demo():
    """Re-enactment of the glossary's four-device demonstration: ring order
    j = (i - step) mod N, exponentials without max subtraction, division at
    the end; the ring result must equal full attention."""
    gold = load_golden("p4_ring_demo.json")
    N, blk, dim = gold["n_devices"], gold["block"], gold["dim"]
    torch.manual_seed(gold["seed"])
    q, k, v = torch.randn(3, N * blk, dim)
    q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
    outs = []
    for i in range(N):
        qi = q64[i * blk:(i + 1) * blk]
        num = np.zeros((blk, dim))
        den = np.zeros((blk, 1))
        for step in range(N):
            j = (i - step) % N
            kj, vj = k64[j * blk:(j + 1) * blk], v64[j * blk:(j + 1) * blk]
            e = np.exp(qi @ kj.T / math.sqrt(dim))
            assert e.shape == tuple(gold["score_block_per_device"])
            num += e @ vj
            den += e.sum(axis=1, keepdims=True)
        outs.append(num / den)
    ring = np.concatenate(outs)
    p = problem(q64[:, None], k64[:, None], v64[:, None], N, oracle.CONTIGUOUS, False, N,
                1.0 / math.sqrt(dim))
    o, _ = oracle.attention_full(p)
    assert o.shape[0] == gold["full_score_matrix"][0]
    assert np.abs(o[:, 0] - ring).max() < TIGHT
    # the page's own check on the fp32 torch demo
    full = torch.softmax(q @ k.T / dim ** 0.5, dim=-1) @ v
    assert torch.allclose(torch.from_numpy(ring).float(), full,
                          atol=gold["atol"]) == gold["matches_full_attention"]


def test_gist_ring_simulation_per_key_update():
    """Re-enactment of the gist's simulation in fp64: every worker keeps its
    query block, starts from its own key/value block and then takes the
    previous worker's; each key updates max, denominator and the
    renormalised output.  Must equal the oracle (no scale)."""
    gold = load_golden("p2_ring_simulation.json")
    n, d, W = gold["n_context"], gold["d_head"], gold["n_workers"]
    torch.manual_seed(gold["seed"])
    q, k, v = torch.randn(n, d), torch.randn(n, d), torch.randn(n, d)
    q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
    c = n // W
    outs = []
    for i in range(W):
        qi = q64[i * c:(i + 1) * c]
        o = np.zeros((c, d))
        m = np.full((c, 1), -np.inf)
        den = np.zeros((c, 1))
        for step in range(W):
            src = (i - step) % W     # block held at this step
            kb, vb = k64[src * c:(src + 1) * c], v64[src * c:(src + 1) * c]
            for t in range(c):
                x = qi @ kb[t:t + 1].T
                m_new = np.maximum(m, x)
                den_new = den * np.exp(m - m_new) + np.exp(x - m_new)
                o = o * (den * np.exp(m - m_new) / den_new) + np.exp(x - m_new) * vb[t:t + 1] / den_new
                m, den = m_new, den_new
        outs.append(o)
    ring = np.concatenate(outs)
    p = problem(q64[:, None], k64[:, None], v64[:, None], W, oracle.CONTIGUOUS, False, W,
                gold["scale"])
    o, _ = oracle.attention_full(p)
    assert np.abs(o[:, 0] - ring).max() < 1e-11
    assert np.allclose(ring, o[:, 0], rtol=gold["rtol"], atol=gold["atol"]) == gold["correct"]


# ----------------------------------------------------------------------------
# Invariants of the blockwise method
# ----------------------------------------------------------------------------

def blockwise_ring(q, k, v, mask, scale, blocks, order):
    """fp64 blockwise evaluation over key blocks in the given order with the
    online-softmax rescale."""
    L, D = q.shape
    m = np.full(L, -np.inf)
    l = np.zeros(L)
    acc = np.zeros((L, D))
    for bi in order:
        idx = blocks[bi]
        s = scale * (q @ k[idx].T)
        s = np.where(mask[:, idx], s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        m_safe = np.where(np.isfinite(m_new), m_new, 0.0)
        a = np.exp(np.where(np.isfinite(m), m - m_safe, -np.inf))
        e = np.exp(s - m_safe[:, None])
        l = l * a + e.sum(axis=1)
        acc = acc * a[:, None] + e @ v[idx]
        m = m_new
    return acc / l[:, None], m + np.log(l)


@pytest.mark.parametrize("layout,causal,P", [(0, False, 6), (0, True, 6), (1, True, 6),
                                             (1, True, 2), (0, False, 3)])
def test_kv_block_order_permutation_invariance(layout, causal, P):
    rng = np.random.default_rng(5)
    L, N, D = 60, 6, 7
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    mask = oracle.allowed_matrix(L, N, layout, causal, P)
    blk = oracle.ring_block(np.arange(L), L, N, layout)
    blocks = [np.flatnonzero(blk == r) for r in range(N)]
    o_ref, l_ref = oracle.attention_full(problem(q[:, None], k[:, None], v[:, None], N, layout,
                                                 causal, P, 0.5))
    for trial in range(5):
        order = rng.permutation(N)
        o, lse = blockwise_ring(q, k, v, mask, 0.5, blocks, order)
        assert np.abs(o - o_ref[:, 0]).max() < TIGHT
        assert np.abs(lse - l_ref[0]).max() < TIGHT


def test_merge_of_disjoint_key_sets_and_associativity():
    rng = np.random.default_rng(9)
    L, D = 40, 6
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    full = np.ones((L, L), dtype=bool)
    parts = np.array_split(rng.permutation(L), 3)
    res = []
    for idx in parts:
        m = np.zeros((L, L), dtype=bool)
        m[:, idx] = True
        res.append(oracle.masked_attention(q, k, v, m, 0.7))
    ref_o, ref_l = oracle.masked_attention(q, k, v, full, 0.7)
    (a_o, a_l), (b_o, b_l), (c_o, c_l) = res
    ab_c = oracle.merge(*oracle.merge(a_o, a_l, b_o, b_l), c_o, c_l)
    a_bc = oracle.merge(a_o, a_l, *oracle.merge(b_o, b_l, c_o, c_l))
    ba = oracle.merge(b_o, b_l, a_o, a_l)
    ab = oracle.merge(a_o, a_l, b_o, b_l)
    for o, l in (ab_c, a_bc):
        assert np.abs(o - ref_o).max() < TIGHT and np.abs(l - ref_l).max() < TIGHT
    assert np.abs(ab[0] - ba[0]).max() < TIGHT and np.abs(ab[1] - ba[1]).max() < TIGHT


def test_merge_empty_sides():
    rng = np.random.default_rng(2)
    o = rng.standard_normal((4, 3))
    l = rng.standard_normal(4)
    e_o = np.zeros((4, 3))
    e_l = np.full(4, -np.inf)
    mo, ml = oracle.merge(o, l, e_o, e_l)
    assert np.array_equal(mo, o) and np.array_equal(ml, l)
    mo, ml = oracle.merge(e_o, e_l, o, l)
    assert np.array_equal(mo, o) and np.array_equal(ml, l)
    mo, ml = oracle.merge(e_o, e_l, e_o, e_l)
    assert np.all(mo == 0) and np.all(ml == -np.inf)


def test_striped_equals_contiguous_after_unpermute():
    rng = np.random.default_rng(4)
    L, N, D = 64, 8, 5
    q, k, v = (rng.standard_normal((L, 1, D)) for _ in range(3))
    o_c, l_c = oracle.attention_full(problem(q, k, v, N, oracle.CONTIGUOUS, True, N, 0.6))
    # stored striped order: position s holds token pos[s]
    pos, _ = explicit_geometry(L, N, oracle.STRIPED)
    o_s, l_s = oracle.attention_full(problem(q[pos], k[pos], v[pos], N, oracle.STRIPED, True,
                                             N, 0.6))
    back = np.empty_like(o_s)
    back[pos] = o_s
    lback = np.empty_like(l_s)
    lback[:, pos] = l_s
    assert np.abs(back - o_c).max() < TIGHT
    assert np.abs(lback - l_c).max() < TIGHT


def test_varlen_equals_each_sequence_alone():
    rng = np.random.default_rng(6)
    lens = [5, 17, 1, 30]
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    T, H, D, N = sum(lens), 2, 4, 3
    q, k, v = (rng.standard_normal((T, H, D)) for _ in range(3))
    o, lse = oracle.attention_full(problem(q, k, v, N, oracle.CONTIGUOUS, True, N, 0.5,
                                           starts, lens))
    for s0, L in zip(starts, lens):
        sl = slice(s0, s0 + L)
        o1, l1 = oracle.attention_full(problem(q[sl], k[sl], v[sl], N, oracle.CONTIGUOUS, True,
                                               N, 0.5))
        assert np.array_equal(o[sl], o1) and np.array_equal(lse[:, sl], l1)


def test_zero_length_sequences_contribute_nothing():
    # cu_seqlens only has to be non-decreasing: an empty sequence owns no row
    # and no key, so the others come out exactly as without it (both layouts,
    # a pass cap below N)
    rng = np.random.default_rng(16)
    lens = [0, 6, 0, 0, 11, 0]
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    kept = [L for L in lens if L > 0]
    kstarts = np.concatenate([[0], np.cumsum(kept)[:-1]])
    T, H, D, N = sum(lens), 2, 4, 3
    q, k, v = (rng.standard_normal((T, H, D)) for _ in range(3))
    for layout in (oracle.CONTIGUOUS, oracle.STRIPED):
        o, lse = oracle.attention_full(problem(q, k, v, N, layout, True, 2, 0.5, starts, lens))
        o2, l2 = oracle.attention_full(problem(q, k, v, N, layout, True, 2, 0.5, kstarts, kept))
        assert np.array_equal(o, o2) and np.array_equal(lse, l2)
        assert np.isfinite(o).all() and np.isfinite(lse).all()


def test_row_sample_equals_full():
    rng = np.random.default_rng(8)
    T, H, D, N = 50, 3, 4, 5
    q, k, v = (rng.standard_normal((T, H, D)).astype(np.float32) for _ in range(3))
    p = problem(q, k, v, N, oracle.STRIPED, True, 2, 0.4)
    o, lse = oracle.attention_full(p)
    rows = rng.integers(0, T, 20)
    heads = rng.integers(0, H, 20)
    so, sl = oracle.attention_rows(p, np.zeros(20, int), heads, rows)
    assert np.array_equal(so, o[rows, heads]) and np.array_equal(sl, lse[heads, rows])


# ----------------------------------------------------------------------------
# Input recipe
# ----------------------------------------------------------------------------

def test_varlen_lengths_recipe():
    w = gen.WORKLOADS["bf16_varlen_t65536_s16_h16_d128_causal_n4_packed"]
    g = torch.Generator().manual_seed(w.seed)
    lens = gen.varlen_lengths(g, w.n_seqs, w.seqlen, *w.len_range)
    assert int(lens.sum()) == 65536 and len(lens) == 16
    assert int(lens.min()) >= 1
    # rescaling keeps lengths near the drawn range
    assert 512 < int(lens.min()) and int(lens.max()) < 9000

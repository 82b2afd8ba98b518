"""The tensor-core forward's own schedule, recorded on the GPU by its
schedule-builder warp (ring_attn_test_dump_schedule), against brute force.

For every work item (256 query rows: two 128-row query tiles) the kernel
visits kv tiles of 128 keys in ring order and classifies each (query tile,
kv tile) pair EMPTY / FULL / PARTIAL; PARTIAL tiles are masked element by
element, FULL tiles not at all, EMPTY ones are skipped.  Bit-exact checks:

  * the visited kv tiles are exactly those with an allowed pair for either
    query tile, each once;
  * the classes equal the brute-force classes of the allowed mask (the
    geometries here keep every tile inside the exact-classification regime);
  * the visit order is ring order: the step (r_q - r_k) mod N of each tile's
    block, relative to the item's first row, never decreases;
  * every head of an item gets the same list.

Cases: both layouts, causal or not, pass caps below N, a ragged length,
varlen sequences (including lengths 0 and 1) and key/value-outer ring steps.
"""

import collections

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
T = 128  # rows per query tile and keys per kv tile


def cls_of(sub):
    if sub.size == 0 or not sub.any():
        return 0
    return 1 if sub.all() else 2


def dumped(run, capacity=1 << 16):
    buf = torch.zeros(4 + 4 * capacity, dtype=torch.int32, device=DEV)
    ra.ring_attn_test_dump_schedule(buf)
    try:
        run()
        torch.cuda.synchronize()
    finally:
        ra.ring_attn_test_dump_schedule(None)
    assert ra.ring_attn_status() == ra.RA_OK
    n = int(buf[0])
    assert 0 < n <= capacity
    recs = buf[4:4 + 4 * n].view(n, 4).cpu().numpy()
    items = collections.defaultdict(list)
    for b, h, qr, e in recs.tolist():
        items[(b, h, qr)].append((e >> 4, e & 3, (e >> 2) & 3))
    return items


def check_items(items, seqs, N, layout, causal, P, heads, q_off=0, k_off=0, q_rows=None,
                k_rows=None):
    """seqs: {b: L}.  q_off/k_off: stored index of the first query row / key of
    the arrays (a ring step's blocks); q_rows/k_rows: their extents."""
    for b, L in seqs.items():
        if L == 0:
            assert not any(key[0] == b for key in items)
            continue
        mask = oracle.allowed_matrix(L, N, layout, causal, P)
        blk = oracle.ring_block(np.arange(L), L, N, layout)
        nq = L if q_rows is None else q_rows
        nk = L if k_rows is None else k_rows
        for qr in range((nq + 2 * T - 1) // (2 * T)):
            r0 = q_off + 2 * T * qr
            t0 = mask[r0:min(r0 + T, q_off + nq)]
            t1 = mask[min(r0 + T, q_off + nq):min(r0 + 2 * T, q_off + nq)]
            want = {}
            for kt in range((nk + T - 1) // T):
                c = slice(k_off + kt * T, k_off + min((kt + 1) * T, nk))
                c0, c1 = cls_of(t0[:, c]), cls_of(t1[:, c])
                if c0 or c1:
                    want[kt] = (c0, c1)
            lists = [items.get((b, h, qr), []) for h in range(heads)]
            assert all(x == lists[0] for x in lists), "heads differ"
            got = lists[0]
            kts = [kt for kt, _, _ in got]
            assert len(kts) == len(set(kts)), "a kv tile visited twice"
            assert {kt: (c0, c1) for kt, c0, c1 in got} == want, (b, qr)
            steps = [(blk[r0] - blk[k_off + kt * T]) % N for kt in kts]
            assert steps == sorted(steps), ("not in ring order", b, qr)


DENSE = [
    # (L, N, layout, causal, P)
    (2048, 8, 0, True, 8),
    (2048, 8, 1, True, 3),
    (4096, 16, 1, True, 4),
    (1000, 5, 0, False, 2),
    (1536, 6, 1, False, 6),
]


@pytest.mark.parametrize("L,N,layout,causal,P", DENSE)
def test_dense_schedule_equals_brute_force(L, N, layout, causal, P):
    w = gen.Workload("dump", "bf16", 1, 2, L, 64, causal, N, layout, P, seed=70)
    inp = gen.make_inputs(w)
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    lse = torch.empty(1, 2, L, device=DEV)
    items = dumped(lambda: ra.ring_attn_fwd(q, k, v, out, lse, 1, 2, L, 64, N, layout, causal,
                                            w.softmax_scale, P))
    check_items(items, {0: L}, N, layout, causal, P, heads=2)


@pytest.mark.parametrize("layout,P", [(0, 4), (1, 2)])
def test_varlen_schedule_equals_brute_force(layout, P):
    lens = [300, 1, 0, 777, 1500]
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0)
    Tt, H, D, N = int(cu[-1]), 2, 64, 4
    g = torch.Generator().manual_seed(71)
    qkv = torch.randn(Tt, 3, H, D, generator=g).to(torch.bfloat16).to(DEV)
    out = torch.empty(Tt, H, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(H, Tt, device=DEV)
    cud = cu.to(DEV)
    items = dumped(lambda: ra.ring_attn_qkvpacked_fwd(qkv, out, lse, len(lens), H, Tt, D, N,
                                                      layout, True, None, P, cud))
    check_items(items, dict(enumerate(lens)), N, layout, True, P, heads=H)


@pytest.mark.parametrize("qb,kb,layout", [(5, 3, 0), (5, 5, 0), (2, 6, 1), (4, 4, 1)])
def test_ring_step_schedule_equals_brute_force(qb, kb, layout):
    # key/value-outer ring step: the builder walks only block kb's tiles and
    # classifies them against block qb's rows in the whole sequence
    L, N, H, D = 2048, 8, 2, 64
    b = L // N
    w = gen.Workload("dump_step", "bf16", 1, H, L, D, True, N, layout, N, seed=72)
    inp = gen.make_inputs(w)
    q = inp["q"][:, qb * b:(qb + 1) * b].contiguous().to(DEV)
    k = inp["k"][:, kb * b:(kb + 1) * b].contiguous().to(DEV)
    v = inp["v"][:, kb * b:(kb + 1) * b].contiguous().to(DEV)
    out = torch.empty(1, b, H, D, device=DEV)
    lse = torch.empty(1, H, b, device=DEV)
    items = dumped(lambda: ra.ring_attn_fwd_step(q, k, v, out, lse, 1, H, L, D, N, qb, kb,
                                                 False, layout, True))
    check_items(items, {0: L}, N, layout, True, N, heads=H, q_off=qb * b, k_off=kb * b,
                q_rows=b, k_rows=b)


def test_hook_off_records_nothing():
    buf = torch.zeros(4 + 4 * 16, dtype=torch.int32, device=DEV)
    ra.ring_attn_test_dump_schedule(buf)
    ra.ring_attn_test_dump_schedule(None)
    x = torch.zeros(1, 256, 1, 64, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(1, 1, 256, device=DEV)
    ra.ring_attn_fwd(x, x, x, torch.empty_like(x), lse, 1, 1, 256, 64, 2, 0, True, 0.1, 2)
    torch.cuda.synchronize()
    assert int(buf[0]) == 0

"""The allocation-free forward, ring_attn_fwd_noalloc, called through the C ABI.

Some callers cannot allocate device memory once they are running: servers
and runtimes that hand out all device memory up front (a fixed pool or
budget, where a late cudaMalloc is a leak or an out-of-memory risk), and code
running where a cudaMalloc would synchronize the device or is not allowed.
ring_attn_fwd cudaMallocs a small scratch (status word, work counters) on its
first call; ring_attn_fwd_noalloc takes that scratch from a fixed array in
the library's device image instead.  These tests check that

  * its results are bitwise those of ring_attn_fwd (the same kernels run) and
    within the parity tolerances of the oracle, on two calls in a row (the
    array keeps the previous call's contents), for the tensor-core kernel
    (dense, causal striped with a pass cap, varlen) and the CUDA-core one;
  * a fresh process that only calls it sees no change in free device memory,
    while the first allocating call afterwards does (so the library's own
    scratch had not been allocated);
  * device-side errors latched under it are read and cleared by
    ring_attn_noalloc_status, and not by ring_attn_status.

The file is collected last; it also passes run alone in a fresh process.
"""

import json
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
from gpu_util import TOL, problem_for

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CODES = {"f32": ra.F32, "bf16": ra.BF16, "f16": ra.F16}


def _call(fn, q, k, v, out, lse, w, batch, seqlen, cu):
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), batch,
              w.heads, seqlen, w.d_head, w.n_ring, w.layout, int(w.causal),
              float(w.softmax_scale), w.passes, None if cu is None else cu.data_ptr(),
              CODES[w.dtype], torch.cuda.current_stream().cuda_stream)


def _oracle_errors(w, inp, out, lse):
    p = problem_for(w, inp)
    o_ref, l_ref = oracle.attention_full(p)
    if w.varlen:
        o, l = out.cpu().float().numpy(), lse.cpu().numpy()
    else:
        B, S, H, D = out.shape
        o = out.cpu().float().numpy().reshape(B * S, H, D)
        l = lse.cpu().permute(1, 0, 2).reshape(H, B * S).numpy()
    return float(np.abs(o - o_ref).max()), float(np.abs(l - l_ref).max())


WORKLOADS = [
    gen.Workload("noalloc_dense", "bf16", 2, 4, 1024, 128, False, 8, gen.CONTIGUOUS, 8, seed=31),
    gen.Workload("noalloc_striped", "bf16", 1, 3, 2048, 128, True, 8, gen.STRIPED, 3, seed=32),
    gen.Workload("noalloc_varlen", "bf16", 4, 2, 3000, 64, True, 4, gen.CONTIGUOUS, 4, seed=33,
                 varlen=True, n_seqs=4, len_range=(300, 1200)),
    gen.Workload("noalloc_fp32", "f32", 1, 2, 1000, 32, True, 5, gen.STRIPED, 5, seed=34,
                 scale=0.2),
]


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_noalloc_equals_allocating_forward_and_oracle(w):
    lib = ra.load_library()
    dev = torch.device("cuda", 0)
    inp = gen.make_inputs(w)
    if w.varlen:
        q, k, v = (inp[n].contiguous().to(dev) for n in ("q", "k", "v"))
        cu = inp["cu_seqlens"].to(dev)
        batch, seqlen = w.n_seqs, q.shape[0]
        lse_shape = (w.heads, seqlen)
    else:
        q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
        cu = None
        batch, seqlen = w.batch, w.seqlen
        lse_shape = (w.batch, w.heads, w.seqlen)
    ref_o = torch.empty_like(q)
    ref_l = torch.empty(lse_shape, device=dev)
    assert _call(lib.ring_attn_fwd, q, k, v, ref_o, ref_l, w, batch, seqlen, cu) == ra.RA_OK
    for _ in range(2):   # two calls in a row share the scratch array
        out = torch.full_like(q, float("nan"))
        lse = torch.full(lse_shape, float("nan"), device=dev)
        assert _call(lib.ring_attn_fwd_noalloc, q, k, v, out, lse, w, batch, seqlen,
                     cu) == ra.RA_OK
        assert ra.ring_attn_noalloc_status() == ra.RA_OK
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    assert ra.ring_attn_status() == ra.RA_OK
    eo, el = _oracle_errors(w, inp, out, lse)
    to, tl = TOL[w.dtype]
    assert eo <= to and el <= tl, (eo, el)


def test_noalloc_status_reports_bad_cu_seqlens_and_clears():
    lib = ra.load_library()
    dev = torch.device("cuda", 0)
    q = torch.zeros(256, 1, 128, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(1, 256, device=dev)
    cu = torch.tensor([0, 200, 100], dtype=torch.int32, device=dev)  # decreasing, wrong total
    w = gen.Workload("bad", "bf16", 2, 1, 256, 128, True, 2, gen.CONTIGUOUS, 2, seed=0,
                     varlen=True, n_seqs=2)
    assert ra.ring_attn_status() == ra.RA_OK
    assert _call(lib.ring_attn_fwd_noalloc, q, q, q, out, lse, w, 2, 256, cu) == ra.RA_OK
    assert ra.ring_attn_noalloc_status() == ra.RA_ERR_INVALID
    assert ra.ring_attn_noalloc_status() == ra.RA_OK      # the read cleared it
    assert ra.ring_attn_status() == ra.RA_OK              # the library's own word is apart


def test_noalloc_status_reports_an_expired_wait():
    lib = ra.load_library()
    w = gen.Workload("noalloc_timeout", "bf16", 1, 2, 512, 128, False, 4, gen.CONTIGUOUS, 4,
                     seed=35)
    inp = gen.make_inputs(w)
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    out = torch.zeros_like(q)
    lse = torch.zeros(1, 2, 512, device=dev)
    prev = ra.ring_attn_test_withhold_q(True)
    try:
        assert _call(lib.ring_attn_fwd_noalloc, q, k, v, out, lse, w, 1, 512, None) == ra.RA_OK
        st = ra.ring_attn_noalloc_status()
    finally:
        ra.ring_attn_test_withhold_q(prev)
    assert st == ra.RA_ERR_TIMEOUT, ra.ring_attn_status_string(st)
    assert ra.ring_attn_noalloc_status() == ra.RA_OK
    # the next call with the hook off runs normally
    assert _call(lib.ring_attn_fwd_noalloc, q, k, v, out, lse, w, 1, 512, None) == ra.RA_OK
    assert ra.ring_attn_noalloc_status() == ra.RA_OK
    eo, el = _oracle_errors(w, inp, out, lse)
    assert eo <= TOL["bf16"][0] and el <= TOL["bf16"][1]


FRESH = r"""
import json, sys, torch
sys.path.insert(0, ROOT)
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
w = gen.Workload("noalloc_fresh", "bf16", 1, 4, 2048, 128, True, 8, gen.STRIPED, 4, seed=36)
inp = gen.make_inputs(w)
q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
out = torch.empty_like(q)
lse = torch.empty(1, 4, 2048, device="cuda")
lib = ra.load_library()
def call():
    return lib.ring_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        lse.data_ptr(), 1, 4, 2048, 128, 8, 1, 1, w.softmax_scale, 4, None, ra.BF16,
        torch.cuda.current_stream().cuda_stream)
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
rc = [call()]                       # first call: address look-up, kernel load
st = [lib.ring_attn_noalloc_status(None)]
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
rc += [call(), call()]
st += [lib.ring_attn_noalloc_status(None)]
torch.cuda.synchronize()
free2 = torch.cuda.mem_get_info()[0]
torch.save({"out": out.cpu(), "lse": lse.cpu()}, OUT)
st_lib = lib.ring_attn_status(None)     # the library's first allocation
torch.cuda.synchronize()
free3 = torch.cuda.mem_get_info()[0]
print(json.dumps(dict(rc=rc, st=st, st_lib=st_lib, free=[free0, free1, free2, free3])))
"""


def test_fresh_process_calling_only_noalloc_allocates_nothing():
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "res.pt")
        code = FRESH.replace("ROOT", repr(ROOT)).replace("OUT", repr(path))
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        res = json.loads(r.stdout.strip().splitlines()[-1])
        got = torch.load(path)
    assert res["rc"] == [ra.RA_OK] * 3 and res["st"] == [ra.RA_OK] * 2, res
    assert res["st_lib"] == ra.RA_OK
    free0, free1, free2, free3 = res["free"]
    # repeated calls leave free device memory exactly as it was
    assert free2 == free1, res
    # the library's scratch was still unallocated: its first allocating call
    # (ring_attn_status) takes device memory only now
    assert free3 < free2, res
    w = gen.Workload("noalloc_fresh", "bf16", 1, 4, 2048, 128, True, 8, gen.STRIPED, 4, seed=36)
    eo, el = _oracle_errors(w, gen.make_inputs(w), got["out"], got["lse"])
    assert eo <= TOL["bf16"][0] and el <= TOL["bf16"][1], (eo, el)

"""The allocation-free forward (ring_attn_fwd_noalloc) against ring_attn_fwd.

Callers that may not allocate device memory (graph capture that forbids it,
fixed memory pools) use ring_attn_fwd_noalloc, whose scratch -- the error
status word and the persistent kernel's work counter -- is a fixed array in
the library's device image.  Its results must equal those of the allocating
entry point, also on consecutive calls (the array keeps the previous call's
contents, so each call has to clear it).  Called through the C ABI directly.
This file is collected last and runs alone in a fresh process as well.
"""

import pytest
import torch

import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 2e-2, 1e-3   # the bf16 tolerances of the parity tests


def _call(fn, q, k, v, out, lse, w):
    B, S, H, D = q.shape
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, S,
              D, w.n_ring, w.layout, int(w.causal), float(w.softmax_scale), w.passes, None,
              ra.BF16, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("causal,layout,passes", [(False, 0, 8), (True, 1, 3)])
def test_noalloc_matches_allocating_forward_on_consecutive_calls(causal, layout, passes):
    lib = ra.load_library()
    dev = torch.device("cuda", 0)
    w = gen.Workload("noalloc", "bf16", 2, 4, 2048, 128, causal, 8, layout, passes, seed=31)
    inp = gen.make_inputs(w)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    B, S, H, D = q.shape
    ref_o = torch.empty_like(q)
    ref_l = torch.empty(B, H, S, device=dev)
    assert _call(lib.ring_attn_fwd, q, k, v, ref_o, ref_l, w) == ra.RA_OK
    for _ in range(2):   # two calls in a row share the scratch array
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, S), float("nan"), device=dev)
        assert _call(lib.ring_attn_fwd_noalloc, q, k, v, out, lse, w) == ra.RA_OK
        torch.cuda.synchronize()
        assert float((out.float() - ref_o.float()).abs().max()) <= TOL_O
        assert float((lse - ref_l).abs().max()) <= TOL_LSE
        assert torch.isfinite(out.float()).all()


def test_noalloc_rejects_bad_arguments_like_the_allocating_call():
    lib = ra.load_library()
    x = torch.zeros(1, 256, 1, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 256, device="cuda")
    st = lib.ring_attn_fwd_noalloc(x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(),
                                   lse.data_ptr(), 1, 1, 250, 128, 4, 0, 1, 0.1, 4, None,
                                   ra.BF16, None)
    assert st == ra.RA_ERR_INVALID   # seqlen not a multiple of the ring blocks

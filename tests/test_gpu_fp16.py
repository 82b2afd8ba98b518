"""fp16 inputs (RA_F16) on the GPU against the fp64 oracle.

The oracle receives exactly the fp16 values the GPU reads (upcast).
ring_attn_fwd runs fp16 on the tensor cores (kind::f16 with fp16 operands, P
in fp16, fp32 accumulation) for d_head 64/128; ring_attn_fwd_simt runs it on
the CUDA cores for every head size.  Tolerances: 4e-3 on O, 1e-3 on lse (see
gpu_util.TOL).
"""

import numpy as np
import pytest
import torch

import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen
from gpu_util import TOL, compare_full, run_gpu

pytestmark = pytest.mark.gpu

FP16_SMALL = [
    # (B, H, S, D, causal, N, layout, P, impl)
    (2, 2, 1024, 128, False, 8, 0, 8, "tc"),
    (1, 3, 1000, 128, True, 8, 0, 8, "tc"),          # ragged tail
    (1, 2, 1024, 128, True, 8, 1, 3, "tc"),          # striped, pass cap
    (1, 2, 640, 64, True, 5, 0, 5, "tc"),
    (1, 2, 512, 32, True, 4, 1, 4, "simt"),          # head size of the CUDA-core kernel only
    (1, 2, 768, 128, True, 4, 0, 2, "simt"),
]


def check(w, err_o, err_l):
    to, tl = TOL[w.dtype]
    assert err_o <= to and err_l <= tl, (w.name, err_o, err_l)


@pytest.mark.parametrize("case", FP16_SMALL, ids=lambda c: "-".join(map(str, c)))
def test_fp16_small_all_rows(case):
    """Every row of small fp16 problems, tensor-core and CUDA-core kernels."""
    B, H, S, D, causal, N, layout, P, impl = case
    w = gen.Workload("fp16", "f16", B, H, S, D, causal, N, layout, P, seed=500 + S)
    inp = gen.make_inputs(w)
    assert inp["q"].dtype == torch.float16
    out, lse = run_gpu(w, inp, impl=impl)
    assert out.dtype == torch.float16
    check(w, *compare_full(w, inp, out, lse))


@pytest.mark.parametrize("causal,N", [(True, 4), (False, 2)])
def test_fp16_varlen_packed_all_rows(causal, N):
    w = gen.Workload("fp16vl", "f16", 4, 2, 3000, 128, causal, N, 0, N, seed=77, varlen=True,
                     packed=True, n_seqs=4, len_range=(300, 1200))
    inp = gen.make_inputs(w)
    out, lse = run_gpu(w, inp)
    check(w, *compare_full(w, inp, out, lse))


def test_fp16_grouped_query_all_rows():
    w = gen.Workload("fp16gqa", "f16", 1, 8, 1024, 128, True, 8, 1, 8, seed=78, heads_kv=2)
    inp = gen.make_inputs(w)
    out, lse = run_gpu(w, inp)
    check(w, *compare_full(w, inp, out, lse))


def test_fp16_tensor_core_matches_cuda_core_kernel():
    """Two independent GPU paths on the same fp16 inputs agree within the
    fp16 tolerance on every row."""
    w = gen.Workload("fp16x", "f16", 1, 2, 2048, 128, True, 8, 1, 8, seed=79)
    inp = gen.make_inputs(w)
    o1, l1 = run_gpu(w, inp, impl="tc")
    o2, l2 = run_gpu(w, inp, impl="simt")
    assert float((o1.float() - o2.float()).abs().max()) <= TOL["f16"][0]
    assert float((l1 - l2).abs().max()) <= TOL["f16"][1]

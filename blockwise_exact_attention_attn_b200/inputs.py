"""Seeded synthetic inputs shared by the tests, the benchmark and smoke().

This module only draws random numbers and describes workload shapes; it holds
none of the attention arithmetic.  Both the CUDA path and the oracle receive
the very arrays produced here (bf16 values reach the oracle upcast exactly).

Every workload draws q, k, v i.i.d. N(0, 1) from ``torch.Generator('cpu')``
seeded per workload (fp32 draws, cast to bf16 where the workload is bf16);
grouped-query workloads draw k and v with their own (smaller) head count.
The varlen workload first draws its sequence lengths from the same generator
(uniform in [1024, 7168] in fp64, rescaled to sum to the total with
largest-remainder rounding, ties to the lower index), then the packed qkv.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

CONTIGUOUS, STRIPED = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str              # "f32", "bf16" or "f16"
    batch: int
    heads: int
    seqlen: int             # per sequence (dense) or total rows (varlen)
    d_head: int
    causal: bool
    n_ring: int
    layout: int
    passes: int
    seed: int
    scale: Optional[float] = None     # None: 1/sqrt(d_head)
    varlen: bool = False
    packed: bool = False
    n_seqs: int = 0                   # varlen only
    len_range: tuple = field(default=(1024, 7168))
    heads_kv: int = 0                 # key/value heads (0: same as heads)

    @property
    def kv_heads(self) -> int:
        return self.heads_kv if self.heads_kv else self.heads

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d_head)

    @property
    def torch_dtype(self):
        return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[self.dtype]


# The five workloads of the benchmark description (sizes, seeds) plus small
# variants used by the tests, one grouped-query workload (8 query heads per
# key/value head) and the headline shape in fp16.
WORKLOADS = {
    "fp32_b1_h1_s1024_d16_noncausal_n16": Workload(
        "fp32_b1_h1_s1024_d16_noncausal_n16", "f32", 1, 1, 1024, 16, False, 16,
        CONTIGUOUS, 16, 1337, scale=0.25),
    "bf16_b2_h16_s8192_d128_noncausal_n8": Workload(
        "bf16_b2_h16_s8192_d128_noncausal_n8", "bf16", 2, 16, 8192, 128, False, 8,
        CONTIGUOUS, 8, 2),
    "bf16_b1_h32_s32768_d128_causal_n8_contiguous": Workload(
        "bf16_b1_h32_s32768_d128_causal_n8_contiguous", "bf16", 1, 32, 32768, 128, True, 8,
        CONTIGUOUS, 8, 3),
    "bf16_b1_h32_s32768_d128_causal_n8_striped": Workload(
        "bf16_b1_h32_s32768_d128_causal_n8_striped", "bf16", 1, 32, 32768, 128, True, 8,
        STRIPED, 8, 3),
    "bf16_varlen_t65536_s16_h16_d128_causal_n4_packed": Workload(
        "bf16_varlen_t65536_s16_h16_d128_causal_n4_packed", "bf16", 16, 16, 65536, 128, True,
        4, CONTIGUOUS, 4, 4, varlen=True, packed=True, n_seqs=16),
    "bf16_b1_h8_s262144_d128_causal_striped_n16_p16": Workload(
        "bf16_b1_h8_s262144_d128_causal_striped_n16_p16", "bf16", 1, 8, 262144, 128, True,
        16, STRIPED, 16, 5),
    "bf16_b1_h8_s262144_d128_causal_striped_n16_p4": Workload(
        "bf16_b1_h8_s262144_d128_causal_striped_n16_p4", "bf16", 1, 8, 262144, 128, True,
        16, STRIPED, 4, 5),
    "f16_b2_h16_s8192_d128_noncausal_n8": Workload(
        "f16_b2_h16_s8192_d128_noncausal_n8", "f16", 2, 16, 8192, 128, False, 8,
        CONTIGUOUS, 8, 7),
    "bf16_b1_h32_kv4_s32768_d128_causal_n8_contiguous": Workload(
        "bf16_b1_h32_kv4_s32768_d128_causal_n8_contiguous", "bf16", 1, 32, 32768, 128, True,
        8, CONTIGUOUS, 8, 6, heads_kv=4),
}


def varlen_lengths(gen: torch.Generator, n_seqs: int, total: int, lo: int, hi: int):
    """Sequence lengths: n_seqs uniform draws in [lo, hi] rescaled to sum to
    total (largest remainder, ties to the lower index)."""
    u = torch.rand(n_seqs, generator=gen, dtype=torch.float64) * (hi - lo) + lo
    ideal = u * (total / float(u.sum()))
    base = torch.floor(ideal).to(torch.int64)
    short = int(total - int(base.sum()))
    frac = ideal - base.to(torch.float64)
    # stable sort by descending fraction keeps ties at the lower index first
    order = sorted(range(n_seqs), key=lambda i: (-float(frac[i]), i))
    for i in order[:short]:
        base[i] += 1
    return base


def make_inputs(w: Workload):
    """Host tensors of the workload.

    Returns a dict with q, k, v (dense: [B, S, H, D]; varlen/packed: qkv
    [T, 3, H, D] and q/k/v views) and, for varlen, cu_seqlens (int32 [B+1])
    and lengths.
    """
    g = torch.Generator().manual_seed(w.seed)
    out = {}
    if w.varlen:
        lens = varlen_lengths(g, w.n_seqs, w.seqlen, *w.len_range)
        cu = torch.zeros(w.n_seqs + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
        qkv = torch.randn(w.seqlen, 3, w.heads, w.d_head, generator=g).to(w.torch_dtype)
        out.update(qkv=qkv, cu_seqlens=cu, lengths=lens,
                   q=qkv[:, 0], k=qkv[:, 1], v=qkv[:, 2])
        return out
    shape = (w.batch, w.seqlen, w.heads, w.d_head)
    kv_shape = (w.batch, w.seqlen, w.kv_heads, w.d_head)
    q = torch.randn(*shape, generator=g).to(w.torch_dtype)
    k = torch.randn(*kv_shape, generator=g).to(w.torch_dtype)
    v = torch.randn(*kv_shape, generator=g).to(w.torch_dtype)
    out.update(q=q, k=k, v=v)
    return out


def make_device_inputs(w: Workload, device="cuda", seed: Optional[int] = None):
    """Same shapes drawn directly on the device (benchmark inputs; values
    differ from make_inputs)."""
    g = torch.Generator(device=device).manual_seed(w.seed if seed is None else seed)
    if w.varlen:
        gh = torch.Generator().manual_seed(w.seed)
        lens = varlen_lengths(gh, w.n_seqs, w.seqlen, *w.len_range)
        cu = torch.zeros(w.n_seqs + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
        qkv = torch.randn(w.seqlen, 3, w.heads, w.d_head, generator=g, device=device,
                          dtype=torch.float32).to(w.torch_dtype)
        return dict(qkv=qkv, cu_seqlens=cu.to(device), lengths=lens)
    shapes = {"q": (w.batch, w.seqlen, w.heads, w.d_head),
              "k": (w.batch, w.seqlen, w.kv_heads, w.d_head),
              "v": (w.batch, w.seqlen, w.kv_heads, w.d_head)}
    return {n: torch.randn(*shapes[n], generator=g, device=device,
                           dtype=torch.float32).to(w.torch_dtype) for n in ("q", "k", "v")}


def small(name: str, **kw) -> Workload:
    """A copy of a named workload with some fields replaced (test sizes)."""
    return replace(WORKLOADS[name], **kw)


def seq_offsets(w: Workload, inputs) -> tuple:
    """(start row, length) per sequence, host ints."""
    if w.varlen:
        cu = inputs["cu_seqlens"].tolist()
        return [cu[i] for i in range(len(cu) - 1)], [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]
    return [b * w.seqlen for b in range(w.batch)], [w.seqlen] * w.batch

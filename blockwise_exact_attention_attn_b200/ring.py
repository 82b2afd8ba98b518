"""Sequence-parallel ring attention across the ranks of a process group.

Rank r of an N-rank group holds ring block r of every sequence in the chosen
layout (contiguous: tokens [r*b, (r+1)*b); striped: tokens r, r+N, r+2N,
...): q, k and v of shape [batch, b, heads, d_head].  Each rank keeps its
query block and the key/value blocks travel around the ring: at ring step s
rank r holds block (r - s) mod N, folds it into the running result of its
queries, and passes it on to rank r+1 while the next one arrives from rank
r-1 ("Ring Attention" glossary, "Come funziona la ring attention": each
device keeps its queries, the key/value blocks rotate, and the block held at
step s came from the previous device; the issue thread "A ring attention with
flash attention kernel implementation": with keys and values on the outer
loop the queries' reduced output and lse are kept and passed back in on the
next pass).  max_ring_passes P < N stops after P steps (own block plus the
P-1 blocks that arrive first).

The fold is ring_attn_fwd_step (fp32 running state).  The exchange is
point-to-point (NCCL over NVLink on GPUs) into local double buffers: the
transfer for step s+1 is issued before the step-s kernel, so the two overlap,
and the kernels only ever read this device's memory.
"""

from __future__ import annotations

import math
from typing import Callable, Optional

CONTIGUOUS, STRIPED = 0, 1


def device_fold(q, k, v, out, lse, q_block: int, kv_block: int, accumulate: bool, seqlen: int,
                n_ring: int, layout: int, causal: bool, scale: float) -> None:
    """Fold key/value block kv_block into (out, lse) on the GPU."""
    from ._binding import ring_attn_fwd_step
    B, b, H, D = q.shape
    ring_attn_fwd_step(q, k, v, out, lse, B, H, seqlen, D, n_ring, q_block, kv_block,
                       accumulate, layout, causal, scale)


def check_device_fold(q, softmax_scale: float) -> None:
    """Raise ValueError when ring_attn_fwd_step would refuse this rank's
    block: 16-bit inputs, d_head 64 or 128, a block of whole 128-row tiles and
    a nonzero scale.  Checked before the first exchange, so that every rank
    (same shapes on all of them) fails before any transfer is in flight."""
    import torch
    B, b, H, D = q.shape
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError(f"the device ring step takes bf16 or fp16 inputs, not {q.dtype}")
    if D not in (64, 128):
        raise ValueError(f"the device ring step takes d_head 64 or 128, not {D}")
    if b % 128 != 0:
        raise ValueError(f"the device ring step needs blocks of whole 128-row tiles, not {b}")
    if softmax_scale == 0.0:
        raise ValueError("the device ring step needs a nonzero softmax scale")


def ring_attention_forward(q, k, v, *, causal: bool = False, layout: int = CONTIGUOUS,
                           softmax_scale: Optional[float] = None,
                           max_ring_passes: Optional[int] = None, group=None,
                           fold: Callable = device_fold, out_dtype=None):
    """Ring attention forward over the ranks of `group` (default: the world).

    q, k, v: this rank's ring block, [batch, b, heads, d_head] (CUDA tensors
    for the default fold).  Returns (out, lse): out [batch, b, heads, d_head]
    in out_dtype (default: the running state's type, float32; float64 for
    float64 inputs), lse [batch, heads, b] in the state's type.  Every rank must call it with the same arguments; the
    sequence length is b times the group size.
    """
    import torch
    import torch.distributed as dist

    N = dist.get_world_size(group)
    r = dist.get_rank(group)
    B, b, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k and v must have the same shape")
    L = b * N
    P = N if max_ring_passes is None else max(1, min(int(max_ring_passes), N))
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    if fold is device_fold:
        check_device_fold(q, scale)
    # the running state is fp32 (what the device step keeps); fp64 inputs
    # (host checks) keep it in fp64
    state = torch.float64 if q.dtype == torch.float64 else torch.float32
    out = torch.empty(B, b, H, D, dtype=state, device=q.device)
    lse = torch.empty(B, H, b, dtype=state, device=q.device)

    def peer(delta: int) -> int:
        rank = (r + delta) % N
        return rank if group is None else dist.get_global_rank(group, rank)

    # two receive buffers; the caller's k/v are only read (step 0)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, P - 1))]
    cur_k, cur_v = k, v
    for s in range(P):
        j = (r - s) % N
        works = []
        if s + 1 < P:
            # Buffer reuse: bufs[s % 2] was last read by the fold of step
            # s - 1, enqueued on the current stream before this call.  With
            # NCCL, batch_isend_irecv makes its communication stream wait for
            # the work already on the current stream when the ops are issued,
            # so the receive cannot overwrite the buffer before that fold has
            # read it; with gloo the ops run on the host after the (host)
            # fold returned.  The w.wait() below orders the next fold after
            # this receive in the other direction.
            nk, nv = bufs[s % 2]
            ops = [dist.P2POp(dist.isend, cur_k, peer(1), group),
                   dist.P2POp(dist.isend, cur_v, peer(1), group),
                   dist.P2POp(dist.irecv, nk, peer(-1), group),
                   dist.P2POp(dist.irecv, nv, peer(-1), group)]
            works = dist.batch_isend_irecv(ops)
        fold(q, cur_k, cur_v, out, lse, r, j, s > 0, L, N, layout, causal, scale)
        for w in works:
            w.wait()
        if s + 1 < P:
            cur_k, cur_v = bufs[s % 2]
    if out_dtype is not None and out_dtype != out.dtype:
        out = out.to(out_dtype)
    return out, lse

"""Helpers shared by the GPU tests: run the CUDA path through the C ABI,
run the oracle on the same inputs, choose sampled rows."""

import numpy as np
import torch

import oracle
import blockwise_exact_attention_attn_b200 as ra
from blockwise_exact_attention_attn_b200 import inputs as gen

# (max |dO|, max |dlse|).  fp16: outputs are rounded to an 11-bit significand
# (half an ulp is 2^-11 relative, under 2e-3 for |O| < 4) and P enters the
# tensor cores in fp16 (2^-11 relative), so 4e-3 on O; lse is computed in fp32
# as for bf16.
TOL = {"f32": (1e-4, 1e-5), "bf16": (2e-2, 1e-3), "f16": (4e-3, 1e-3)}


def run_gpu(w, inp, impl="tc", stream=None):
    """Run the workload on cuda:0; returns (out, lse) on the host in the
    library's layouts ([T, H, D] / [H, T] token-major over all sequences)."""
    dev = torch.device("cuda", 0)
    fn = ra.ring_attn_fwd if impl == "tc" else ra.ring_attn_fwd_simt
    if w.varlen:
        qkv = inp["qkv"].to(dev)
        cu = inp["cu_seqlens"].to(dev)
        T = qkv.shape[0]
        out = torch.empty(T, w.heads, w.d_head, dtype=qkv.dtype, device=dev)
        lse = torch.empty(w.heads, T, dtype=torch.float32, device=dev)
        if w.packed and impl == "tc":
            ra.ring_attn_qkvpacked_fwd(qkv, out, lse, w.n_seqs, w.heads, T, w.d_head, w.n_ring,
                                       w.layout, w.causal, w.softmax_scale, w.passes, cu)
        else:
            q, k, v = (qkv[:, i].contiguous() for i in range(3))
            fn(q, k, v, out, lse, w.n_seqs, w.heads, T, w.d_head, w.n_ring, w.layout, w.causal,
               w.softmax_scale, w.passes, cu)
        torch.cuda.synchronize()
        assert ra.ring_attn_status() == ra.RA_OK
        return out.cpu(), lse.cpu()
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    B, S, H, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    if w.kv_heads != w.heads:
        # one entry point for both kernels: fp32 runs on the CUDA cores
        ra.ring_attn_gqa_fwd(q, k, v, out, lse, B, H, w.kv_heads, S, D, w.n_ring, w.layout,
                             w.causal, w.softmax_scale, w.passes)
    else:
        fn(q, k, v, out, lse, B, H, S, D, w.n_ring, w.layout, w.causal, w.softmax_scale,
           w.passes)
    torch.cuda.synchronize()
    assert ra.ring_attn_status() == ra.RA_OK
    # to token-major [T, H, D] / [H, T]
    return out.cpu().reshape(B * S, H, D), lse.cpu().permute(1, 0, 2).reshape(H, B * S)


def problem_for(w, inp, heads=None):
    """oracle.Problem over the given heads (all by default), float32 arrays
    holding exactly the values the GPU sees."""
    if w.varlen:
        q, k, v = inp["q"], inp["k"], inp["v"]
    else:
        q = inp["q"].reshape(-1, w.heads, w.d_head)
        k, v = (inp[n].reshape(-1, w.kv_heads, w.d_head) for n in ("k", "v"))
    if heads is not None:
        # the listed query heads with the key/value head each of them reads
        kvh = [oracle.kv_head(h, w.heads, w.kv_heads) for h in heads]
        q, k, v = q[:, heads], k[:, kvh], v[:, kvh]
    starts, lens = gen.seq_offsets(w, inp)
    return oracle.Problem(q=q.float().numpy(), k=k.float().numpy(), v=v.float().numpy(),
                          seq_start=np.array(starts), seq_len=np.array(lens), n_ring=w.n_ring,
                          layout=w.layout, causal=w.causal, passes=w.passes,
                          scale=w.softmax_scale)


def sample_rows(w, inp, rng, n_random=256, max_tiles=64, heads=(0,)):
    """(seq, head_index_into_heads, row) triples: first and last row of every
    ring block, of up to max_tiles 128-row tiles (evenly spread, both ends
    included) and n_random random rows, for each listed head."""
    starts, lens = gen.seq_offsets(w, inp)
    seqs, hs, rows = [], [], []
    for b, L in enumerate(lens):
        pick = set()
        blk = oracle.ring_block(np.arange(L), L, w.n_ring, w.layout)
        edges = np.flatnonzero(np.diff(blk)) + 1
        for e in edges:
            pick.update((int(e) - 1, int(e)))
        pick.update((0, L - 1))
        nt = (L + 127) // 128
        for t in np.unique(np.linspace(0, nt - 1, min(nt, max_tiles)).astype(int)):
            pick.update((128 * int(t), min(L - 1, 128 * int(t) + 127)))
        nr = max(1, n_random // len(lens))
        pick.update(int(x) for x in rng.integers(0, L, nr))
        for hi in range(len(heads)):
            for r in sorted(pick):
                seqs.append(b)
                hs.append(hi)
                rows.append(r)
    return np.array(seqs), np.array(hs), np.array(rows)


def compare_rows(w, inp, out, lse, seqs, hs, rows, heads):
    """Max |dO| and |dlse| between the GPU result and the oracle on the
    sampled rows."""
    p = problem_for(w, inp, heads=list(heads))
    o_ref, l_ref = oracle.attention_rows(p, seqs, hs, rows)
    starts, _ = gen.seq_offsets(w, inp)
    g = np.array(starts)[seqs] + rows
    hh = np.array(heads)[hs]
    o_gpu = out[g, hh].float().numpy()
    l_gpu = lse[hh, g].numpy()
    return float(np.abs(o_gpu - o_ref).max()), float(np.abs(l_gpu - l_ref).max())


def compare_full(w, inp, out, lse):
    p = problem_for(w, inp)
    o_ref, l_ref = oracle.attention_full(p)
    return (float(np.abs(out.float().numpy() - o_ref).max()),
            float(np.abs(lse.numpy() - l_ref).max()))

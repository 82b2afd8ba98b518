// ra_work.cuh -- map a CTA to its work item (sequence, query range, head).
//
// Dense inputs: CTA index w -> (batch, head, query range) with the query
// range fastest, so the CTAs running together share a few heads' K/V in L2;
// causal ranges are ordered heaviest first (see decode_work).
// Varlen inputs (cu_seqlens, "Tensorflow flash attention" page: cumulative
// sequence lengths of shape (batch_size + 1,) index ragged, unpadded
// tensors): CTA index w -> (flat range, head) with the head fastest; the flat
// range is located among the sequences by a warp-wide scan of their range
// counts ceil(L_b / rows_per_cta), and inside a sequence the ranges run from
// the last to the first for causal contiguous inputs.
#pragma once

#include <stdint.h>

#include "ra_common.cuh"
#include "ra_params.h"

namespace ra {

struct SeqWork {
  int b, qr, h;   // sequence, query range within it, head
  int base;       // global row of the sequence's first token
  int L;          // sequence length
  bool live;      // false: nothing to do for this CTA
};

// Work item `item` (a CTA index of the non-persistent grid).  Must be called
// by all 32 lanes of a warp (any warp; every warp computes the same answer).
// Latches ST_INVALID for malformed cu_seqlens.
__device__ __forceinline__ SeqWork find_work_item(const FwdParams& p, int rows_per_cta,
                                                  int item) {
  SeqWork w;
  w.live = false;
  w.b = w.qr = w.h = w.base = w.L = 0;
  const int lane = threadIdx.x & 31;
  if (!p.cu_seqlens) {
    const WorkItem it = decode_work(p, item);
    w.b = it.b;
    w.qr = it.qr;
    w.h = it.h;
    const int rows = q_rows_per_seq(p);
    w.base = it.b * rows;
    w.L = p.seqlen;
    w.live = (int64_t)it.qr * rows_per_cta < rows;
    return w;
  }
  const int flat = item / p.heads;
  w.h = item - flat * p.heads;
  if (lane == 0 && threadIdx.x == 0 && item == 0 &&
      (p.cu_seqlens[0] != 0 || p.cu_seqlens[p.batch] != p.total_rows))
    latch_status(p.status, ST_INVALID);
  int acc = 0;
  for (int b0 = 0; b0 < p.batch; b0 += 32) {
    const int b = b0 + lane;
    int n = 0, s0 = 0, len = 0;
    if (b < p.batch) {
      s0 = p.cu_seqlens[b];
      const int s1 = p.cu_seqlens[b + 1];
      len = s1 - s0;
      if (s0 < 0 || len < 0 || s1 > p.total_rows) {
        if (w.h == 0 && flat == 0) latch_status(p.status, ST_INVALID);
        len = 0;
      }
      n = (len + rows_per_cta - 1) / rows_per_cta;
    }
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - n;
    const bool mine = n > 0 && flat >= acc + excl && flat < acc + incl;
    const unsigned hit = __ballot_sync(0xffffffffu, mine);
    if (hit) {
      const int src = __ffs(hit) - 1;
      w.b = __shfl_sync(0xffffffffu, b, src);
      w.base = __shfl_sync(0xffffffffu, s0, src);
      w.L = __shfl_sync(0xffffffffu, len, src);
      const int nq = __shfl_sync(0xffffffffu, n, src);
      const int qi = flat - acc - __shfl_sync(0xffffffffu, excl, src);
      w.qr = p.order == 1 ? nq - 1 - qi : qi;
      w.live = true;
      return w;
    }
    acc += __shfl_sync(0xffffffffu, incl, 31);
  }
  return w;
}

__device__ __forceinline__ SeqWork find_work(const FwdParams& p, int rows_per_cta) {
  return find_work_item(p, rows_per_cta, (int)blockIdx.x);
}

// Causal striped dense inputs whose ring blocks hold a whole number of work
// items: order the items by local position (heaviest first).
inline void set_striped_order(FwdParams& p, int rows_per_cta) {
  if (p.cu_seqlens || p.step || !p.causal || p.layout != 1) return;
  const int blk = p.seqlen / p.n_ring;
  if (blk % rows_per_cta != 0 || blk == 0) return;
  p.order = 2;
  p.qr_per_block = blk / rows_per_cta;
}

// Launch size: dense n_qranges * batch * heads; varlen (ceil(total /
// rows_per_cta) + batch) * heads, an upper bound of the ranges of all
// sequences.
inline int64_t work_grid(const FwdParams& p, int rows_per_cta) {
  if (!p.cu_seqlens) {
    const int64_t nq = ((int64_t)q_rows_per_seq(p) + rows_per_cta - 1) / rows_per_cta;
    return nq * p.batch * p.heads;
  }
  const int64_t nq = ((int64_t)p.total_rows + rows_per_cta - 1) / rows_per_cta + p.batch;
  return nq * p.heads;
}

}  // namespace ra

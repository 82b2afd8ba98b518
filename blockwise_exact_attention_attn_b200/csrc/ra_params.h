// ra_params.h -- launch parameters shared by the host API and the kernels.
#pragma once

#include <stdint.h>

namespace ra {

// Element formats of the 16-bit inputs, as the kind::f16 MMA encodes them
// (A and B always share one).
constexpr int kFmtF16 = 0;
constexpr int kFmtBF16 = 1;
// 8-bit e4m3 inputs on kind::f8f6f4 MMAs (the output is bf16)
constexpr int kFmtE4M3 = 2;

// One forward call, in the form every forward kernel consumes.  Rows of all
// sequences are addressed as one token axis: token row r of sequence b is
// global row seq_base(b) + r, with seq_base(b) = b * seqlen (dense) or
// cu_seqlens[b] (varlen).
struct FwdParams {
  const void* q;            // element (row, h, d) at q + row*tok_stride + h*d_head + d
  const void* k;            // element (row, hk, d) at k + row*kv_tok_stride + hk*d_head + d
  const void* v;            // (same layout as k)
  int64_t tok_stride;       // elements between consecutive rows of q
  int64_t kv_tok_stride;    // elements between consecutive rows of k/v
  void* out;                // [rows, heads, d_head], same dtype as q
  float* lse;               // see lse_seq_stride / lse_head_stride
  int64_t lse_seq_stride;   // dense: heads*seqlen; varlen: 0
  int64_t lse_head_stride;  // dense: seqlen;       varlen: total rows
  const int32_t* cu_seqlens;  // NULL for dense
  int batch, heads, seqlen, d_head;
  int heads_kv;             // key/value heads; query head h reads hk = h / kv_group
  int kv_group;             // heads / heads_kv
  int n_ring, layout, causal, passes;
  int total_rows;           // rows of q/k/v/out (dense: batch*seqlen)
  int n_qranges;            // query ranges per sequence (ceil(seqlen / rows per CTA))
  int order;                // query-range order inside a (sequence, head): 0 natural,
                            // 1 last to first, 2 striped (local position descending)
  int qr_per_block;         // order 2: query ranges per ring block
  float scale;              // softmax scale
  float scale_log2;         // scale * log2(e)
  float out_scale;          // multiplies O / l in the epilogue (1, or fp8's v descale)
  int* status;              // device status word (never NULL at launch)
  int* work_counter;        // persistent kernels: next work item (zeroed per launch)
  // Key/value-outer ring step (ring_attn_fwd_step): q, out and lse hold the
  // step_rows rows of ring block q_block of each sequence, k and v those of
  // kv_block; seqlen stays the whole sequence (the ring geometry).  out is
  // fp32; with accumulate the call folds into the running (out, lse).
  int step;                 // 0: whole-sequence call
  int q_block, kv_block, step_rows;
  int accumulate;
  // Ring steps whose items do not fill the last wave of CTAs split the
  // last step_split items in two halves of their key tiles: launch items
  // [0, n - step_split) are whole, then item n - step_split + s comes as
  // halves 0 and 1 (launch items n - step_split + 2s and + 2s + 1).  Half 0
  // folds into (out, lse) like a whole item; half 1 starts from the empty
  // state and writes its partial (normalised O, lse) to split_out [s][row]
  // [d_head] and split_lse [s][row] (rows of the item, 256), which a merge
  // kernel then folds into (out, lse).  0 and NULL otherwise.
  int step_split;
  float* split_out;
  float* split_lse;
  // Failure-detection test hook (0 in normal use): the tensor-core kernel's
  // producer issues no query-tile load, so the MMA issuers' bounded wait for
  // Q expires and the launch unwinds with ST_TIMEOUT.
  int withhold_q;
  // Schedule-dump test hook (NULL in normal use): the tensor-core kernel's
  // schedule builder appends one record {b, h, qr, entry} per visited kv
  // tile to sched_dump + 4, counting records in sched_dump[0] (atomically;
  // only the first sched_dump_cap are stored).  entry = (kv tile << 4) |
  // (class of query tile 1 << 2) | class of query tile 0.
  int* sched_dump;
  int64_t sched_dump_cap;
};

// Query rows per dense sequence held by q/out: the whole sequence, or one
// ring block in a step call.  (Varlen calls size each sequence from
// cu_seqlens instead.)
#if defined(__CUDACC__)
__host__ __device__ __forceinline__
#else
inline
#endif
int q_rows_per_seq(const FwdParams& p) { return p.step ? p.step_rows : p.seqlen; }

// Map a linear work index to (query range, batch, head).  The (batch, head)
// pair is the slowest index, so the work running at one time shares the K/V
// of a few heads in L2.  Inside a head the causal query ranges come heaviest
// first: from the last to the first (contiguous layout), or, striped, by
// local position inside the ring blocks from the last to the first (a
// striped query range at local position j of its block sees keys up to j of
// every block).
struct WorkItem {
  int qr, b, h;
};

#if defined(__CUDACC__)
__host__ __device__ __forceinline__
#else
inline
#endif
WorkItem decode_work(const FwdParams& p, int64_t w) {
  WorkItem it;
  const int64_t bh = w / p.n_qranges;
  const int qr = (int)(w - bh * p.n_qranges);
  it.b = (int)(bh / p.heads);
  it.h = (int)(bh - (int64_t)it.b * p.heads);
  if (p.order == 1) {
    it.qr = p.n_qranges - 1 - qr;
  } else if (p.order == 2) {
    const int jj = qr / p.n_ring, r = qr - jj * p.n_ring;
    it.qr = r * p.qr_per_block + (p.qr_per_block - 1 - jj);
  } else {
    it.qr = qr;
  }
  return it;
}

}  // namespace ra

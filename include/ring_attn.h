/*
 * ring_attn.h -- C ABI of the single-GPU blockwise exact ("ring") attention
 * forward for NVIDIA B200 (sm_100a).
 *
 * What is computed (per batch b, head h and query row i):
 *
 *     O[i]   = sum_{j in A(i)} exp(s_ij - m_i) v_j / l_i
 *     lse[i] = m_i + ln(l_i),    s_ij = softmax_scale * <q_i, k_j>,
 *     m_i = max_{j in A(i)} s_ij, l_i = sum_{j in A(i)} exp(s_ij - m_i)
 *
 * The sequence is split into N = n_ring_blocks "virtual devices" (ring
 * blocks).  Query block r meets key/value block (r - step) mod N at ring step
 * step = 0 .. N-1, and every block's partial result is folded into the output
 * with the online-softmax rescale (running row max, running denominator,
 * output rescaled by exp(m_old - m_new)); the division by l happens once at
 * the end.  Sources: "Ring Attention" (Ultralytics glossary), section
 * "Come funziona la ring attention" and its four-device demo; "Ring Attention
 * simulation" (gist ring_attention_simulation.py), the flashattention()
 * per-token update and Device.run ring loop.  On one GPU the ring is a block
 * iteration order: no data moves between devices.
 *
 * Allowed set A(i).  Let pos(t) be the original token index of stored row t
 * within its sequence (length L), rb(t) its ring block:
 *   contiguous layout: pos(t) = t, rb(t) = floor(t * N / L)
 *   striped layout   : ring block r holds tokens r, r+N, r+2N, ... stored
 *                      consecutively, blocks stored in order r = 0..N-1
 *                      ("Ring Attention" glossary: Striped Attention gives each
 *                      device tokens spread evenly over the sequence; the
 *                      issue thread below asks for striped causal masking to
 *                      even out the work).
 * j is in A(i) iff (1) i and j are in the same sequence, (2) causal == 0 or
 * pos(j) <= pos(i), and (3) (rb(i) - rb(j)) mod N < min(max_ring_passes, N)
 * (the issue thread's cap on ring passes: a query block sees its own block and
 * the max_ring_passes - 1 blocks that precede it in the ring).
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never frees or retains them.  The library allocates one 4-byte device
 *    status word per device on first use and nothing per call.
 *  - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *    stream).  The return value reports host-side validation and launch
 *    errors only; device-side errors (bad cu_seqlens contents, a pipeline wait
 *    that exceeded its bound) are latched in the status word and reported by
 *    ring_attn_status().
 *  - Every tensor pointer must be 16-byte aligned (cu_seqlens: 4-byte).
 *    Violations return RA_ERR_INVALID before anything is launched.
 *  - Thread safety: calls on different streams may run concurrently; the
 *    status word is shared per device.
 */
#ifndef RING_ATTN_H
#define RING_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID = 1,     /* bad argument; nothing was launched */
  RA_ERR_UNSUPPORTED = 2, /* valid request this build has no kernel for */
  RA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  RA_ERR_TIMEOUT = 4      /* a bounded in-kernel wait expired (device side) */
} ra_status;

typedef enum { RA_LAYOUT_CONTIGUOUS = 0, RA_LAYOUT_STRIPED = 1 } ra_layout;

/* Element type of q, k, v and out.  The "Tensorflow flash attention" page
 * lists fp16 and bf16 as the flash-attention input types; fp32 is the gist's
 * (and the fp32 workload's) type. */
typedef enum { RA_F32 = 0, RA_BF16 = 1, RA_F16 = 2 } ra_dtype;
/* (8-bit e4m3 inputs have their own entry point, ring_attn_fwd_fp8, because
 * they come with scale factors.) */

/*
 * ring_attn_fwd -- exact attention forward, ring-ordered blockwise.
 *
 * Source: "Ring Attention" glossary, "Come funziona la ring attention" (query
 * block kept in place, key/value blocks visited in ring order, partials
 * combined by the running softmax); "Ring Attention simulation" gist,
 * flashattention() update; issue thread "A ring attention with flash
 * attention kernel implementation" (lse is returned so that blockwise results
 * can be combined; maximum ring passes; striped masking; varlen variant).
 *
 * Arguments
 *  q, k, v   dtype elements.  Dense: [batch, seqlen, heads, d_head]
 *            contiguous (BSHD).  Varlen (cu_seqlens != NULL):
 *            [seqlen, heads, d_head], seqlen = total rows = cu_seqlens[batch].
 *  out       same shape and dtype as q; written for every valid row.
 *  lse       float32.  Dense: [batch, heads, seqlen].  Varlen: [heads, seqlen].
 *            Natural-log log-sum-exp of the scaled scores.
 *  batch     number of sequences (>= 1).
 *  heads     number of heads (>= 1).
 *  seqlen    dense: tokens per sequence (multiple of n_ring_blocks).
 *            varlen: total rows of q/k/v/out, which must equal
 *            cu_seqlens[batch] (the host never reads cu_seqlens, so the call
 *            stays asynchronous; the kernels check it).
 *  d_head    head dimension: RA_F32 accepts 16, 32, 64, 128;
 *            RA_BF16 and RA_F16 accept 64, 128 (tensor cores; bf16 or fp16
 *            products accumulated in fp32).
 *  n_ring_blocks  N >= 1, the number of virtual ring devices per sequence.
 *  layout    ra_layout; buffers are in that stored order and out/lse are
 *            returned in the same order.
 *  causal    0 or 1; causal in ORIGINAL token positions.
 *  softmax_scale  finite scale applied to q.k (the gist uses 1, the glossary
 *            demo 1/sqrt(d_head)).
 *  max_ring_passes  P >= 1; values above N are clamped to N.
 *  cu_seqlens  NULL for dense, else DEVICE int32[batch + 1] (4-byte aligned),
 *            cu_seqlens[0] = 0, non-decreasing, cu_seqlens[batch] = seqlen.
 *            Sequence b is rows [cu_seqlens[b], cu_seqlens[b+1]); its ring
 *            blocks follow its own length (any length >= 0, no divisibility
 *            requirement; a zero-length sequence owns no row and is
 *            skipped).  A negative length or an offset beyond seqlen
 *            latches RA_ERR_INVALID in the status word and that sequence's
 *            rows are left unwritten; a wrong cu_seqlens[0] or
 *            cu_seqlens[batch] latches RA_ERR_INVALID too.
 *  dtype     ra_dtype of q, k, v and out.
 *  stream    cudaStream_t to launch on.
 *
 * Errors: RA_ERR_INVALID for a null or misaligned pointer, a non-positive
 * size, seqlen % n_ring_blocks != 0 (dense), max_ring_passes < 1, a
 * non-finite softmax_scale, causal not in {0,1}, an unknown layout/dtype, or
 * a d_head outside {16,32,64,128}; RA_ERR_UNSUPPORTED for a d_head the dtype
 * has no kernel for, or for sizes past 32-bit row indices (dense
 * batch * seqlen, or batch * heads, above 2^31 - 1); RA_ERR_CUDA when a launch
 * fails.
 */
ra_status ring_attn_fwd(const void* q, const void* k, const void* v, void* out,
                        float* lse, int batch, int heads, int seqlen,
                        int d_head, int n_ring_blocks, int layout, int causal,
                        float softmax_scale, int max_ring_passes,
                        const int32_t* cu_seqlens, int dtype, void* stream);

/*
 * ring_attn_gqa_fwd -- ring_attn_fwd with fewer key/value heads than query
 * heads (grouped-query attention; heads_kv = 1 is multi-query attention).
 *
 * Source: "Tensorflow flash attention" page: multi-query and grouped-query
 * attention, in which several query heads attend to one key/value head.  The
 * page does not say which heads share; here query head h reads key/value
 * head h / (heads / heads_kv), i.e. consecutive groups of query heads share.
 *
 *  q, out    dense: [batch, seqlen, heads, d_head]; varlen: [seqlen, heads,
 *            d_head].
 *  k, v      dense: [batch, seqlen, heads_kv, d_head]; varlen: [seqlen,
 *            heads_kv, d_head].
 *  heads_kv  >= 1 and a divisor of heads; heads_kv == heads is ring_attn_fwd.
 *  lse       as ring_attn_fwd (one row per query head).
 * All other arguments as ring_attn_fwd.  Errors as ring_attn_fwd, plus
 * RA_ERR_INVALID when heads_kv < 1 or heads % heads_kv != 0.
 */
ra_status ring_attn_gqa_fwd(const void* q, const void* k, const void* v,
                            void* out, float* lse, int batch, int heads,
                            int heads_kv, int seqlen, int d_head,
                            int n_ring_blocks, int layout, int causal,
                            float softmax_scale, int max_ring_passes,
                            const int32_t* cu_seqlens, int dtype,
                            void* stream);

/*
 * ring_attn_fwd_fp8 -- ring_attn_gqa_fwd for 8-bit e4m3 (fp8, "E4M3FN":
 * 1 sign, 4 exponent, 3 mantissa bits, no infinities) q, k, v with one
 * scale factor per tensor: the values are q = descale_q * q8, k = descale_k
 * * k8, v = descale_v * v8.  The output is bf16.
 *
 * Source: "Tensorflow flash attention" page, which lists the input types
 * flash attention takes (fp8 with bf16/fp16); the method is ring_attn_fwd's.
 * The products run on the tensor cores in e4m3 (kind::f8f6f4, fp32
 * accumulation): scores from q8 and k8 scaled by softmax_scale * descale_q
 * * descale_k, and P = exp(s - m) rounded to e4m3 (round to nearest even;
 * relative error at most 2^-4 for P >= 2^-6 relative to the running
 * reference, absolute error at most 2^-10 below) before P V; l and lse use
 * the unrounded P in fp32.
 *
 *  q         uint8 holding e4m3, dense [batch, seqlen, heads, 128], varlen
 *            [seqlen, heads, 128].
 *  k, v      e4m3 with heads_kv heads (a divisor of heads).
 *  out       bf16, q's shape: descale_v * sum_j P_ij v8_j / l_i.
 *  lse       float32, as ring_attn_fwd (of the scaled scores).
 *  descale_q, descale_k, descale_v  finite per-tensor scale factors.
 * Other arguments as ring_attn_gqa_fwd.  Errors as ring_attn_gqa_fwd, plus
 * RA_ERR_INVALID for a non-finite descale (or a non-finite product with
 * softmax_scale) and RA_ERR_UNSUPPORTED for d_head != 128 or a zero
 * combined scale.
 */
ra_status ring_attn_fwd_fp8(const void* q, const void* k, const void* v,
                            void* out, float* lse, int batch, int heads,
                            int heads_kv, int seqlen, int d_head,
                            int n_ring_blocks, int layout, int causal,
                            float softmax_scale, int max_ring_passes,
                            const int32_t* cu_seqlens, float descale_q,
                            float descale_k, float descale_v, void* stream);

/*
 * ring_attn_fwd_step -- one key/value-outer ring step: the queries of ring
 * block q_block fold the keys and values of ring block kv_block into their
 * running result (out, lse), in place.
 *
 * Source: issue thread "A ring attention with flash attention kernel
 * implementation": with the keys and values iterated on the outer loop, the
 * reduced outputs and lse of the queries are stored and passed back in on
 * the next ring pass.  The fold is the online-softmax update started from
 * the stored state (m = lse, l = 1, O = out), the same arithmetic as folding
 * a partial result with ring_attn_merge.
 *
 *  q         dtype [batch, seqlen / n_ring_blocks, heads, d_head]: the rows
 *            of ring block q_block in stored order (contiguous: tokens
 *            [q_block * b, (q_block + 1) * b); striped: tokens q_block,
 *            q_block + N, ...).
 *  k, v      same shape: the rows of ring block kv_block.
 *  out       float32, same shape as q: the running normalised output.  Read
 *            when accumulate (rows with lse = -inf may hold anything), always
 *            written for rows that see a key of the block; with accumulate =
 *            0 rows that see none get 0.
 *  lse       float32 [batch, heads, seqlen / n_ring_blocks]: the running
 *            log-sum-exp, -inf for "nothing folded yet"; updated like out
 *            (-inf written with accumulate = 0 for rows that see no key).
 *  seqlen    tokens of the whole sequence (the ring geometry; causal masking
 *            compares original positions over the whole sequence).
 *  q_block, kv_block  ring blocks in [0, n_ring_blocks).
 *  accumulate  1: fold into (out, lse); 0: start from the empty state.
 * No pass limit applies: the caller chooses which blocks to fold.  An
 * accumulating step over a block pair the mask hides entirely (causal
 * contiguous, kv_block > q_block) returns RA_OK without launching anything.
 * Errors: as ring_attn_fwd, plus RA_ERR_INVALID for a block index out of
 * range or accumulate not in {0,1}; RA_ERR_UNSUPPORTED for RA_F32, a zero
 * scale, or a block size seqlen / n_ring_blocks that is not a multiple of
 * 128 (the step runs on the tensor cores with whole tiles per block).
 * Launch: one persistent thread block per SM, as a programmatic dependent of
 * the launch before it on the stream, so that its set-up overlaps that
 * launch's last blocks; it reads no input before that launch has completed,
 * so ordering on the stream is the same as for any kernel.  When the work
 * items (256 query rows of one head) leave the last wave of thread blocks at
 * most half full, those items are split in two halves of the block's key
 * tiles: the second halves write partial results to scratch taken from the
 * stream-ordered pool (cudaMallocAsync, returned with cudaFreeAsync on the
 * same stream), and a second kernel folds them into (out, lse).  If the pool
 * has no room the step runs unsplit.
 */
ra_status ring_attn_fwd_step(const void* q, const void* k, const void* v,
                             float* out, float* lse, int batch, int heads,
                             int seqlen, int d_head, int n_ring_blocks,
                             int layout, int causal, float softmax_scale,
                             int q_block, int kv_block, int accumulate,
                             int dtype, void* stream);

/*
 * ring_attn_bwd -- gradients of the forward: dq, dk, dv of sum(dout * out)
 * for out = ring_attn_fwd (or ring_attn_gqa_fwd) of q, k, v.
 *
 * Source: issue thread "A ring attention with flash attention kernel
 * implementation": the backward is the part an implementation got wrong,
 * and the returned lse is what the blockwise method keeps.  The gradients
 * are plain calculus on out_i = sum_j P_ij v_j, P_ij = exp(scale q_i.k_j -
 * lse_i) over the allowed keys: dV = P^T dout, dS = P (dP - D) with dP =
 * dout v^T and D_i = dout_i . out_i, dQ = scale dS K, dK = scale dS^T Q.
 * P is recomputed from the forward's lse.  Two kernels, so that every
 * gradient element has one writer: a query-outer one for dq (it also forms
 * D_i) and a key/value-outer one for dk and dv.  RA_BF16 and RA_F16 with
 * d_head 64 or 128 run on the tensor cores (16-bit products, fp32
 * accumulation; P and dS are rounded to the input type before their
 * products); everything else runs on CUDA cores in fp32 arithmetic.  The
 * tensor-core path takes batch * heads * seqlen (varlen: heads * seqlen)
 * floats of stream-ordered scratch per call (cudaMallocAsync / cudaFreeAsync
 * on `stream`, from the device's default memory pool).
 *
 *  q, k, v, out, lse  as passed to / returned by the forward (k, v with
 *            heads_kv heads; heads_kv == heads for ring_attn_fwd).
 *  dout      dtype, shape of out.
 *  dq        dtype, shape of q; written.
 *  dk, dv    dtype, shape of k / v; written (summed over the query heads
 *            that share a key/value head).
 * Other arguments as ring_attn_gqa_fwd; d_head in {16, 32, 64, 128} for
 * every dtype.  Errors as ring_attn_gqa_fwd.
 */
ra_status ring_attn_bwd(const void* q, const void* k, const void* v,
                        const void* out, const float* lse, const void* dout,
                        void* dq, void* dk, void* dv, int batch, int heads,
                        int heads_kv, int seqlen, int d_head,
                        int n_ring_blocks, int layout, int causal,
                        float softmax_scale, int max_ring_passes,
                        const int32_t* cu_seqlens, int dtype, void* stream);

/*
 * ring_attn_bwd_simt -- ring_attn_bwd computed by the CUDA-core kernels
 * (fp32 arithmetic) for every dtype and d_head; for RA_BF16 / RA_F16 it is
 * an independent second GPU path used to cross-check the tensor-core
 * backward.  Arguments and errors as ring_attn_bwd; allocates nothing.
 */
ra_status ring_attn_bwd_simt(const void* q, const void* k, const void* v,
                             const void* out, const float* lse,
                             const void* dout, void* dq, void* dk, void* dv,
                             int batch, int heads, int heads_kv, int seqlen,
                             int d_head, int n_ring_blocks, int layout,
                             int causal, float softmax_scale,
                             int max_ring_passes, const int32_t* cu_seqlens,
                             int dtype, void* stream);

/*
 * ring_attn_qkvpacked_fwd -- same computation, q/k/v packed in one tensor.
 *
 * Source: issue thread "A ring attention with flash attention kernel
 * implementation": ring_flash_attn_qkvpacked_func (mirrors
 * flash_attn_qkvpacked_func) and its varlen variant; the cu_seqlens shape
 * (batch_size + 1,) is stated on the "Tensorflow flash attention" page.
 *
 *  qkv   dense: [batch, seqlen, 3, heads, d_head]; varlen: [seqlen, 3, heads,
 *        d_head] (seqlen = total rows).  Index 0/1/2 of the "3" axis is q/k/v.
 *  out   dense: [batch, seqlen, heads, d_head]; varlen: [seqlen, heads, d_head].
 *  lse   as ring_attn_fwd.
 * All other arguments and errors as ring_attn_fwd.
 */
ra_status ring_attn_qkvpacked_fwd(const void* qkv, void* out, float* lse,
                                  int batch, int heads, int seqlen, int d_head,
                                  int n_ring_blocks, int layout, int causal,
                                  float softmax_scale, int max_ring_passes,
                                  const int32_t* cu_seqlens, int dtype,
                                  void* stream);

/*
 * ring_attn_fwd_simt -- the same contract as ring_attn_fwd computed by the
 * CUDA-core (SIMT, fp32 arithmetic) kernel for every dtype and d_head in
 * {16,32,64,128}.  It is the kernel RA_F32 always uses; for RA_BF16 it is an
 * independent second GPU path used to cross-check the tensor-core kernel on
 * every row.  Arguments and errors as ring_attn_fwd.
 */
ra_status ring_attn_fwd_simt(const void* q, const void* k, const void* v,
                             void* out, float* lse, int batch, int heads,
                             int seqlen, int d_head, int n_ring_blocks,
                             int layout, int causal, float softmax_scale,
                             int max_ring_passes, const int32_t* cu_seqlens,
                             int dtype, void* stream);

/*
 * ring_attn_merge -- fold partial result (out_b, lse_b) into (out_a, lse_a)
 * in place:
 *     lse = max(la, lb) + log1p(exp(min(la, lb) - max(la, lb)))
 *     out = exp(la - lse) * out_a + exp(lb - lse) * out_b
 * with lse = -inf and out = 0 when both sides are -inf, and the other side
 * copied exactly when one side is -inf.
 *
 * Source: issue thread "A ring attention with flash attention kernel
 * implementation": returning lse is what lets blockwise (per ring step)
 * results be combined, and the KV-outer variant stores outputs and lse and
 * passes them back in on the next ring pass.
 *
 *  out_a, out_b  dtype [batch, seqlen, heads, d_head] (varlen results: batch
 *                = 1, seqlen = total rows).  out_a is overwritten.
 *  lse_a, lse_b  float32 [batch, heads, seqlen].  lse_a is overwritten.
 *  d_head        RA_F32: 4, 8, 16, 32, 64 or 128; RA_BF16 and RA_F16: 8, 16,
 *                32, 64, 128 or 256 (a row is 1 to 32 whole 16-byte chunks).
 * Errors: RA_ERR_INVALID for null/misaligned pointers, non-positive sizes,
 * an unsupported d_head or dtype; RA_ERR_UNSUPPORTED when batch * seqlen *
 * heads rows exceed 2^31 - 1; RA_ERR_CUDA when the launch fails.
 */
ra_status ring_attn_merge(void* out_a, float* lse_a, const void* out_b,
                          const float* lse_b, int batch, int heads, int seqlen,
                          int d_head, int dtype, void* stream);

/*
 * ring_attn_fwd_noalloc -- ring_attn_fwd that allocates no device memory.
 * (The pages have no counterpart: this is a deployment variant of the same
 * call.)
 *
 * Who needs it: callers whose device memory is all handed out up front and
 * must not move afterwards -- inference servers and runtimes that reserve a
 * fixed pool or budget at start-up and treat any later cudaMalloc as a leak
 * or an out-of-memory risk, and code that runs where a cudaMalloc would
 * synchronize the device or is not permitted at all.  ring_attn_fwd
 * allocates a small device scratch (the error status word and the work
 * counters) with cudaMalloc on its first call on a device; this entry point
 * uses a 256-byte array that is part of the library's device image instead
 * (every device that loads the library holds it until the process exits) and
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *  - Arguments, layouts, ownership and host-side errors are those of
 *    ring_attn_fwd, and so are the results (the same kernels run).
 *  - Scratch limit: 256 bytes, of which each call uses the status word and
 *    one work counter.  No problem size changes that; a call that would need
 *    more than the array holds returns RA_ERR_UNSUPPORTED.
 *  - Set-up: the first call on each device looks the array's device address
 *    up (cudaGetSymbolAddress) with that device current.  Make that first
 *    call before any stream capture.
 *  - All calls share the array, which keeps the last call's contents: each
 *    call zeroes the work counter on its stream before its kernel starts.
 *    Calls that overlap on the GPU (e.g. on different streams) race on the
 *    array and may compute wrong results; issue them on one stream or order
 *    them.
 *  - Device-side errors (malformed cu_seqlens, an expired wait) are latched in
 *    the array's status word (the first error wins) and stay there until
 *    ring_attn_noalloc_status reads and clears them; ring_attn_status does
 *    not see them.
 */
ra_status ring_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                void* out, float* lse, int batch, int heads,
                                int seqlen, int d_head, int n_ring_blocks,
                                int layout, int causal, float softmax_scale,
                                int max_ring_passes, const int32_t* cu_seqlens,
                                int dtype, void* stream);

/*
 * ring_attn_noalloc_status -- synchronize `stream`, then return and clear the
 * status word of the ring_attn_fwd_noalloc calls on the current device
 * (RA_OK when none latched an error since the last read).  Allocates nothing
 * either: it copies the word into a host variable and clears it with
 * synchronous CUDA calls.  Returns RA_ERR_CUDA when a CUDA call fails.
 */
ra_status ring_attn_noalloc_status(void* stream);

/*
 * ring_attn_fwd_host -- ring_attn_fwd on HOST buffers, with the transfers
 * overlapped with the computation.
 *
 * Source: "Ring Attention" glossary, "Come funziona la ring attention": a
 * device computes on the block it holds while the next block is in flight,
 * so the transfer hides behind the computation.  Here the blocks are groups
 * of heads moving between host memory and the GPU: the heads are split into
 * chunks of head_chunk heads; chunk c's q/k/v are copied in while chunk c-1
 * is computed and chunk c-2's out/lse are copied out, on two library
 * streams plus `stream`, through two device slots of `workspace`.
 *
 *  q, k, v   HOST, page-locked (cudaHostAlloc / cudaHostRegister) dtype
 *            [batch, seqlen, heads, d_head].
 *  out       HOST, page-locked, same shape and dtype; written.
 *  lse       HOST, page-locked float32 [batch, heads, seqlen]; written.
 *  head_chunk  heads per chunk (>= 1), or 0 to let the library choose
 *            (ceil(heads / 8)).
 *  workspace DEVICE memory of at least ring_attn_fwd_host_workspace(...)
 *            bytes, 256-byte aligned, owned by the caller; one call at a
 *            time may use it.
 * Other arguments as ring_attn_fwd (dense inputs; no cu_seqlens).
 * Asynchronous on `stream`: the call returns once everything is enqueued;
 * out and lse are complete when `stream` is synchronized (then read device
 * errors with ring_attn_status).  Work already on `stream` runs first.
 * Calls from several host threads are serialised while they enqueue.
 * Errors: as ring_attn_fwd, plus RA_ERR_INVALID when a host buffer is not
 * page-locked, the workspace is not device memory, is misaligned or too
 * small, or head_chunk < 0.
 */
ra_status ring_attn_fwd_host(const void* q, const void* k, const void* v,
                             void* out, float* lse, int batch, int heads,
                             int seqlen, int d_head, int n_ring_blocks,
                             int layout, int causal, float softmax_scale,
                             int max_ring_passes, int dtype, int head_chunk,
                             void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * ring_attn_fwd_host_workspace -- bytes of device workspace ring_attn_fwd_host
 * needs for these sizes (two slots of one chunk's q, k, v, out and lse; one
 * slot when there is a single chunk).  Returns 0 for invalid sizes.  Host
 * only; never fails otherwise.
 */
size_t ring_attn_fwd_host_workspace(int batch, int heads, int seqlen,
                                    int d_head, int dtype, int head_chunk);

/*
 * ring_attn_status -- synchronize `stream`, then return and clear the current
 * device's status word (RA_OK when no device-side error was latched since the
 * last call).  Returns RA_ERR_CUDA when the synchronization itself fails.
 */
ra_status ring_attn_status(void* stream);

/*
 * ring_attn_test_withhold_q -- failure-detection test hook; leave it off (0)
 * in normal use.  While on, every tensor-core forward launch made by this
 * process (bf16/fp16 ring_attn_fwd, _gqa_fwd, _fwd_step, _qkvpacked_fwd,
 * _fwd_noalloc) loads no query tile: the MMA warps' bounded wait for Q gives
 * up after about one second, every role of the CTA unwinds (copies and MMAs
 * already issued are drained, tensor memory is freed) and RA_ERR_TIMEOUT is
 * latched in the status word; the output is left unspecified.  The device
 * context stays usable.  Host-only: the setting is read when a call builds
 * its launch parameters, so it can be toggled without a GPU.
 *  on  nonzero = on, 0 = off.
 * Returns the previous setting (0 or 1).  Never fails.
 */
int ring_attn_test_withhold_q(int on);

/*
 * ring_attn_test_dump_schedule -- test hook that makes the tensor-core
 * forward's own schedule visible; leave it off (buf = NULL) in normal use.
 * While set, every tensor-core forward launch made by this process
 * (ring_attn_fwd, _gqa_fwd, _fwd_step, _qkvpacked_fwd, _fwd_noalloc, bf16 or
 * fp16) appends, from the kernel's schedule-builder warp, one record of four
 * int32 per visited key/value tile of 128 keys:
 *     {sequence b, head h, query range qr, entry}
 * where the work item (b, h, qr) is query rows [256 qr, 256 qr + 256) of
 * sequence b (in a ring step: of the query block), and entry = (kv tile << 4)
 * | (class of the item's second 128-row query tile << 2) | (class of its
 * first), class 0 = EMPTY, 1 = FULL, 2 = PARTIAL; kv tile counts 128-key
 * tiles from the sequence start (in a ring step: from the key block's
 * start).  The records of one item appear in visit order.
 *  buf       DEVICE int32 array of 4 + 4 * capacity elements; buf[0] counts
 *            the records (atomically, also past capacity; only the first
 *            capacity are stored from buf[4] on).  The caller zeroes buf[0]
 *            before the launch and keeps buf alive while the hook is set.
 *  capacity  records buf holds (>= 0).
 * Host-only setting, read when a call builds its launch parameters.
 * Returns RA_ERR_INVALID for a negative capacity or a NULL buf with
 * capacity > 0 (the setting is unchanged then), RA_OK otherwise.
 */
ra_status ring_attn_test_dump_schedule(int32_t* buf, int64_t capacity);

/* Human-readable name of a status code (static storage, never NULL). */
const char* ring_attn_status_string(int status);

/*
 * ring_attn_schedule -- host-side view of the ring-step scheduler, the same
 * code the kernels run on the device.  For one sequence of length seqlen it
 * lists, for every q-tile of q_tile rows (in stored order), the kv-tiles of
 * kv_tile rows it visits, in visit (ring) order, with their class:
 *   1 = FULL (every query/key pair of the two tiles is allowed, no mask),
 *   2 = PARTIAL (mixed; the element mask is applied).
 * EMPTY pairs (no allowed pair) are not visited and not listed.
 * The classification is exact whenever the ring-block index ranges the two
 * tiles span, multiplied, are at most 64 (empty blocks inside a range, which
 * exist when a sequence is shorter than N, count); beyond that a pair that is
 * really EMPTY or FULL may be listed as PARTIAL (never the reverse).
 *
 *  q_tiles_per_item  1: each q-tile walks alone.  2: consecutive pairs of
 *                 q-tiles (the tensor-core kernel's work items of
 *                 2 * q_tile rows; the last may hold one tile) walk one
 *                 shared key/value stream, in the ring order of the pair's
 *                 first row; each tile's visited pairs are listed in stream
 *                 order, the first tile's entry before the second's.
 *  out_q, out_kv  int32 tile indices; out_class int8.  HOST arrays of
 *                 `capacity` entries (may be NULL when capacity is 0).
 * Returns the total number of visited pairs (which may exceed capacity; only
 * the first `capacity` are written), or -1 for invalid arguments.
 */
int64_t ring_attn_schedule(int seqlen, int n_ring_blocks, int layout,
                           int causal, int max_ring_passes, int q_tile,
                           int kv_tile, int q_tiles_per_item, int32_t* out_q,
                           int32_t* out_kv, int8_t* out_class,
                           int64_t capacity);

#ifdef __cplusplus
}
#endif

#endif /* RING_ATTN_H */

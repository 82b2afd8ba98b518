// ra_api.cu -- the C ABI declared in include/ring_attn.h: argument
// validation (before any CUDA call), the per-device status word, and the
// choice of kernel (tensor-core kernel for bf16, CUDA-core kernel for fp32).
#include <cmath>
#include <cstdint>
#include <atomic>
#include <mutex>

#include <cuda_runtime.h>

#include "ra_params.h"
#include "ra_sched.h"
#include "ring_attn.h"

namespace ra {
cudaError_t launch_fwd_tc(const FwdParams& p, int fmt, cudaStream_t stream);
cudaError_t launch_fwd_simt(const FwdParams& p, int dtype, cudaStream_t stream);
cudaError_t launch_bwd_simt(const FwdParams& f, const void* o, const void* dout, void* dq,
                            void* dk, void* dv, int dtype, cudaStream_t stream);
cudaError_t launch_bwd_tc(const FwdParams& f, const void* o, const void* dout, void* dq,
                          void* dk, void* dv, float* dsum, int fmt, int num_sms,
                          cudaStream_t stream);
cudaError_t launch_merge(void* out_a, float* lse_a, const void* out_b, const float* lse_b,
                         int batch, int heads, int seqlen, int d_head, int dtype, int num_sms,
                         cudaStream_t stream);
}  // namespace ra

namespace {

constexpr int kMaxDevices = 64;
// Per device, one allocation: the status word at [0] and, from
// [kCounterBase], a ring of work counters handed one per persistent launch
// (distinct launches in flight on different streams use distinct counters).
constexpr int kCounterBase = 32;
constexpr int kCounterSlots = 256;
std::mutex g_mu;
int* g_status[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};
unsigned g_next_slot[kMaxDevices] = {0};
// Failure-detection test hook, read by every forward call (ring_attn_test_withhold_q).
std::atomic<int> g_withhold_q{0};
// Schedule-dump test hook (ring_attn_test_dump_schedule): device buffer and
// record capacity, read by every forward call.
std::atomic<int*> g_sched_dump{nullptr};
std::atomic<int64_t> g_sched_dump_cap{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device, its status word (allocated and zeroed on first use) and SM
// count.
ra_status device_state(int** status, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status[dev]) {
    int* p = nullptr;
    const size_t bytes = sizeof(int) * (kCounterBase + kCounterSlots);
    if (cudaMalloc(&p, bytes) != cudaSuccess) return RA_ERR_CUDA;
    if (cudaMemset(p, 0, bytes) != cudaSuccess) {
      cudaFree(p);
      return RA_ERR_CUDA;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaFree(p);
      return RA_ERR_CUDA;
    }
    g_status[dev] = p;
    g_num_sms[dev] = sms;
  }
  *status = g_status[dev];
  if (num_sms) *num_sms = g_num_sms[dev];
  return RA_OK;
}

// A work counter for one persistent launch on the current device.
int* next_counter(int* status) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned slot = g_next_slot[dev]++ % kCounterSlots;
  return status + kCounterBase + slot;
}

// Shared validation of the forward calls; fills everything but the tensor
// pointers' derived fields.
ra_status validate_fwd(int batch, int heads, int heads_kv, int seqlen, int d_head, int n_ring,
                       int layout, int causal, float scale, int passes,
                       const int32_t* cu_seqlens, int dtype) {
  if (batch < 1 || heads < 1 || seqlen < 1 || n_ring < 1) return RA_ERR_INVALID;
  if (heads_kv < 1 || heads % heads_kv != 0) return RA_ERR_INVALID;
  if (layout != RA_LAYOUT_CONTIGUOUS && layout != RA_LAYOUT_STRIPED) return RA_ERR_INVALID;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID;
  if (!std::isfinite(scale)) return RA_ERR_INVALID;
  if (passes < 1) return RA_ERR_INVALID;
  if (dtype != RA_F32 && dtype != RA_BF16 && dtype != RA_F16) return RA_ERR_INVALID;
  if (d_head != 16 && d_head != 32 && d_head != 64 && d_head != 128) return RA_ERR_INVALID;
  if (!cu_seqlens && seqlen % n_ring != 0) return RA_ERR_INVALID;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return RA_ERR_INVALID;
  // every row index must fit in 32 bits
  if (!cu_seqlens && (int64_t)batch * seqlen > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  if ((int64_t)batch * heads > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

// The parameters every forward kernel consumes.  q/out rows are tok_stride
// elements apart, k/v rows kv_tok_stride; query head h reads key/value head
// h / (heads / heads_kv).
ra::FwdParams make_params(const void* q, const void* k, const void* v, int64_t tok_stride,
                          int heads_kv, int64_t kv_tok_stride, void* out, float* lse,
                          int batch, int heads, int seqlen, int d_head, int n_ring, int layout,
                          int causal, float scale, int passes, const int32_t* cu_seqlens) {
  ra::FwdParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.tok_stride = tok_stride;
  p.kv_tok_stride = kv_tok_stride;
  p.out = out;
  p.lse = lse;
  p.cu_seqlens = cu_seqlens;
  p.batch = batch;
  p.heads = heads;
  p.heads_kv = heads_kv;
  p.kv_group = heads / heads_kv;
  p.seqlen = seqlen;
  p.d_head = d_head;
  p.n_ring = n_ring;
  p.layout = layout;
  p.causal = causal;
  p.passes = passes < n_ring ? passes : n_ring;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.out_scale = 1.f;
  p.n_qranges = 0;
  // heaviest query ranges first (the kernel launchers refine this per tile size)
  p.order = (causal && layout == RA_LAYOUT_CONTIGUOUS) ? 1 : 0;
  p.qr_per_block = 0;
  if (cu_seqlens) {
    // varlen: seqlen is the total row count of the packed tensors
    p.total_rows = seqlen;
    p.lse_seq_stride = 0;
    p.lse_head_stride = seqlen;
  } else {
    p.total_rows = batch * seqlen;
    p.lse_seq_stride = (int64_t)heads * seqlen;
    p.lse_head_stride = seqlen;
  }
  p.status = nullptr;
  p.work_counter = nullptr;
  p.step = 0;
  p.q_block = p.kv_block = p.step_rows = 0;
  p.accumulate = 0;
  p.step_split = 0;
  p.split_out = nullptr;
  p.split_lse = nullptr;
  p.withhold_q = g_withhold_q.load(std::memory_order_relaxed);
  p.sched_dump = g_sched_dump.load(std::memory_order_relaxed);
  p.sched_dump_cap = g_sched_dump_cap.load(std::memory_order_relaxed);
  return p;
}

// bf16 and fp16 with a nonzero scale run on the tensor cores.  A zero scale
// (a plain average over the allowed keys) has no log2-domain reference there;
// the CUDA-core kernel handles it, and fp32.
bool uses_tc(const ra::FwdParams& p, int dtype, bool force_simt) {
  return (dtype == RA_BF16 || dtype == RA_F16) && !force_simt && p.scale != 0.f;
}

// Launch the kernel for p (status and, on the tensor-core path, a zeroed work
// counter already in p).
ra_status dispatch(const ra::FwdParams& p, int dtype, bool force_simt, cudaStream_t s) {
  cudaError_t e;
  if (uses_tc(p, dtype, force_simt)) {
    if (p.d_head != 64 && p.d_head != 128) return RA_ERR_UNSUPPORTED;
    // TMA row strides are multiples of 16 bytes
    if (((p.tok_stride * 2) & 15) != 0 || ((p.kv_tok_stride * 2) & 15) != 0)
      return RA_ERR_INVALID;
    e = ra::launch_fwd_tc(p, dtype == RA_BF16 ? ra::kFmtBF16 : ra::kFmtF16, s);
  } else {
    e = ra::launch_fwd_simt(p, dtype == RA_F32 ? 0 : (dtype == RA_BF16 ? 1 : 2), s);
  }
  if (e == cudaErrorInvalidValue) return RA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status run_fwd(const ra::FwdParams& params, int dtype, void* stream, bool force_simt) {
  ra::FwdParams p = params;
  int* status = nullptr;
  ra_status st = device_state(&status, nullptr);
  if (st != RA_OK) return st;
  p.status = status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // (ring steps need no counter: their CTAs take items by a static stride,
  // so no memset runs between consecutive step launches, which are
  // programmatic dependents of each other)
  if (uses_tc(p, dtype, force_simt) && !p.step) {
    p.work_counter = next_counter(status);
    if (cudaMemsetAsync(p.work_counter, 0, sizeof(int), s) != cudaSuccess) return RA_ERR_CUDA;
  }
  return dispatch(p, dtype, force_simt, s);
}

}  // namespace

extern "C" {

ra_status ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                        int batch, int heads, int seqlen, int d_head, int n_ring_blocks,
                        int layout, int causal, float softmax_scale, int max_ring_passes,
                        const int32_t* cu_seqlens, int dtype, void* stream) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, dtype);
  if (st != RA_OK) return st;
  const int64_t hd = (int64_t)heads * d_head;
  return run_fwd(make_params(q, k, v, hd, heads, hd, out, lse, batch, heads, seqlen, d_head,
                             n_ring_blocks, layout, causal, softmax_scale, max_ring_passes,
                             cu_seqlens),
                 dtype, stream, false);
}

ra_status ring_attn_fwd_step(const void* q, const void* k, const void* v, float* out,
                             float* lse, int batch, int heads, int seqlen, int d_head,
                             int n_ring_blocks, int layout, int causal, float softmax_scale,
                             int q_block, int kv_block, int accumulate, int dtype,
                             void* stream) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, n_ring_blocks, nullptr, dtype);
  if (st != RA_OK) return st;
  if (q_block < 0 || q_block >= n_ring_blocks || kv_block < 0 || kv_block >= n_ring_blocks)
    return RA_ERR_INVALID;
  if (accumulate != 0 && accumulate != 1) return RA_ERR_INVALID;
  // the step runs on the tensor cores only, with whole 128-row tiles per block
  const int rows = seqlen / n_ring_blocks;
  if (dtype == RA_F32 || softmax_scale == 0.f || rows % 128 != 0) return RA_ERR_UNSUPPORTED;
  // An accumulating step over a block pair that the mask hides entirely
  // leaves the state as it is: nothing to launch.
  const ra::RingGeom g = ra::make_geom(seqlen, n_ring_blocks, layout, causal, n_ring_blocks);
  if (accumulate && ra::classify(g, q_block * rows, (q_block + 1) * rows, kv_block * rows,
                                 (kv_block + 1) * rows) == ra::CLS_EMPTY)
    return RA_OK;
  const int64_t hd = (int64_t)heads * d_head;
  ra::FwdParams p = make_params(q, k, v, hd, heads, hd, out, lse, batch, heads, seqlen, d_head,
                                n_ring_blocks, layout, causal, softmax_scale, n_ring_blocks,
                                nullptr);
  p.step = 1;
  p.q_block = q_block;
  p.kv_block = kv_block;
  p.step_rows = rows;
  p.accumulate = accumulate;
  p.total_rows = batch * rows;
  p.lse_seq_stride = (int64_t)heads * rows;
  p.lse_head_stride = rows;
  p.order = 0;
  return run_fwd(p, dtype, stream, false);
}

}  // extern "C"

namespace {

// The backward: the tensor-core kernels for 16-bit inputs with d_head 64 or
// 128 (unless force_simt), the CUDA-core kernels otherwise.
ra_status run_bwd(const void* q, const void* k, const void* v, const void* out,
                  const float* lse, const void* dout, void* dq, void* dk, void* dv, int batch,
                  int heads, int heads_kv, int seqlen, int d_head, int n_ring_blocks,
                  int layout, int causal, float softmax_scale, int max_ring_passes,
                  const int32_t* cu_seqlens, int dtype, void* stream, bool force_simt) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads_kv, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, dtype);
  if (st != RA_OK) return st;
  ra::FwdParams p = make_params(q, k, v, (int64_t)heads * d_head, heads_kv,
                                (int64_t)heads_kv * d_head, nullptr, const_cast<float*>(lse),
                                batch, heads, seqlen, d_head, n_ring_blocks, layout, causal,
                                softmax_scale, max_ring_passes, cu_seqlens);
  int* status = nullptr;
  int sms = 0;
  st = device_state(&status, &sms);
  if (st != RA_OK) return st;
  p.status = status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  const bool tc = !force_simt && (dtype == RA_BF16 || dtype == RA_F16) &&
                  (d_head == 64 || d_head == 128);
  if (tc) {
    // D = <dO, O> per query row passes from the dq kernel to the dk/dv
    // kernel through stream-ordered scratch in lse layout
    const size_t n_lse = cu_seqlens ? (size_t)heads * seqlen : (size_t)batch * heads * seqlen;
    float* dsum = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void**>(&dsum), n_lse * sizeof(float), s) !=
        cudaSuccess)
      return RA_ERR_CUDA;
    p.work_counter = next_counter(status);
    e = cudaMemsetAsync(p.work_counter, 0, sizeof(int), s);
    if (e == cudaSuccess)
      e = ra::launch_bwd_tc(p, out, dout, dq, dk, dv, dsum,
                            dtype == RA_BF16 ? ra::kFmtBF16 : ra::kFmtF16, sms, s);
    const cudaError_t ef = cudaFreeAsync(dsum, s);
    if (e == cudaSuccess) e = ef;
  } else {
    e = ra::launch_bwd_simt(p, out, dout, dq, dk, dv,
                            dtype == RA_F32 ? 0 : (dtype == RA_BF16 ? 1 : 2), s);
  }
  if (e == cudaErrorInvalidValue) return RA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

extern "C" {

ra_status ring_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv,
                        int batch, int heads, int heads_kv, int seqlen, int d_head,
                        int n_ring_blocks, int layout, int causal, float softmax_scale,
                        int max_ring_passes, const int32_t* cu_seqlens, int dtype,
                        void* stream) {
  return run_bwd(q, k, v, out, lse, dout, dq, dk, dv, batch, heads, heads_kv, seqlen, d_head,
                 n_ring_blocks, layout, causal, softmax_scale, max_ring_passes, cu_seqlens,
                 dtype, stream, false);
}

ra_status ring_attn_bwd_simt(const void* q, const void* k, const void* v, const void* out,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int batch, int heads, int heads_kv, int seqlen, int d_head,
                             int n_ring_blocks, int layout, int causal, float softmax_scale,
                             int max_ring_passes, const int32_t* cu_seqlens, int dtype,
                             void* stream) {
  return run_bwd(q, k, v, out, lse, dout, dq, dk, dv, batch, heads, heads_kv, seqlen, d_head,
                 n_ring_blocks, layout, causal, softmax_scale, max_ring_passes, cu_seqlens,
                 dtype, stream, true);
}

ra_status ring_attn_gqa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                            int batch, int heads, int heads_kv, int seqlen, int d_head,
                            int n_ring_blocks, int layout, int causal, float softmax_scale,
                            int max_ring_passes, const int32_t* cu_seqlens, int dtype,
                            void* stream) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads_kv, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, dtype);
  if (st != RA_OK) return st;
  return run_fwd(make_params(q, k, v, (int64_t)heads * d_head, heads_kv,
                             (int64_t)heads_kv * d_head, out, lse, batch, heads, seqlen, d_head,
                             n_ring_blocks, layout, causal, softmax_scale, max_ring_passes,
                             cu_seqlens),
                 dtype, stream, false);
}

ra_status ring_attn_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
                            int batch, int heads, int heads_kv, int seqlen, int d_head,
                            int n_ring_blocks, int layout, int causal, float softmax_scale,
                            int max_ring_passes, const int32_t* cu_seqlens, float descale_q,
                            float descale_k, float descale_v, void* stream) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID;
  // the shape and mask checks of the 16-bit call
  ra_status st = validate_fwd(batch, heads, heads_kv, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, RA_BF16);
  if (st != RA_OK) return st;
  if (!std::isfinite(descale_q) || !std::isfinite(descale_k) || !std::isfinite(descale_v))
    return RA_ERR_INVALID;
  // the q and k descales fold into the score scale, v's into the output
  const double sc = (double)softmax_scale * descale_q * descale_k;
  if (!std::isfinite((float)sc)) return RA_ERR_INVALID;
  if (d_head != 128 || (float)sc == 0.f) return RA_ERR_UNSUPPORTED;
  ra::FwdParams p = make_params(q, k, v, (int64_t)heads * d_head, heads_kv,
                                (int64_t)heads_kv * d_head, out, lse, batch, heads, seqlen,
                                d_head, n_ring_blocks, layout, causal, (float)sc,
                                max_ring_passes, cu_seqlens);
  p.out_scale = descale_v;
  int* status = nullptr;
  st = device_state(&status, nullptr);
  if (st != RA_OK) return st;
  p.status = status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  p.work_counter = next_counter(status);
  if (cudaMemsetAsync(p.work_counter, 0, sizeof(int), s) != cudaSuccess) return RA_ERR_CUDA;
  const cudaError_t e = ra::launch_fwd_tc(p, ra::kFmtE4M3, s);
  if (e == cudaErrorInvalidValue) return RA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status ring_attn_fwd_simt(const void* q, const void* k, const void* v, void* out,
                             float* lse, int batch, int heads, int seqlen, int d_head,
                             int n_ring_blocks, int layout, int causal, float softmax_scale,
                             int max_ring_passes, const int32_t* cu_seqlens, int dtype,
                             void* stream) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, dtype);
  if (st != RA_OK) return st;
  const int64_t hd = (int64_t)heads * d_head;
  return run_fwd(make_params(q, k, v, hd, heads, hd, out, lse, batch, heads, seqlen, d_head,
                             n_ring_blocks, layout, causal, softmax_scale, max_ring_passes,
                             cu_seqlens),
                 dtype, stream, true);
}

ra_status ring_attn_qkvpacked_fwd(const void* qkv, void* out, float* lse, int batch, int heads,
                                  int seqlen, int d_head, int n_ring_blocks, int layout,
                                  int causal, float softmax_scale, int max_ring_passes,
                                  const int32_t* cu_seqlens, int dtype, void* stream) {
  if (!qkv || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(lse)) return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, dtype);
  if (st != RA_OK) return st;
  const int esize = dtype == RA_F32 ? 4 : 2;
  const int64_t hd = (int64_t)heads * d_head;
  const char* base = static_cast<const char*>(qkv);
  return run_fwd(make_params(base, base + hd * esize, base + 2 * hd * esize, 3 * hd, heads,
                             3 * hd, out, lse, batch, heads, seqlen, d_head, n_ring_blocks,
                             layout, causal, softmax_scale, max_ring_passes, cu_seqlens),
                 dtype, stream, false);
}

ra_status ring_attn_merge(void* out_a, float* lse_a, const void* out_b, const float* lse_b,
                          int batch, int heads, int seqlen, int d_head, int dtype,
                          void* stream) {
  if (!out_a || !lse_a || !out_b || !lse_b) return RA_ERR_INVALID;
  if (!aligned16(out_a) || !aligned16(out_b) || !aligned16(lse_a) || !aligned16(lse_b))
    return RA_ERR_INVALID;
  if (batch < 1 || heads < 1 || seqlen < 1 || d_head < 1) return RA_ERR_INVALID;
  if (dtype != RA_F32 && dtype != RA_BF16 && dtype != RA_F16) return RA_ERR_INVALID;
  const int esize = dtype == RA_F32 ? 4 : 2;
  if ((d_head * esize) % 16 != 0) return RA_ERR_INVALID;
  const int chunks = d_head * esize / 16;
  if (chunks > 32 || (chunks & (chunks - 1)) != 0) return RA_ERR_INVALID;
  if ((int64_t)batch * seqlen * heads > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  int* status = nullptr;
  int sms = 0;
  ra_status st = device_state(&status, &sms);
  if (st != RA_OK) return st;
  cudaError_t e = ra::launch_merge(out_a, lse_a, out_b, lse_b, batch, heads, seqlen, d_head,
                                   dtype == RA_F32 ? 0 : (dtype == RA_BF16 ? 1 : 2), sms,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status ring_attn_status(void* stream) {
  int* status = nullptr;
  ra_status st = device_state(&status, nullptr);
  if (st != RA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return RA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return RA_ERR_CUDA;
  if (v != 0 && cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
  return static_cast<ra_status>(v);
}

int ring_attn_test_withhold_q(int on) {
  return g_withhold_q.exchange(on ? 1 : 0);
}

ra_status ring_attn_test_dump_schedule(int32_t* buf, int64_t capacity) {
  if (capacity < 0 || (buf == nullptr && capacity != 0)) return RA_ERR_INVALID;
  g_sched_dump_cap.store(buf ? capacity : 0, std::memory_order_relaxed);
  g_sched_dump.store(buf, std::memory_order_relaxed);
  return RA_OK;
}

const char* ring_attn_status_string(int status) {
  switch (status) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID: return "RA_ERR_INVALID";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED";
    case RA_ERR_CUDA: return "RA_ERR_CUDA";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT";
  }
  return "RA_ERR_UNKNOWN";
}

int64_t ring_attn_schedule(int seqlen, int n_ring_blocks, int layout, int causal,
                           int max_ring_passes, int q_tile, int kv_tile, int q_tiles_per_item,
                           int32_t* out_q, int32_t* out_kv, int8_t* out_class,
                           int64_t capacity) {
  if (seqlen < 1 || n_ring_blocks < 1 || max_ring_passes < 1 || q_tile < 1 || kv_tile < 1)
    return -1;
  if (q_tiles_per_item != 1 && q_tiles_per_item != 2) return -1;
  if (layout != RA_LAYOUT_CONTIGUOUS && layout != RA_LAYOUT_STRIPED) return -1;
  if (causal != 0 && causal != 1) return -1;
  if (capacity > 0 && (!out_q || !out_kv || !out_class)) return -1;
  const ra::RingGeom g = ra::make_geom(seqlen, n_ring_blocks, layout, causal, max_ring_passes);
  int64_t n = 0;
  auto emit = [&](int qt, int kt, int c) {
    if (n < capacity) {
      out_q[n] = qt;
      out_kv[n] = kt;
      out_class[n] = (int8_t)c;
    }
    ++n;
  };
  const int64_t item_rows = (int64_t)q_tile * q_tiles_per_item;
  for (int64_t i0 = 0; i0 < seqlen; i0 += item_rows) {
    // one work item: query tiles [q0, qm) and [qm, q1), walked together over
    // one key/value stream as the tensor-core kernel's schedule builder does
    const int q0 = (int)i0;
    const int qm = (int)(i0 + q_tile < seqlen ? i0 + q_tile : seqlen);
    const int q1 = (int)(i0 + item_rows < seqlen ? i0 + item_rows : seqlen);
    ra::TileWalk w;
    w.init(g, q0, qm, q1, kv_tile);
    int kt, c0, c1;
    while (w.next(&kt, &c0, &c1)) {
      if (c0 != ra::CLS_EMPTY) emit(q0 / q_tile, kt, c0);
      if (c1 != ra::CLS_EMPTY && qm < q1) emit(q0 / q_tile + 1, kt, c1);
    }
  }
  return n;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward on host buffers (ring_attn_fwd_host).
//
// The heads are processed in chunks.  Each chunk's q/k/v columns are copied
// from the page-locked host tensors into one of two device slots of the
// caller's workspace (a strided 2-D copy: the chunk's heads of every token
// row), the forward runs on the slot, and out/lse go back into the host
// tensors' columns.  Copies in, forwards and copies out run on three streams
// (two library streams per device and the caller's), so chunk c's forward
// overlaps chunk c+1's copy in and chunk c-1's copy out.
// ---------------------------------------------------------------------------

namespace {

constexpr int kHostSlots = 2;
constexpr size_t kHostAlign = 256;

struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t loaded[kHostSlots] = {}, computed[kHostSlots] = {}, drained[kHostSlots] = {};
};
HostPipe g_pipe[kMaxDevices];
// Held while a call enqueues its work: the per-device streams and events are
// shared, and each event must be waited on right after it is recorded.
std::mutex g_pipe_mu;

size_t align_up(size_t x) { return (x + kHostAlign - 1) & ~(kHostAlign - 1); }

// Heads per chunk: the caller's choice, or about eight chunks.
int host_head_chunk(int heads, int head_chunk) {
  if (head_chunk > 0) return head_chunk < heads ? head_chunk : heads;
  const int hc = (heads + 7) / 8;
  return hc < 1 ? 1 : hc;
}

// Byte offsets of q, k, v, out, lse inside one slot, and the slot size.
size_t host_slot_layout(int batch, int seqlen, int hc, int d_head, int esize, size_t off[5]) {
  const size_t tens = (size_t)batch * seqlen * hc * d_head * esize;
  const size_t lse = (size_t)batch * hc * seqlen * sizeof(float);
  size_t o = 0;
  for (int i = 0; i < 4; ++i) {
    off[i] = o;
    o += align_up(tens);
  }
  off[4] = o;
  return o + align_up(lse);
}

bool is_host_pinned(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

bool is_device(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice;
}

ra_status host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kHostSlots; ++i)
      ok = cudaEventCreateWithFlags(&hp.loaded[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.computed[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.drained[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return RA_ERR_CUDA;  // (created handles are kept for the next try)
    hp.ready = true;
  }
  *out = &hp;
  return RA_OK;
}

}  // namespace

extern "C" size_t ring_attn_fwd_host_workspace(int batch, int heads, int seqlen, int d_head,
                                               int dtype, int head_chunk) {
  if (batch < 1 || heads < 1 || seqlen < 1 || d_head < 1) return 0;
  if (dtype != RA_F32 && dtype != RA_BF16 && dtype != RA_F16) return 0;
  const int hc = host_head_chunk(heads, head_chunk);
  const int nchunks = (heads + hc - 1) / hc;
  size_t off[5];
  const size_t slot =
      host_slot_layout(batch, seqlen, hc, d_head, dtype == RA_F32 ? 4 : 2, off);
  return slot * (size_t)(nchunks < kHostSlots ? nchunks : kHostSlots);
}

extern "C" ra_status ring_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                                        float* lse, int batch, int heads, int seqlen,
                                        int d_head, int n_ring_blocks, int layout, int causal,
                                        float softmax_scale, int max_ring_passes, int dtype,
                                        int head_chunk, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !lse || !workspace) return RA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kHostAlign - 1)) != 0) return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, nullptr, dtype);
  if (st != RA_OK) return st;
  if (head_chunk < 0) return RA_ERR_INVALID;
  const int esize = dtype == RA_F32 ? 4 : 2;
  const int hc = host_head_chunk(heads, head_chunk);
  const int nchunks = (heads + hc - 1) / hc;
  const int nslots = nchunks < kHostSlots ? nchunks : kHostSlots;
  size_t off[5];
  const size_t slot_bytes = host_slot_layout(batch, seqlen, hc, d_head, esize, off);
  if (workspace_bytes < slot_bytes * nslots) return RA_ERR_INVALID;
  if (!is_host_pinned(q) || !is_host_pinned(k) || !is_host_pinned(v) || !is_host_pinned(out) ||
      !is_host_pinned(lse) || !is_device(workspace))
    return RA_ERR_INVALID;
  // the per-chunk rows: each token row holds `heads` head vectors
  const size_t row_bytes = (size_t)heads * d_head * esize;
  const size_t rows = (size_t)batch * seqlen;

  HostPipe* hp = nullptr;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  st = host_pipe(&hp);
  if (st != RA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto ck = [](cudaError_t e) { return e == cudaSuccess; };
  // the copy streams start after the work already on the caller's stream
  if (!ck(cudaEventRecord(hp->start, s)) || !ck(cudaStreamWaitEvent(hp->h2d, hp->start, 0)) ||
      !ck(cudaStreamWaitEvent(hp->d2h, hp->start, 0)))
    return RA_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  for (int c = 0; c < nchunks; ++c) {
    const int b = c % nslots;
    const int h0 = c * hc;
    const int nh = heads - h0 < hc ? heads - h0 : hc;
    char* sl = ws + (size_t)b * slot_bytes;
    const size_t w = (size_t)nh * d_head * esize;  // bytes of the chunk in one token row
    const size_t col = (size_t)h0 * d_head * esize;
    // copies in: wait until the slot's previous forward has read its inputs
    if (c >= nslots && !ck(cudaStreamWaitEvent(hp->h2d, hp->computed[b], 0))) return RA_ERR_CUDA;
    const void* src[3] = {q, k, v};
    for (int t = 0; t < 3; ++t)
      if (!ck(cudaMemcpy2DAsync(sl + off[t], w, static_cast<const char*>(src[t]) + col,
                                row_bytes, w, rows, cudaMemcpyHostToDevice, hp->h2d)))
        return RA_ERR_CUDA;
    if (!ck(cudaEventRecord(hp->loaded[b], hp->h2d)) ||
        !ck(cudaStreamWaitEvent(s, hp->loaded[b], 0)))
      return RA_ERR_CUDA;
    // forward: wait until the slot's previous results have been copied out
    if (c >= nslots && !ck(cudaStreamWaitEvent(s, hp->drained[b], 0))) return RA_ERR_CUDA;
    const int64_t hd = (int64_t)nh * d_head;
    ra::FwdParams p = make_params(sl + off[0], sl + off[1], sl + off[2], hd, nh, hd,
                                  sl + off[3], reinterpret_cast<float*>(sl + off[4]), batch, nh,
                                  seqlen, d_head, n_ring_blocks, layout, causal, softmax_scale,
                                  max_ring_passes, nullptr);
    st = run_fwd(p, dtype, stream, false);
    if (st != RA_OK) return st;
    if (!ck(cudaEventRecord(hp->computed[b], s)) ||
        !ck(cudaStreamWaitEvent(hp->d2h, hp->computed[b], 0)))
      return RA_ERR_CUDA;
    // copies out: out columns of every token row, lse rows of every sequence
    if (!ck(cudaMemcpy2DAsync(static_cast<char*>(out) + col, row_bytes, sl + off[3], w, w, rows,
                              cudaMemcpyDeviceToHost, hp->d2h)))
      return RA_ERR_CUDA;
    const size_t lw = (size_t)nh * seqlen * sizeof(float);
    if (!ck(cudaMemcpy2DAsync(lse + (size_t)h0 * seqlen, (size_t)heads * seqlen * sizeof(float),
                              sl + off[4], lw, lw, (size_t)batch, cudaMemcpyDeviceToHost,
                              hp->d2h)))
      return RA_ERR_CUDA;
    if (!ck(cudaEventRecord(hp->drained[b], hp->d2h))) return RA_ERR_CUDA;
  }
  // the caller's stream orders after the last copy out
  if (!ck(cudaEventRecord(hp->done, hp->d2h)) || !ck(cudaStreamWaitEvent(s, hp->done, 0)))
    return RA_ERR_CUDA;
  return RA_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of ring_attn_fwd.
//
// The tensor-core forward needs a little device scratch: the word that
// latches device-side errors and the counter its persistent CTAs claim work
// items from.  ring_attn_fwd takes both from memory the library allocates
// with cudaMalloc on the first call on a device.  ring_attn_fwd_noalloc takes
// them from the fixed array below instead, so it never allocates.
// ---------------------------------------------------------------------------

namespace {

constexpr int kNoAllocWords = 64;       // 256 bytes per device
constexpr int kNoAllocStatus = 0;       // device status word of these calls
constexpr int kNoAllocCounter = 32;     // work counter (own 128-byte line)

}  // namespace

// Lives in every device context that loads the library, until it exits.
static __device__ __align__(256) int g_noalloc_scratch[kNoAllocWords];

namespace {

int* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up once
// per device, with that device current).
ra_status noalloc_scratch(int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return RA_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<int*>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return RA_OK;
}

}  // namespace

extern "C" ra_status ring_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                           void* out, float* lse, int batch, int heads,
                                           int seqlen, int d_head, int n_ring_blocks,
                                           int layout, int causal, float softmax_scale,
                                           int max_ring_passes, const int32_t* cu_seqlens,
                                           int dtype, void* stream) {
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID;
  ra_status st = validate_fwd(batch, heads, heads, seqlen, d_head, n_ring_blocks, layout,
                              causal, softmax_scale, max_ring_passes, cu_seqlens, dtype);
  if (st != RA_OK) return st;
  // Scratch this call needs: the status word and one work counter.  Both
  // sit at fixed offsets, so no problem size can outgrow the array; the check
  // keeps that true if a kernel ever needs more.
  constexpr size_t need = sizeof(int) * (kNoAllocCounter + 1);
  static_assert(need <= sizeof(int) * kNoAllocWords, "no-alloc scratch too small");
  if (need > sizeof(int) * kNoAllocWords) return RA_ERR_UNSUPPORTED;

  int* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != RA_OK) return st;

  const int64_t hd = (int64_t)heads * d_head;
  ra::FwdParams p = make_params(q, k, v, hd, heads, hd, out, lse, batch, heads, seqlen, d_head,
                                n_ring_blocks, layout, causal, softmax_scale, max_ring_passes,
                                cu_seqlens);
  p.status = scratch + kNoAllocStatus;
  p.work_counter = scratch + kNoAllocCounter;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents.  The counter starts from
  // zero for every launch; the status word is left alone, so an error
  // latched by an earlier call stays readable (ring_attn_noalloc_status)
  // until it is read.
  if (cudaMemsetAsync(scratch + kNoAllocCounter, 0, sizeof(int), s) != cudaSuccess)
    return RA_ERR_CUDA;
  return dispatch(p, dtype, false, s);
}

// Reads and clears the status word of the allocation-free calls.  It uses no
// allocation either: a synchronous copy into a local variable and, only when
// an error was latched, a synchronous clear.
extern "C" ra_status ring_attn_noalloc_status(void* stream) {
  int* scratch = nullptr;
  ra_status st = noalloc_scratch(&scratch);
  if (st != RA_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, scratch + kNoAllocStatus, sizeof(int), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return RA_ERR_CUDA;
  if (v != 0 && cudaMemset(scratch + kNoAllocStatus, 0, sizeof(int)) != cudaSuccess)
    return RA_ERR_CUDA;
  return static_cast<ra_status>(v);
}

// ra_fwd_simt.cu -- ring-ordered blockwise attention forward on CUDA cores
// (fp32 arithmetic), for fp32 inputs and as an independent cross-check of
// the tensor-core kernel for bf16 inputs.
//
// Each CTA owns one range of query rows of one (sequence, head) and walks the
// key/value tiles in ring order (ra_sched.h).  Every tile is folded into the
// running state of each query row with the online-softmax rescale: new row
// max, old output and denominator scaled by exp(m_old - m_new), then the
// tile's exponentials added ("Ring Attention simulation" gist, the
// flashattention() update of output, maxima and denominators; "Ring
// Attention" glossary, "Come funziona la ring attention": a running sum of
// exponentiated scores and of weighted values, divided at the end).  Here the
// division by the denominator is deferred to the end, as in the glossary.
//
// A query row is served by 8 threads: the row's dimensions are split over
// d_head / min(d_head, 32) of them (dot products completed with warp
// shuffles) and its keys over the rest (key lanes merged at the end).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ra_common.cuh"
#include "ra_convert.cuh"
#include "ra_params.h"
#include "ra_sched.h"
#include "ra_work.cuh"

namespace ra {

constexpr int kSimtThreads = 128;
constexpr int kSimtBN = 64;

// Thread layout: 8 threads serve one query row, 16 rows per CTA.  The row's
// dimensions are split over TPRD = D / min(D, 32) threads and its keys over
// KL = 8 / TPRD key lanes; lane index within the row = kl * TPRD + part.  A
// thread keeps its own online-softmax state (m, l, O) over the keys of its
// lane; the lanes are merged at the end (max of m, rescale, sum).
template <typename T, int D>
struct SimtShape {
  static constexpr int DPT = D < 32 ? D : 32;           // dims per thread
  static constexpr int TPRD = D / DPT;                  // threads per row (dims)
  static constexpr int KL = 8 / TPRD;                   // key lanes per row
  static constexpr int ROWS = kSimtThreads / 8;         // query rows per CTA
  static constexpr int KPL = kSimtBN / KL;              // keys per lane per tile
  static constexpr int STRIDE = D + 4;                  // smem row stride (floats)
};

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
    fwd_simt_kernel(const FwdParams p) {
  using Sh = SimtShape<T, D>;
  constexpr int DPT = Sh::DPT, TPRD = Sh::TPRD, KL = Sh::KL, ROWS = Sh::ROWS, KPL = Sh::KPL;
  constexpr int BN = kSimtBN, ST = Sh::STRIDE;

  extern __shared__ float smem_f[];
  float* Ks = smem_f;             // [BN][ST]
  float* Vs = smem_f + BN * ST;   // [BN][ST]

  const SeqWork it = find_work(p, ROWS);
  if (!it.live) return;  // uniform across the CTA
  const int base = it.base, L = it.L;
  const int q0 = it.qr * ROWS;
  const int q1 = min(q0 + ROWS, L);

  const int tid = threadIdx.x;
  const int rloc = tid >> 3;
  const int part = tid & (TPRD - 1);
  const int kl = (tid & 7) / TPRD;
  const int sq = q0 + rloc;          // stored row of this thread's query
  const bool valid = sq < L;

  const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
  int rq = 0, tq = 0;
  if (valid) {
    rq = block_of(g, sq);
    tq = token_of(g, sq, rq);
  }

  const int hk = it.h / p.kv_group;  // key/value head read by this query head
  const T* qg = static_cast<const T*>(p.q);
  const T* kg = static_cast<const T*>(p.k);
  const T* vg = static_cast<const T*>(p.v);

  float qr[DPT], o[DPT];
#pragma unroll
  for (int d = 0; d < DPT; ++d) {
    qr[d] = valid ? to_f32(qg[(int64_t)(base + sq) * p.tok_stride + (int64_t)it.h * D +
                              part * DPT + d])
                  : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY;  // running max of this lane's keys, log2 domain
  float l = 0.f;        // running denominator relative to m

  TileWalk walk;
  walk.init(g, q0, q1, q1, BN);
  int kt, c0, c1;
  while (walk.next(&kt, &c0, &c1)) {
    const int k0 = kt * BN;
    const int nk = min(BN, L - k0);
    __syncthreads();  // previous tile fully consumed
    for (int e = tid; e < BN * D; e += kSimtThreads) {
      const int c = e / D, d = e % D;
      float kv = 0.f, vv = 0.f;
      if (c < nk) {
        const int64_t off =
            (int64_t)(base + k0 + c) * p.kv_tok_stride + (int64_t)hk * D + d;
        kv = to_f32(kg[off]);
        vv = to_f32(vg[off]);
      }
      Ks[c * ST + d] = kv;
      Vs[c * ST + d] = vv;
    }
    __syncthreads();

    float s[KPL];
    float tile_max = -INFINITY;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int c = kl + KL * j;
      const float* kr = Ks + c * ST + part * DPT;
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < DPT; ++d) acc = fmaf(qr[d], kr[d], acc);
#pragma unroll
      for (int off = 1; off < TPRD; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      float x = acc * p.scale_log2;
      bool ok = c < nk;
      if (ok && c0 == CLS_PARTIAL && valid) ok = allowed(g, sq, rq, tq, k0 + c);
      x = ok ? x : -INFINITY;
      s[j] = x;
      tile_max = fmaxf(tile_max, x);
    }
    const float m_new = fmaxf(m, tile_max);
    if (m_new == -INFINITY) continue;  // nothing allowed for this lane yet
    const float alpha = exp2f(m - m_new);  // 0 when m == -inf
    l *= alpha;
#pragma unroll
    for (int d = 0; d < DPT; ++d) o[d] *= alpha;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const float pc = exp2f(s[j] - m_new);
      l += pc;
      const float* vr = Vs + (kl + KL * j) * ST + part * DPT;
#pragma unroll
      for (int d = 0; d < DPT; ++d) o[d] = fmaf(pc, vr[d], o[d]);
    }
    m = m_new;
  }

  // merge the KL key lanes of the row: common maximum, rescale, sum
  float m_all = m;
#pragma unroll
  for (int off = TPRD; off < 8; off <<= 1)
    m_all = fmaxf(m_all, __shfl_xor_sync(0xffffffffu, m_all, off));
  const float f = (m == -INFINITY) ? 0.f : exp2f(m - m_all);
  l *= f;
#pragma unroll
  for (int d = 0; d < DPT; ++d) o[d] *= f;
#pragma unroll
  for (int off = TPRD; off < 8; off <<= 1) {
    l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
    for (int d = 0; d < DPT; ++d) o[d] += __shfl_xor_sync(0xffffffffu, o[d], off);
  }

  if (!valid || kl != 0) return;
  T* og = static_cast<T*>(p.out);
  const float inv_l = 1.f / l;
  const int64_t orow = (int64_t)(base + sq) * p.heads * D + (int64_t)it.h * D + part * DPT;
#pragma unroll
  for (int d = 0; d < DPT; ++d) og[orow + d] = from_f32<T>(o[d] * inv_l);
  if (part == 0) {
    const int64_t li = (int64_t)it.b * p.lse_seq_stride + (int64_t)it.h * p.lse_head_stride +
                       (p.cu_seqlens ? base : 0) + sq;
    // lse = ln(l) + m / log2(e), with m in the log2 domain
    p.lse[li] = (m_all + log2f(l)) * 0.69314718055994530942f;
  }
}

template <typename T, int D>
static cudaError_t launch_simt_t(const FwdParams& p, cudaStream_t stream) {
  using Sh = SimtShape<T, D>;
  FwdParams pp = p;
  pp.n_qranges = (p.seqlen + Sh::ROWS - 1) / Sh::ROWS;
  set_striped_order(pp, Sh::ROWS);
  const int64_t grid = work_grid(pp, Sh::ROWS);
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const size_t smem = 2 * kSimtBN * Sh::STRIDE * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fwd_simt_kernel<T, D><<<(unsigned)grid, kSimtThreads, smem, stream>>>(pp);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_d(const FwdParams& p, cudaStream_t stream) {
  switch (p.d_head) {
    case 16: return launch_simt_t<T, 16>(p, stream);
    case 32: return launch_simt_t<T, 32>(p, stream);
    case 64: return launch_simt_t<T, 64>(p, stream);
    case 128: return launch_simt_t<T, 128>(p, stream);
  }
  return cudaErrorInvalidValue;
}

// dtype: 0 = fp32, 1 = bf16, 2 = fp16.  Returns cudaErrorInvalidValue for an
// unsupported head dimension or dtype.
cudaError_t launch_fwd_simt(const FwdParams& p, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch_simt_d<float>(p, stream);
    case 1: return launch_simt_d<__nv_bfloat16>(p, stream);
    case 2: return launch_simt_d<__half>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ra

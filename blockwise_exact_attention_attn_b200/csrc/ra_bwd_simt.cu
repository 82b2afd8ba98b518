// ra_bwd_simt.cu -- backward of the ring-ordered blockwise attention on CUDA
// cores (fp32 arithmetic) for fp32, bf16 and fp16 inputs.
//
// Gradients of sum(dO * O) for O_i = sum_j P_ij v_j, P_ij = exp(s_ij - lse_i),
// s_ij = scale <q_i, k_j> over the allowed keys (plain calculus).  The lse the
// forward returns is reused, so P is recomputed exactly as the forward
// normalised it -- the issue thread "A ring attention with flash attention
// kernel implementation" points out that the returned lse is what makes the
// blockwise method work, and that the backward is where an implementation
// went wrong.
//   D_i = <dO_i, O_i>,  dP_ij = <dO_i, v_j>,  dS_ij = P_ij (dP_ij - D_i)
//   dQ_i = scale sum_j dS_ij k_j
//       (bwd_dq: CTAs of query rows walk their key tiles in ring order)
//   dK_j = scale sum_i dS_ij q_i,  dV_j = sum_i P_ij dO_i
//       (bwd_dkdv: CTAs of key rows walk the query tiles that can see them;
//        with grouped queries they loop over the query heads of their group,
//        so no gradient is accumulated by two CTAs)
//
// Thread layout as in the forward CUDA-core kernel: 8 threads per row, the
// row's dimensions split over TPRD of them (dot products completed with
// shuffles) and the tile's keys (or queries) over the other LANES.
#include <cuda_runtime.h>

#include "ra_common.cuh"
#include "ra_convert.cuh"
#include "ra_params.h"
#include "ra_sched.h"
#include "ra_work.cuh"

namespace ra {

// One backward call.  f describes the forward (inputs, geometry, lse as an
// input, status word); heads_q is the number of query heads.
struct BwdParams {
  FwdParams f;
  int heads_q;
  const void* o;     // forward output [rows, heads_q, D], same dtype as q
  const void* dout;  // [rows, heads_q, D]
  void* dq;          // [rows, heads_q, D]
  void* dk;          // [rows, heads_kv, D]
  void* dv;          // [rows, heads_kv, D]
};

constexpr int kBwdThreads = 128;
constexpr int kBwdBN = 32;  // keys (dq) or queries (dkdv) per shared-memory tile

// kMaxDPT: dims per thread at most.  Both kernels use 16, with 32-row tiles
// and 4 resident CTAs per SM: the kernels are latency-bound, and twice the
// resident warps measured 16 % faster than 32 dims per thread with 64-row
// tiles, despite some spilling at the 128-register cap.
template <int D, int kMaxDPT = 32>
struct BwdShape {
  static constexpr int DPT = D < kMaxDPT ? D : kMaxDPT;  // dims per thread
  static constexpr int TPRD = D / DPT;                 // threads per row (dims)
  static constexpr int LANES = 8 / TPRD;               // key / query lanes per row
  static constexpr int ROWS = kBwdThreads / 8;         // rows per CTA
  static constexpr int PER = kBwdBN / LANES;           // tile entries per lane
  static constexpr int ST = D + 4;                     // smem row stride (floats)
};

template <int TPRD>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int off = 1; off < TPRD; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ int64_t lse_index(const FwdParams& p, const SeqWork& it, int h,
                                             int row) {
  return (int64_t)it.b * p.lse_seq_stride + (int64_t)h * p.lse_head_stride +
         (p.cu_seqlens ? it.base : 0) + row;
}

template <typename T, int D>
__global__ void __launch_bounds__(kBwdThreads, 4) bwd_dq_kernel(const BwdParams bp) {
  using Sh = BwdShape<D, 16>;
  constexpr int DPT = Sh::DPT, TPRD = Sh::TPRD, LANES = Sh::LANES, ROWS = Sh::ROWS;
  constexpr int PER = Sh::PER, BN = kBwdBN, ST = Sh::ST;
  const FwdParams& p = bp.f;
  extern __shared__ float smem_f[];
  float* Ks = smem_f;             // [BN][ST]
  float* Vs = smem_f + BN * ST;   // [BN][ST]

  const SeqWork it = find_work(p, ROWS);
  if (!it.live) return;  // uniform across the CTA
  const int base = it.base, L = it.L;
  const int q0 = it.qr * ROWS, q1 = min(q0 + ROWS, L);
  const int tid = threadIdx.x;
  const int rloc = tid >> 3, part = tid & (TPRD - 1), lane = (tid & 7) / TPRD;
  const int sq = q0 + rloc;
  const bool valid = sq < L;
  const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
  int rq = 0, tq = 0;
  if (valid) {
    rq = block_of(g, sq);
    tq = token_of(g, sq, rq);
  }
  const int hk = it.h / p.kv_group;
  const int64_t qoff = (int64_t)(base + sq) * p.tok_stride + (int64_t)it.h * D + part * DPT;
  const int64_t ooff = (int64_t)(base + sq) * bp.heads_q * D + (int64_t)it.h * D + part * DPT;
  const T* qg = static_cast<const T*>(p.q);
  const T* kg = static_cast<const T*>(p.k);
  const T* vg = static_cast<const T*>(p.v);
  const T* og = static_cast<const T*>(bp.o);
  const T* dog = static_cast<const T*>(bp.dout);

  float qr[DPT], dor[DPT], dq[DPT];
  float dsum = 0.f;
#pragma unroll
  for (int d = 0; d < DPT; ++d) {
    qr[d] = valid ? to_f32(qg[qoff + d]) : 0.f;
    dor[d] = valid ? to_f32(dog[ooff + d]) : 0.f;
    dsum = fmaf(dor[d], valid ? to_f32(og[ooff + d]) : 0.f, dsum);
    dq[d] = 0.f;
  }
  const float Drow = row_sum<TPRD>(dsum);
  const float lse2 = valid ? p.lse[lse_index(p, it, it.h, sq)] * 1.4426950408889634f : 0.f;

  TileWalk walk;
  walk.init(g, q0, q1, q1, BN);
  int kt, c0, c1;
  while (walk.next(&kt, &c0, &c1)) {
    const int k0 = kt * BN;
    const int nk = min(BN, L - k0);
    __syncthreads();  // previous tile fully consumed
    for (int e = tid; e < BN * D; e += kBwdThreads) {
      const int c = e / D, d = e % D;
      float kv = 0.f, vv = 0.f;
      if (c < nk) {
        const int64_t off = (int64_t)(base + k0 + c) * p.kv_tok_stride + (int64_t)hk * D + d;
        kv = to_f32(kg[off]);
        vv = to_f32(vg[off]);
      }
      Ks[c * ST + d] = kv;
      Vs[c * ST + d] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < PER; ++j) {
      const int c = lane + LANES * j;
      const float* kr = Ks + c * ST + part * DPT;
      const float* vr = Vs + c * ST + part * DPT;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int d = 0; d < DPT; ++d) {
        s = fmaf(qr[d], kr[d], s);
        dp = fmaf(dor[d], vr[d], dp);
      }
      s = row_sum<TPRD>(s);
      dp = row_sum<TPRD>(dp);
      bool ok = valid && c < nk;
      if (ok && c0 == CLS_PARTIAL) ok = allowed(g, sq, rq, tq, k0 + c);
      const float P = ok ? ex2_approx(fmaf(s, p.scale_log2, -lse2)) : 0.f;
      const float ds = P * (dp - Drow);
#pragma unroll
      for (int d = 0; d < DPT; ++d) dq[d] = fmaf(ds, kr[d], dq[d]);
    }
  }
  // sum the key lanes of the row
#pragma unroll
  for (int off = TPRD; off < 8; off <<= 1) {
#pragma unroll
    for (int d = 0; d < DPT; ++d) dq[d] += __shfl_xor_sync(0xffffffffu, dq[d], off);
  }
  if (!valid || lane != 0) return;
  T* dqg = static_cast<T*>(bp.dq);
#pragma unroll
  for (int d = 0; d < DPT; ++d) dqg[ooff + d] = from_f32<T>(dq[d] * p.scale);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBwdThreads, 4) bwd_dkdv_kernel(const BwdParams bp) {
  using Sh = BwdShape<D, 16>;
  constexpr int DPT = Sh::DPT, TPRD = Sh::TPRD, LANES = Sh::LANES, ROWS = Sh::ROWS;
  constexpr int PER = Sh::PER, BQ = kBwdBN, ST = Sh::ST;
  const FwdParams& p = bp.f;  // heads = key/value heads here (work decode)
  extern __shared__ float smem_f[];
  float* Qs = smem_f;                 // [BQ][ST]
  float* dOs = smem_f + BQ * ST;      // [BQ][ST]
  float* Os = smem_f + 2 * BQ * ST;   // [BQ][ST]
  float* lse_s = smem_f + 3 * BQ * ST;  // [BQ], log2 units
  float* D_s = lse_s + BQ;              // [BQ]

  const SeqWork it = find_work(p, ROWS);
  if (!it.live) return;  // uniform across the CTA
  const int base = it.base, L = it.L;
  const int hk = it.h;
  const int k_lo = it.qr * ROWS, k_hi = min(k_lo + ROWS, L);
  const int tid = threadIdx.x;
  const int rloc = tid >> 3, part = tid & (TPRD - 1), lane = (tid & 7) / TPRD;
  const int sk = k_lo + rloc;
  const bool valid = sk < L;
  const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
  const int64_t koff = (int64_t)(base + sk) * p.kv_tok_stride + (int64_t)hk * D + part * DPT;
  const T* qg = static_cast<const T*>(p.q);
  const T* kg = static_cast<const T*>(p.k);
  const T* vg = static_cast<const T*>(p.v);
  const T* og = static_cast<const T*>(bp.o);
  const T* dog = static_cast<const T*>(bp.dout);

  float kr[DPT], vr[DPT], dk[DPT], dv[DPT];
#pragma unroll
  for (int d = 0; d < DPT; ++d) {
    kr[d] = valid ? to_f32(kg[koff + d]) : 0.f;
    vr[d] = valid ? to_f32(vg[koff + d]) : 0.f;
    dk[d] = dv[d] = 0.f;
  }

  const int nqt = (L + BQ - 1) / BQ;
  for (int h = hk * p.kv_group; h < (hk + 1) * p.kv_group; ++h) {
    for (int qt = 0; qt < nqt; ++qt) {
      const int q_lo = qt * BQ, q_hi = min(q_lo + BQ, L);
      const int cls = classify(g, q_lo, q_hi, k_lo, k_hi);
      if (cls == CLS_EMPTY) continue;  // uniform across the CTA
      __syncthreads();  // previous tile fully consumed
      for (int e = tid; e < BQ * D; e += kBwdThreads) {
        const int c = e / D, d = e % D;
        float qv = 0.f, dov = 0.f, ov = 0.f;
        if (q_lo + c < q_hi) {
          const int64_t row = base + q_lo + c;
          qv = to_f32(qg[row * p.tok_stride + (int64_t)h * D + d]);
          const int64_t oo = (row * bp.heads_q + h) * D + d;
          dov = to_f32(dog[oo]);
          ov = to_f32(og[oo]);
        }
        Qs[c * ST + d] = qv;
        dOs[c * ST + d] = dov;
        Os[c * ST + d] = ov;
      }
      __syncthreads();
      if (tid < BQ) {
        float acc = 0.f;
        for (int d = 0; d < D; ++d) acc = fmaf(dOs[tid * ST + d], Os[tid * ST + d], acc);
        D_s[tid] = acc;
        lse_s[tid] = q_lo + tid < q_hi
                         ? p.lse[lse_index(p, it, h, q_lo + tid)] * 1.4426950408889634f
                         : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int j = 0; j < PER; ++j) {
        const int c = lane + LANES * j;
        const float* qrow = Qs + c * ST + part * DPT;
        const float* drow = dOs + c * ST + part * DPT;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < DPT; ++d) {
          s = fmaf(qrow[d], kr[d], s);
          dp = fmaf(drow[d], vr[d], dp);
        }
        s = row_sum<TPRD>(s);
        dp = row_sum<TPRD>(dp);
        const int i = q_lo + c;
        bool ok = valid && i < q_hi;
        if (ok && cls == CLS_PARTIAL) {
          const int ri = block_of(g, i);
          ok = allowed(g, i, ri, token_of(g, i, ri), sk);
        }
        const float P = ok ? ex2_approx(fmaf(s, p.scale_log2, -lse_s[c])) : 0.f;
        const float ds = P * (dp - D_s[c]);
#pragma unroll
        for (int d = 0; d < DPT; ++d) {
          dv[d] = fmaf(P, drow[d], dv[d]);
          dk[d] = fmaf(ds, qrow[d], dk[d]);
        }
      }
    }
  }
  // sum the query lanes of the row
#pragma unroll
  for (int off = TPRD; off < 8; off <<= 1) {
#pragma unroll
    for (int d = 0; d < DPT; ++d) {
      dk[d] += __shfl_xor_sync(0xffffffffu, dk[d], off);
      dv[d] += __shfl_xor_sync(0xffffffffu, dv[d], off);
    }
  }
  if (!valid || lane != 0) return;
  const int64_t goff = (int64_t)(base + sk) * p.heads * D + (int64_t)hk * D + part * DPT;
  T* dkg = static_cast<T*>(bp.dk);
  T* dvg = static_cast<T*>(bp.dv);
#pragma unroll
  for (int d = 0; d < DPT; ++d) {
    dkg[goff + d] = from_f32<T>(dk[d] * p.scale);
    dvg[goff + d] = from_f32<T>(dv[d]);
  }
}

template <typename T, int D>
static cudaError_t launch_bwd_t(const BwdParams& bp, cudaStream_t stream) {
  using Sh = BwdShape<D, 16>;
  using ShK = BwdShape<D, 16>;
  static_assert(Sh::ROWS == ShK::ROWS && Sh::ST == ShK::ST, "shared tile shapes");
  // dq: work items over (sequence, query head, 16 query rows)
  BwdParams pq = bp;
  pq.f.n_qranges = (bp.f.seqlen + Sh::ROWS - 1) / Sh::ROWS;
  const int64_t gq = work_grid(pq.f, Sh::ROWS);
  // dk/dv: work items over (sequence, key/value head, 16 key rows), natural
  // order (in causal contiguous inputs the first keys are seen the most)
  BwdParams pk = bp;
  pk.f.heads = bp.f.heads_kv;
  pk.f.order = 0;
  pk.f.n_qranges = pq.f.n_qranges;
  const int64_t gk = work_grid(pk.f, Sh::ROWS);
  if (gq > 0x7fffffffLL || gk > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const size_t smem_q = 2 * kBwdBN * Sh::ST * sizeof(float);
  const size_t smem_k = (3 * kBwdBN * Sh::ST + 2 * kBwdBN) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_k);
  if (e != cudaSuccess) return e;
  if (gq > 0) bwd_dq_kernel<T, D><<<(unsigned)gq, kBwdThreads, smem_q, stream>>>(pq);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (gk > 0) bwd_dkdv_kernel<T, D><<<(unsigned)gk, kBwdThreads, smem_k, stream>>>(pk);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_bwd_d(const BwdParams& bp, cudaStream_t stream) {
  switch (bp.f.d_head) {
    case 16: return launch_bwd_t<T, 16>(bp, stream);
    case 32: return launch_bwd_t<T, 32>(bp, stream);
    case 64: return launch_bwd_t<T, 64>(bp, stream);
    case 128: return launch_bwd_t<T, 128>(bp, stream);
  }
  return cudaErrorInvalidValue;
}

// dtype: 0 = fp32, 1 = bf16, 2 = fp16.
cudaError_t launch_bwd_simt(const FwdParams& f, const void* o, const void* dout, void* dq,
                            void* dk, void* dv, int dtype, cudaStream_t stream) {
  BwdParams bp;
  bp.f = f;
  bp.heads_q = f.heads;
  bp.o = o;
  bp.dout = dout;
  bp.dq = dq;
  bp.dk = dk;
  bp.dv = dv;
  switch (dtype) {
    case 0: return launch_bwd_d<float>(bp, stream);
    case 1: return launch_bwd_d<__nv_bfloat16>(bp, stream);
    case 2: return launch_bwd_d<__half>(bp, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ra

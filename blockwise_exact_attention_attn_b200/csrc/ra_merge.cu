// ra_merge.cu -- fold a partial attention result (out_b, lse_b) into
// (out_a, lse_a) in place.
//
// The issue thread "A ring attention with flash attention kernel
// implementation" explains that the returned log-sum-exp is what makes
// blockwise evaluation possible (partial results over disjoint key sets are
// combined through it), and that a key/value-outer ring pass stores outputs
// and lse and passes them back in.  The combination used here is the stable
// log-add-exp:
//     lse = hi + log1p(exp(lo - hi)),   hi/lo = max/min(lse_a, lse_b)
//     out = exp(lse_a - lse) * out_a + exp(lse_b - lse) * out_b
// with the empty-side cases handled exactly.
//
// Memory-bound: every 16-byte chunk of out_a/out_b is read once and out_a
// written once; one warp covers whole rows (d_head * sizeof(T) / 16 chunks per
// row divides 32), so the row's lse is read by its lanes before lane 0 of the
// row overwrites it (separated by __syncwarp).  Loads of several chunk groups
// are issued together, ahead of the arithmetic, to keep HBM busy.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ra_common.cuh"

namespace ra {

// Division of 32-bit unsigned n by a fixed divisor d >= 1 with one high
// multiply (Granlund & Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (t + ((n - t) >> 1)) >> (l - 1)
// where t = mulhi(m, n) (l = 0, i.e. d = 1, is handled separately).
struct FastDiv {
  uint32_t d, m, sh;
  void init(uint32_t div) {
    d = div;
    uint32_t l = 0;
    while ((1ull << l) < div) ++l;
    sh = l;
    m = l == 0 ? 0u : (uint32_t)((((1ull << l) - div) << 32) / div + 1);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    if (sh == 0) return n;
    const uint32_t t = __umulhi(m, n);
    return (t + ((n - t) >> 1)) >> (sh - 1);
  }
};

struct MergeParams {
  void* out_a;
  float* lse_a;
  const void* out_b;
  const float* lse_b;
  int batch, heads, seqlen, d_head;
  int64_t rows;     // batch * seqlen * heads (< 2^31, checked by the host)
  int log2_chunks;  // 16-byte chunks per row = 1 << log2_chunks (divides 32)
  FastDiv div_heads, div_seqlen;
};

__device__ __forceinline__ void merge_weights(float la, float lb, float* wa, float* wb,
                                              float* lse) {
  const bool ea = la == -INFINITY, eb = lb == -INFINITY;
  if (ea && eb) { *wa = 0.f; *wb = 0.f; *lse = -INFINITY; return; }
  if (ea) { *wa = 0.f; *wb = 1.f; *lse = lb; return; }
  if (eb) { *wa = 1.f; *wb = 0.f; *lse = la; return; }
  const float hi = fmaxf(la, lb), lo = fminf(la, lb);
  const float s = hi + log1pf(expf(lo - hi));
  *wa = expf(la - s);
  *wb = expf(lb - s);
  *lse = s;
}

// fp32: a chunk is 4 floats
__device__ __forceinline__ uint4 combine_f32(uint4 x, uint4 y, float wa, float wb) {
  uint4 r;
  r.x = __float_as_uint(wa * __uint_as_float(x.x) + wb * __uint_as_float(y.x));
  r.y = __float_as_uint(wa * __uint_as_float(x.y) + wb * __uint_as_float(y.y));
  r.z = __float_as_uint(wa * __uint_as_float(x.z) + wb * __uint_as_float(y.z));
  r.w = __float_as_uint(wa * __uint_as_float(x.w) + wb * __uint_as_float(y.w));
  return r;
}

// Pairs of 16-bit values to and from float2.
__device__ __forceinline__ float2 to_float2(__nv_bfloat162 v) { return __bfloat1622float2(v); }
__device__ __forceinline__ float2 to_float2(__half2 v) { return __half22float2(v); }
template <typename T2>
__device__ __forceinline__ T2 from_float2(float x, float y);
template <>
__device__ __forceinline__ __nv_bfloat162 from_float2<__nv_bfloat162>(float x, float y) {
  return __floats2bfloat162_rn(x, y);
}
template <>
__device__ __forceinline__ __half2 from_float2<__half2>(float x, float y) {
  return __floats2half2_rn(x, y);
}

// 16-bit elements (T2 = __nv_bfloat162 or __half2): a chunk is 8 values
template <typename T2>
__device__ __forceinline__ uint4 combine_16(uint4 x, uint4 y, float wa, float wb) {
  uint4 r;
  const T2* xa = reinterpret_cast<const T2*>(&x);
  const T2* yb = reinterpret_cast<const T2*>(&y);
  T2* rr = reinterpret_cast<T2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = to_float2(xa[i]);
    const float2 fb = to_float2(yb[i]);
    rr[i] = from_float2<T2>(wa * fa.x + wb * fb.x, wa * fa.y + wb * fb.y);
  }
  return r;
}

// Chunk groups (32 consecutive 16-byte chunks, one per lane) each warp
// handles per loop trip.  All their loads -- both lse values and both output
// chunks -- are issued before any result is computed, so a thread keeps
// groups * 32 bytes of outputs in flight instead of waiting for the lse round
// trip before each chunk.  Measured on B200 over 2, 4 and 8 groups: 8 is
// fastest for fp32 rows, 4 for 16-bit rows (same bytes per row in flight).
template <int kType>
constexpr int merge_groups() {
  return kType == 0 ? 8 : 4;
}
constexpr int kMergeThreads = 256;

// kType: 0 = fp32, 1 = bf16, 2 = fp16
template <int kType>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeParams p) {
  constexpr int G = merge_groups<kType>();
  const int64_t total = p.rows << p.log2_chunks;
  const uint32_t cmask = (1u << p.log2_chunks) - 1u;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  uint4* oa = static_cast<uint4*>(p.out_a);
  const uint4* ob = static_cast<const uint4*>(p.out_b);
  for (int64_t wbase = warp0 * (32 * G); wbase < total; wbase += nwarps * (32 * G)) {
    uint4 x[G], y[G];
    float la[G], lb[G];
    int64_t li[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int64_t chunk = wbase + g * 32 + lane;
      x[g] = y[g] = make_uint4(0u, 0u, 0u, 0u);
      la[g] = lb[g] = 0.f;
      li[g] = 0;
      if (chunk < total) {
        const uint32_t row = (uint32_t)(chunk >> p.log2_chunks);
        // out rows are [batch, seqlen, heads]; lse is [batch, heads, seqlen]
        const uint32_t bs = p.div_heads.div(row);
        const uint32_t h = row - bs * (uint32_t)p.heads;
        const uint32_t b = p.div_seqlen.div(bs);
        const uint32_t s = bs - b * (uint32_t)p.seqlen;
        li[g] = ((int64_t)b * p.heads + h) * p.seqlen + s;
        la[g] = p.lse_a[li[g]];
        lb[g] = __ldcs(p.lse_b + li[g]);
        x[g] = oa[chunk];
        y[g] = __ldcs(ob + chunk);
      }
    }
    // a row lies inside one group (its chunks divide 32 and groups are
    // 32-aligned): every lane has read the row's lse_a before the row's first
    // lane overwrites it
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int64_t chunk = wbase + g * 32 + lane;
      if (chunk < total) {
        float wa, wb, lse;
        merge_weights(la[g], lb[g], &wa, &wb, &lse);
        uint4 r;
        if (la[g] == -INFINITY && lb[g] == -INFINITY) {
          r = make_uint4(0u, 0u, 0u, 0u);  // no key on either side
        } else if (lb[g] == -INFINITY) {
          r = x[g];  // b empty: a passes through bit for bit
        } else if (la[g] == -INFINITY) {
          r = y[g];  // a empty: b passes through bit for bit
        } else if (kType == 0) {
          r = combine_f32(x[g], y[g], wa, wb);
        } else if (kType == 1) {
          r = combine_16<__nv_bfloat162>(x[g], y[g], wa, wb);
        } else {
          r = combine_16<__half2>(x[g], y[g], wa, wb);
        }
        __stcs(oa + chunk, r);
        if (((uint32_t)chunk & cmask) == 0u) p.lse_a[li[g]] = lse;
      }
    }
  }
}

// dtype: 0 = fp32, 1 = bf16, 2 = fp16.  The host checks that the chunks per row are a
// power of two dividing 32 and that rows < 2^31.
cudaError_t launch_merge(void* out_a, float* lse_a, const void* out_b, const float* lse_b,
                         int batch, int heads, int seqlen, int d_head, int dtype,
                         int num_sms, cudaStream_t stream) {
  MergeParams p;
  p.out_a = out_a;
  p.lse_a = lse_a;
  p.out_b = out_b;
  p.lse_b = lse_b;
  p.batch = batch;
  p.heads = heads;
  p.seqlen = seqlen;
  p.d_head = d_head;
  p.rows = (int64_t)batch * seqlen * heads;
  const int chunks = d_head * (dtype == 0 ? 4 : 2) / 16;
  p.log2_chunks = 0;
  while ((1 << p.log2_chunks) < chunks) ++p.log2_chunks;
  p.div_heads.init((uint32_t)heads);
  p.div_seqlen.init((uint32_t)seqlen);
  const int64_t total = p.rows * chunks;
  if (total == 0) return cudaSuccess;
  const int threads = kMergeThreads;
  // every block resident at once: the SM count times the blocks one SM holds
  // (a grid-stride loop covers the rest)
  static int per_sm[3] = {0, 0, 0};
  if (per_sm[dtype] == 0) {
    int n = 0;
    cudaError_t e = dtype == 0   ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                       &n, merge_kernel<0>, threads, 0)
                    : dtype == 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                       &n, merge_kernel<1>, threads, 0)
                                 : cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                       &n, merge_kernel<2>, threads, 0);
    if (e != cudaSuccess) return e;
    per_sm[dtype] = n > 0 ? n : 1;
  }
  int64_t blocks = (int64_t)num_sms * per_sm[dtype];
  const int groups = dtype == 0 ? merge_groups<0>() : merge_groups<1>();
  const int64_t need = (total + threads * groups - 1) / (threads * groups);
  if (need < blocks) blocks = need;
  if (dtype == 0)
    merge_kernel<0><<<(unsigned)blocks, threads, 0, stream>>>(p);
  else if (dtype == 1)
    merge_kernel<1><<<(unsigned)blocks, threads, 0, stream>>>(p);
  else
    merge_kernel<2><<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ra

// ra_bwd_tc.cu -- backward of the ring-ordered blockwise attention on the
// sm_100a tensor cores (tcgen05 + TMEM), bf16 or fp16 inputs, fp32
// accumulation: dq, dk, dv of sum(dout * out).
//
// The gradients are plain calculus on out_i = sum_j P_ij v_j with P_ij =
// exp(scale q_i.k_j - lse_i) over the allowed keys: dV = P^T dO, dP = dO V^T,
// dS = P (dP - D) with D_i = <dO_i, O_i>, dQ = scale dS K, dK = scale dS^T Q.
// P is recomputed from the forward's lse, the quantity the issue thread "A
// ring attention with flash attention kernel implementation" says the
// blockwise method keeps (and the backward is the part that thread found
// wrong in an implementation).  Two kernels, so every gradient element has
// one writer and no atomics are needed:
//
//  bwd_dq_kernel (query-outer, the forward's ring walk over 128-key tiles,
//   one 128-row query tile per item): per kv tile S = Q K^T and dP = dO V^T
//   into tensor memory; the gradient warps read both, form dS = P (dP - D)
//   and write it as 16-bit over the dP columns they have read; then
//   dQ += dS K takes dS from tensor memory.  dP alternates between two
//   buffers, so S and dP of the next kv tile are computed while the
//   gradient warps work on this one.  It also writes D per query row for
//   the second kernel.
//   warps 0-7   gradient warps: warp w owns query rows 32 (w % 4) .. + 31
//               (its TMEM lane quadrant) and keys 64 (w / 4) .. + 63
//   warp  8     TMA producer: Q, dO per item; K and V tiles into rings of
//               their own (V(t) is free after dP(t), K(t) only after dQ(t))
//   warp  9     MMA issuer;  warp 10 schedule builder;  warp 11 idle
//   TMEM: S 128 | dP_A 128 | dP_B 128 | dQ D.
//
//  bwd_dkdv_kernel (key/value-outer): a CTA owns 128 keys of one (sequence,
//   key/value head), one TMEM lane each, and walks the 128-row query tiles
//   of every query head of its group that see them, one tile a step:
//   S^T = K Q^T and dP^T = V dO^T into tensor memory, the gradient warps
//   write P^T and dS^T = P^T (dP^T - D) as 16-bit over the score columns
//   they have read, then dV += P^T dO and dK += dS^T Q take them from tensor
//   memory; the next step's dP^T is computed while the gradient warps work.
//   warps 0-3 / 4-7  gradient warps for query columns 0-63 / 64-127
//   warp  8          TMA producer (and the per-tile lse / D vectors)
//   warp  9          MMA issuer;  warp 10 schedule builder;  warp 11 idle
//   TMEM: S^T 128 | dP^T 128 | dV D | dK D.
// Every wait is bounded like the forward's: an expired wait latches
// ST_TIMEOUT, the CTA drains what it issued and frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ra_common.cuh"
#include "ra_list.cuh"
#include "ra_params.h"
#include "ra_sched.h"
#include "ra_work.cuh"

namespace ra {
namespace tcb {

constexpr int BM = 128;   // query rows per item (one TMEM lane each)
constexpr int BN = 128;   // keys per kv tile
constexpr int kThreads = 384;
constexpr int kProducer = 8, kMma = 9, kBuilder = 10;  // warp 11 idle
constexpr int kConsumers = 10;  // producer, issuer, 8 gradient warps
// K and V tiles in two rings: V(t) is free once dP(t) has run, K(t) only
// after dQ(t), so K gets one slot more and both are loaded a step ahead.
constexpr int kKSlots = 3, kVSlots = 2;
constexpr int kRegsGrad = 184, kRegsControl = 136;  // 256*184 + 128*136 = 384*168
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanel = 128 * 128;          // 128 rows x 128 B
  static constexpr int kTile = kPanels * kPanel;    // a Q, dO, K or V tile
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kTile;
  static constexpr int kKOff = 2 * kTile;           // K ring
  static constexpr int kVOff = kKOff + kKSlots * kTile;  // V ring
  static constexpr int kListOff = kVOff + kVSlots * kTile;
  static constexpr int kCtrlOff = kListOff + kListBufs * kListChunk * 4;
  static constexpr int kSmemBytes = kCtrlOff + 512 + 1024;
  static constexpr uint32_t kColS = 0;      // S
  static constexpr uint32_t kColDP = 128;   // dP buffer b at 128 + 128 b (dS over it)
  static constexpr uint32_t kColDQ = 384;   // dQ
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kColDQ + D <= kTmemCols, "tensor memory budget");
};

struct Ctrl {
  uint64_t q_full, q_free;
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t v_full[kVSlots], v_empty[kVSlots];
  uint64_t s_full, s_free, ds_full;
  uint64_t dq_full, dq_free;
  uint64_t list_full[kListBufs], list_empty[kListBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Ctrl) <= 512, "control block");

struct Maps {
  CUtensorMap q, dout, k, v;
};

// Launch parameters of both kernels.  f holds the forward's inputs,
// geometry, lse, status word and work counter; for the dK/dV kernel f.heads
// counts the key/value heads (the work decode runs over them).
struct Params {
  FwdParams f;
  int heads_q;      // query heads
  const void* o;    // forward output, q's layout
  const void* dout; // q's layout
  void* dq;         // q's layout
  void* dk;         // k's layout
  void* dv;         // v's layout
  float* dsum;      // D = <dO, O> per query row, lse layout (written by bwd_dq_kernel)
};

__device__ __forceinline__ int entry_tile(int e) { return e >> 4; }
__device__ __forceinline__ int entry_cls(int e, int i) { return (e >> (2 * i)) & 3; }

// Leading allowed columns of kv tile [k0, k0 + nk) for query (rq, tq) when the
// tile lies in ring block rk (allowed keys of one block form a prefix).
__device__ __forceinline__ int block_limit(const RingGeom& g, int rq, int tq, int rk, int k0,
                                           int nk) {
  if (!pass_ok(g, rq, rk)) return 0;
  if (!g.causal) return nk;
  int last;
  if (g.layout == LAYOUT_CONTIGUOUS) {
    last = tq;
  } else {
    if (tq < rk) return 0;
    last = block_start(g, rk) + (tq - rk) / g.N;
  }
  const int lim = last - k0 + 1;
  return lim < 0 ? 0 : (lim > nk ? nk : lim);
}

__device__ __forceinline__ uint32_t bit_range(int lo, int hi) {
  const uint32_t upto = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}

// Allowed columns of the tile as two 32-bit masks.
__device__ __forceinline__ void tile_mask(uint32_t mw[2], const FwdParams& p, int L, bool valid,
                                          int cls, int rq, int tq, int k0, int nk) {
  if (!valid) {
    mw[0] = mw[1] = 0u;
    return;
  }
  // causal rows of the contiguous layout without a pass limit see every
  // stored key up to their own position tq: one interval, no block lookups
  const bool prefix =
      cls == CLS_FULL || (p.causal && p.layout == LAYOUT_CONTIGUOUS && p.passes >= p.n_ring);
  if (prefix) {
    const int lim = cls == CLS_FULL ? nk : min(nk, tq - k0 + 1);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int n = min(max(lim - 32 * w, 0), 32);
      mw[w] = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
    }
    return;
  }
  const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
  mw[0] = mw[1] = 0u;
  const int kend = k0 + nk;
  int c = k0;
  for (int rk = block_of(g, k0); c < kend && rk < g.N; ++rk) {
    const int be = min(block_start(g, rk + 1), kend);
    if (be <= c) continue;
    const int a = c - k0, bnd = a + block_limit(g, rq, tq, rk, c, be - c);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int lo = max(a - 32 * w, 0), hi = min(bnd - 32 * w, 32);
      if (hi > lo) mw[w] |= bit_range(lo, hi);
    }
    c = be;
  }
}

// S = A B^T for the query tile: A (128 query rows) and B (128 key rows),
// both K-major in 128-byte-swizzled panels kPanel apart; M = N = 128,
// K = D in steps of 16 (start address field + panel * kPanel / 16 +
// 2 * (kk % 4)).
template <int D>
__device__ __forceinline__ void issue_rows(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc) {
  using C = Cfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)((kk >> 2) * (C::kPanel >> 4) + (kk & 3) * 2);
    umma_ss(d_tmem, adesc + off, bdesc + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// dQ (+)= dS K: A = dS in tensor memory, 16-bit pairs (keys 0-63 in columns
// [a, a + 32), keys 64-127 in [a + 64, a + 96)), B = the K tile MN-major
// (N = D in panels kPanel apart; 8-key groups 1024 bytes apart).  Step kk
// covers 16 keys.
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                         uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk)
    umma_ts(d_tmem, a_tmem + (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8),
            bdesc + (uint64_t)(kk * 128), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

template <int D, int kFmt>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const Params bp, const __grid_constant__ Maps maps, int n_items,
                  int claim_limit) {
  using C = Cfg<D>;
  const FwdParams& p = bp.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + C::kCtrlOff);
  volatile int* abort_flag = &ctrl->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int* list = reinterpret_cast<int*>(smem + C::kListOff);

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->q_full, 1);
    mbar_init(&ctrl->q_free, 1);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&ctrl->k_full[s], 1);
      mbar_init(&ctrl->k_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(&ctrl->v_full[s], 1);
      mbar_init(&ctrl->v_empty[s], 1);
    }
    mbar_init(&ctrl->s_full, 1);
    mbar_init(&ctrl->s_free, 256);
    mbar_init(&ctrl->ds_full, 256);
    mbar_init(&ctrl->dq_full, 1);
    mbar_init(&ctrl->dq_free, 256);
    mbar_init(&ctrl->drain, 1);
    for (int b = 0; b < kListBufs; ++b) {
      mbar_init(&ctrl->list_full[b], 1);
      mbar_init(&ctrl->list_empty[b], kConsumers);
    }
    ctrl->abort = 0;
    mbar_fence_init();
  }
  if (warp == kMma) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the dK/dV kernel that follows on the stream is a programmatic dependent:
  // it may start loading its tiles as this launch's CTAs finish (it reads D,
  // the only thing this kernel writes that it needs, after griddepcontrol.wait)
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t tmem = ctrl->tmem_base;
  ListReader rd;
  rd.list = smem_u32(list);
  rd.full = ctrl->list_full;
  rd.empty = ctrl->list_empty;

  if (warp >= 8) {
    regs_dec<kRegsControl>();
    if (warp == kBuilder) {
      // ---------------------------------------------------------- schedule
      ListWriter wr;
      wr.list = smem_u32(list);
      wr.full = ctrl->list_full;
      wr.empty = ctrl->list_empty;
      wr.abort = abort_flag;
      bool ok = true;
      auto put = [&](int v) -> bool { return wr.put(v); };
      auto flush = [&]() -> bool { return wr.flush(); };
      int j = 0;
      while (ok) {
        if (claim_limit > 0 && j >= claim_limit) {
          if (lane == 0) ok = put(kAllDone) && flush();
          break;
        }
        if (lane == 0 && j > 0) {
          ok = flush();
          if (ok) ok = mbar_wait(&ctrl->q_full, (j - 1) & 1, abort_flag);
        }
        int item = 0;
        if (lane == 0 && ok) item = atomicAdd(p.work_counter, 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        item = __shfl_sync(0xffffffffu, item, 0);
        if (!ok) break;
        if (item >= n_items) {
          if (lane == 0) ok = put(kAllDone) && flush();
          break;
        }
        const SeqWork it = find_work_item(p, BM, item);
        if (!it.live) continue;
        if (lane == 0) {
          const int q0 = it.qr * BM, q1 = min(q0 + BM, it.L);
          const RingGeom g = make_geom(it.L, p.n_ring, p.layout, p.causal, p.passes);
          ok = put_item(wr, item, it);
          // one query range: the walk's second sub-range is empty
          TileWalk walk;
          walk.init(g, q0, q1, q1, BN);
          int kt, c0, c1;
          while (ok && walk.next(&kt, &c0, &c1)) ok = put((kt << 4) | c0);
          if (ok) ok = put(kItemEnd);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        ++j;
      }
      if (lane == 0 && !ok) {
        *abort_flag = 1;
        latch_status(p.status, ST_TIMEOUT);
      }
      __syncwarp();
    } else if (warp == kProducer) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.dout);
        tma_prefetch_desc(&maps.k);
        tma_prefetch_desc(&maps.v);
      }
      int n = 0, k = 0, nq = 0;
      bool ok = true;
      int nv = 0;  // V tiles issued (n counts K tiles)
      // K and V of kv tile `row`, each into the next slot of its ring
      auto load_kv = [&](int hk, int row) -> bool {
        const int ks = n % kKSlots, vs = nv % kVSlots;
        if (n >= kKSlots &&
            !mbar_wait(&ctrl->k_empty[ks], ((n / kKSlots) - 1) & 1, abort_flag))
          return false;
        mbar_arrive_expect_tx(&ctrl->k_full[ks], C::kTile);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(smem + C::kKOff + ks * C::kTile + pn * C::kPanel, &maps.k,
                      &ctrl->k_full[ks], pn * 64, hk, row);
        ++n;
        if (nv >= kVSlots &&
            !mbar_wait(&ctrl->v_empty[vs], ((nv / kVSlots) - 1) & 1, abort_flag))
          return false;
        mbar_arrive_expect_tx(&ctrl->v_full[vs], C::kTile);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(smem + C::kVOff + vs * C::kTile + pn * C::kPanel, &maps.v,
                      &ctrl->v_full[vs], pn * 64, hk, row);
        ++nv;
        return true;
      };
      while (ok) {
        int h = 0;
        if (lane == 0) ok = rd.next(&h, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        h = __shfl_sync(0xffffffffu, h, 0);
        if (!ok || h == kAllDone) break;
        if (lane == 0) {
          SeqWork it;
          ok = read_item<false>(rd, &it, abort_flag);
          const int hk = it.h / p.kv_group;
          int e = -1;
          if (ok) ok = rd.next(&e, abort_flag);
          // the item's first (K, V) enters the ring before Q and dO wait for
          // the previous item's last S and dP MMAs (q_free)
          if (ok && e >= 0) ok = load_kv(hk, it.base + entry_tile(e) * BN);
          if (ok && k > 0) ok = mbar_wait(&ctrl->q_free, (k - 1) & 1, abort_flag);
          if (ok) {
            const int q_row = it.base + it.qr * BM;
            mbar_arrive_expect_tx(&ctrl->q_full, 2 * C::kTile);
            for (int pn = 0; pn < C::kPanels; ++pn) {
              tma_load_3d(smem + C::kQOff + pn * C::kPanel, &maps.q, &ctrl->q_full, pn * 64,
                          it.h, q_row);
              tma_load_3d(smem + C::kDOOff + pn * C::kPanel, &maps.dout, &ctrl->q_full, pn * 64,
                          it.h, q_row);
            }
            ++nq;
          }
          while (ok && e >= 0) {
            ok = rd.next(&e, abort_flag);
            if (ok && e >= 0) ok = load_kv(hk, it.base + entry_tile(e) * BN);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        ++k;
      }
      if (lane == 0 && !ok) {
        *abort_flag = 1;
        latch_status(p.status, ST_TIMEOUT);
        // let the copies already issued land before the CTA can exit
        for (int u = (n > kKSlots ? n - kKSlots : 0); u < n; ++u)
          mbar_wait(&ctrl->k_full[u % kKSlots], (u / kKSlots) & 1, nullptr);
        for (int u = (nv > kVSlots ? nv - kVSlots : 0); u < nv; ++u)
          mbar_wait(&ctrl->v_full[u % kVSlots], (u / kVSlots) & 1, nullptr);
        if (nq > 0) mbar_wait(&ctrl->q_full, (nq - 1) & 1, nullptr);
      }
      __syncwarp();
    } else if (warp == kMma) {
      // ---------------------------------------------------------- MMA issuer
      // Per kv tile t: S(t+1) and dP(t+1) as soon as the gradient warps have
      // read S(t) and dP(t) (s_free), dP into the buffer dP(t) does not use;
      // then dQ += dS(t) K(t) once dS(t) is in tensor memory (ds_full).  One
      // thread issues everything, so dP(t+2) overwrites dS(t) only after the
      // dQ MMA of tile t has read it.  V(t)'s slot is released after dP(t),
      // K(t)'s after dQ(t).  S/dP number n and dQ number n share buffer n % 2
      // and are kv tile n of the rings.
      const uint32_t idesc_s = idesc_f16kind_f32(BM, BN, 0, kFmt);
      constexpr uint32_t idesc_q = idesc_f16kind_f32(BM, D, 1, kFmt);
      const uint64_t qdesc = smem_desc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
      const uint64_t dodesc = smem_desc_sw128(smem_u32(smem + C::kDOOff), 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + C::kKOff), 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + C::kVOff), 16, 1024);
      const uint64_t kmn0 = smem_desc_sw128(smem_u32(smem + C::kKOff), C::kPanel, 1024);
      constexpr uint64_t kSlotStep = (uint64_t)(C::kTile >> 4);
      const uint32_t tS = tmem + C::kColS;
      const uint32_t tDQ = tmem + C::kColDQ;
      uint32_t ns = 0, nd = 0;
      int k = 0;
      bool ok = true, issued_any = false;
      // S and dP of kv tile ns; S overwrites the previous tile's, which the
      // gradient warps must have read
      auto issue_sdp = [&]() {
        if (ns > 0) {
          ok = mbar_wait(&ctrl->s_free, (ns - 1) & 1, abort_flag);
          if (!ok) return;
        }
        const int ks = (int)(ns % kKSlots), vs = (int)(ns % kVSlots);
        ok = mbar_wait(&ctrl->k_full[ks], (ns / kKSlots) & 1, abort_flag);
        if (!ok) return;
        tc_fence_after();
        issue_rows<D>(tS, qdesc, kdesc0 + ks * kSlotStep, idesc_s);
        ok = mbar_wait(&ctrl->v_full[vs], (ns / kVSlots) & 1, abort_flag);
        if (!ok) return;
        tc_fence_after();
        issue_rows<D>(tmem + C::kColDP + 128u * (ns & 1), dodesc, vdesc0 + vs * kSlotStep,
                      idesc_s);
        umma_commit(&ctrl->v_empty[vs]);
        umma_commit(&ctrl->s_full);
        ++ns;
        issued_any = true;
      };
      while (ok) {
        int h = 0;
        if (lane == 0) ok = rd.next(&h, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        h = __shfl_sync(0xffffffffu, h, 0);
        if (!ok || h == kAllDone) break;
        if (lane == 0) {
          SeqWork skip;
          ok = read_item<false>(rd, &skip, abort_flag);
          if (ok) ok = mbar_wait(&ctrl->q_full, k & 1, abort_flag);
          tc_fence_after();
          bool started = false;
          int e = -1;
          if (ok) ok = rd.next(&e, abort_flag);
          if (ok && e >= 0) {
            issue_sdp();
            while (ok) {
              int en = -1;
              ok = rd.next(&en, abort_flag);
              if (!ok) break;
              if (en >= 0) {
                issue_sdp();
                if (!ok) break;
              } else {
                umma_commit(&ctrl->q_free);  // every S/dP of this item issued
              }
              ok = mbar_wait(&ctrl->ds_full, nd & 1, abort_flag);
              if (!ok) break;
              tc_fence_after();
              if (!started && k > 0) {
                // the previous item's dQ has been read out
                ok = mbar_wait(&ctrl->dq_free, (k - 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
              }
              const int ks = (int)(nd % kKSlots);
              issue_dq(tDQ, tmem + C::kColDP + 128u * (nd & 1), kmn0 + ks * kSlotStep, idesc_q,
                       started);
              umma_commit(&ctrl->k_empty[ks]);
              ++nd;
              started = true;
              if (en < 0) break;
            }
          } else if (ok) {
            umma_commit(&ctrl->q_free);
          }
          if (ok) {
            if (!started && k > 0) {
              // no dQ MMA this item: the read-out of the previous one must
              // still finish before dq_full is signalled again
              ok = mbar_wait(&ctrl->dq_free, (k - 1) & 1, abort_flag);
              tc_fence_after();
            }
            if (ok) umma_commit(&ctrl->dq_full);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        ++k;
      }
      if (lane == 0 && !ok) {
        *abort_flag = 1;
        latch_status(p.status, ST_TIMEOUT);
        if (issued_any) {
          umma_commit(&ctrl->drain);
          mbar_wait(&ctrl->drain, 0, nullptr);
        }
      }
      __syncwarp();
    }
  } else {
    regs_inc<kRegsGrad>();
    // ---------------------------------------------------------- gradient warps
    const int half = warp >> 2;   // keys [64 half, 64 half + 64) of each kv tile
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + 64 * half;
    constexpr int kOutCols = D / 2;  // dQ columns this warp writes out
    const uint32_t tDQ = tmem + lane_off + C::kColDQ + kOutCols * half;
    uint32_t sphase = 0, nstep = 0;
    int k = 0;
    bool ok = true;
    while (true) {
      int h;
      ok = rd.next_warp(&h, abort_flag);
      if (!ok || h == kAllDone) break;
      SeqWork it;
      ok = read_item<true>(rd, &it, abort_flag);
      if (!ok) break;
      const int L = it.L;
      const int sq = it.qr * BM + r;
      const bool valid = sq < L;
      int rq = 0, tq = 0;
      if (valid) {
        const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
        rq = block_of(g, sq);
        tq = token_of(g, sq, rq);
      }
      const int64_t li = (int64_t)it.b * p.lse_seq_stride + (int64_t)it.h * p.lse_head_stride +
                         (p.cu_seqlens ? it.base : 0) + sq;
      const int64_t roff = ((int64_t)(it.base + sq) * bp.heads_q + it.h) * D;
      // D = <dO, O> for the warp's 32 rows, fp32 over the 16-bit inputs.  The
      // lanes read them together: an instruction covers two rows, 16 bytes
      // per lane (whole lines), and each row is summed over its 16 lanes by
      // shuffles and handed to the row's own lane.  Both warps of a row form
      // it; the first writes it for the dK/dV kernel.
      float dsum = 0.f, lse2 = 0.f;
      {
        const int sub = lane >> 4, ch = lane & 15;  // row of the pair, 16-byte chunk
        const int row0 = sq - lane;                  // the warp's first row
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int sr = row0 + 2 * i + sub;
          float part = 0.f;
          if (sr < L && ch < D / 8) {
            const int64_t ro = ((int64_t)(it.base + sr) * bp.heads_q + it.h) * D;
            const uint4 a = reinterpret_cast<const uint4*>(
                static_cast<const uint16_t*>(bp.dout) + ro)[ch];
            const uint4 b =
                reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(bp.o) + ro)[ch];
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float a0, a1, b0, b1;
              if (kFmt == kFmtBF16) {
                a0 = __uint_as_float(av[j] << 16);
                a1 = __uint_as_float(av[j] & 0xffff0000u);
                b0 = __uint_as_float(bv[j] << 16);
                b1 = __uint_as_float(bv[j] & 0xffff0000u);
              } else {
                const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&av[j]));
                const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&bv[j]));
                a0 = fa.x; a1 = fa.y; b0 = fb.x; b1 = fb.y;
              }
              part = fmaf(a0, b0, part);
              part = fmaf(a1, b1, part);
            }
          }
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
          const float t0 = __shfl_sync(0xffffffffu, part, 0);
          const float t1 = __shfl_sync(0xffffffffu, part, 16);
          if (lane == 2 * i) dsum = t0;
          if (lane == 2 * i + 1) dsum = t1;
        }
      }
      if (valid) {
        lse2 = p.lse[li] * 1.4426950408889634f;
        if (bp.dsum && half == 0) bp.dsum[li] = dsum;
      }
      bool any = false;
      while (true) {
        int e;
        ok = rd.next_warp(&e, abort_flag);
        if (!ok || e < 0) break;
        const int cls = entry_cls(e, 0);
        ok = warp_wait(&ctrl->s_full, sphase, abort_flag);
        sphase ^= 1;
        if (!ok) break;
        tc_fence_after();
        // this warp's 64 keys of S and of dP (buffer nstep % 2)
        const uint32_t tDP = tmem + lane_off + C::kColDP + 128u * (nstep & 1) + 64 * half;
        float s[64], dp[64];
        {
          uint32_t* sr = reinterpret_cast<uint32_t*>(s);
          uint32_t* dr = reinterpret_cast<uint32_t*>(dp);
          RA_TMEM_LD32(tS, sr);
          RA_TMEM_LD32(tS + 32, (sr + 32));
          RA_TMEM_LD32(tDP, dr);
          RA_TMEM_LD32(tDP + 32, (dr + 32));
          tmem_wait_ld();
        }
        tc_fence_before();
        mbar_arrive(&ctrl->s_free);
        const int k0 = entry_tile(e) * BN + 64 * half;
        const int nk = min(64, L - k0);
        uint32_t mw[2];
        tile_mask(mw, p, L, valid, cls, rq, tq, k0, nk);
        // P = ex2(S scale - lse) and dS = P (dP - D) in paired fp32
        // instructions (the same roundings as the scalar forms)
        const uint64_t sc2 = f32x2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nl2 = f32x2_pack(-lse2, -lse2), nd2 = f32x2_pack(-dsum, -dsum);
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c0 = 2 * j, c1 = 2 * j + 1;
          const bool a0 = (mw[c0 >> 5] >> (c0 & 31)) & 1u;
          const bool a1 = (mw[c1 >> 5] >> (c1 & 31)) & 1u;
          float y0, y1;
          ffma2(s[c0], s[c1], sc2, nl2, y0, y1);
          const float p0 = a0 ? ex2_approx(y0) : 0.f;
          const float p1 = a1 ? ex2_approx(y1) : 0.f;
          const uint64_t r2 = mul2(f32x2_pack(p0, p1), add2(f32x2_pack(dp[c0], dp[c1]), nd2));
          pk[j] = pack_x2<kFmt>(f32x2_lo(r2), f32x2_hi(r2));
        }
        // dS over the first 32 of this warp's dP columns (already read)
        RA_TMEM_ST32(tDP, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctrl->ds_full);
        ++nstep;
        any = true;
      }
      if (!ok) break;
      // epilogue: this warp's half of the row's dQ, scaled, in the input format
      ok = warp_wait(&ctrl->dq_full, k & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kOutCols; c += 32) {
        uint32_t o[32];
        if (any) {
          RA_TMEM_LD32(tDQ + c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pk[j] = pack_x2<kFmt>(__uint_as_float(o[2 * j]) * p.scale,
                                __uint_as_float(o[2 * j + 1]) * p.scale);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(bp.dq) + roff +
                                                kOutCols * half + c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&ctrl->dq_free);
      ++k;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) latch_status(p.status, ST_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) !=
            cudaSuccess ||
        qres != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, heads, D] 16-bit view, box 64 x 1 x box_rows, 128-byte swizzle.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int heads, int D,
                     int64_t tok_stride, int fmt, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)tok_stride * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt =
      fmt == kFmtBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return enc(map, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int D, int kFmt>
static cudaError_t launch_t(const Params& bp_in, cudaStream_t stream, int num_sms) {
  using C = Cfg<D>;
  Params bp = bp_in;
  FwdParams& p = bp.f;
  p.n_qranges = (p.seqlen + BM - 1) / BM;
  const int64_t items = work_grid(p, BM);
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const bool per_item = p.causal && !p.cu_seqlens;
  const int64_t grid = per_item ? items : (items < num_sms ? items : num_sms);
  Maps maps;
  if (!make_map(&maps.q, p.q, p.total_rows, p.heads, D, p.tok_stride, kFmt, BM) ||
      !make_map(&maps.dout, bp.dout, p.total_rows, bp.heads_q, D, (int64_t)bp.heads_q * D,
                kFmt, BM) ||
      !make_map(&maps.k, p.k, p.total_rows, p.heads_kv, D, p.kv_tok_stride, kFmt, BN) ||
      !make_map(&maps.v, p.v, p.total_rows, p.heads_kv, D, p.kv_tok_stride, kFmt, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D, kFmt>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D, kFmt><<<(unsigned)grid, kThreads, C::kSmemBytes, stream>>>(
      bp, maps, (int)items, per_item ? 1 : 0);
  return cudaGetLastError();
}


namespace kv {

// Key/value-outer kernel: one CTA per 128 keys of a (sequence, key/value
// head), 128-query steps.  Per step t the tensor core computes
//   S^T(t) = K Q(t)^T and dP^T(t) = V dO(t)^T     (M = 128 keys, N = 128)
// into tensor memory; the gradient warps read dP^T first (its columns are
// then free: dp_free), then the scores chunk by chunk, and write P^T and
// dS^T as 16-bit pairs over the score columns they have just read; then
//   dV += P^T(t) dO(t) and dK += dS^T(t) Q(t)     (A from tensor memory).
// dP^T(t+1) is issued as soon as dP^T(t) has been read, so it runs while
// the gradient warps compute; S^T(t+1) follows dV(t) and dK(t) from the
// same issuing thread (the tensor core runs one thread's MMAs in issue
// order, so it overwrites P^T(t), dS^T(t) only after they have been read),
// and the commit announcing step t+1 covers both of its products.
// Gradient warp w works on key rows 32 (w % 4) .. + 31 (its TMEM lane
// quadrant) and query columns 64 (w / 4) .. + 63, in two chunks of 32
// queries: chunk c's P^T goes to the first 16 of the 32 score columns it
// came from, its dS^T to the other 16, so no warp writes a column another
// has not read yet (an MMA step takes its 16 queries' 8 columns from the
// chunk that holds them).
constexpr int BK = 128;  // keys per CTA
constexpr int BQ = 128;  // query rows per step
constexpr int kMma = 9;
constexpr int kKvConsumers = 10;  // producer, issuer, 8 gradient warps
constexpr int kQStages = 2;       // (Q, dO) pairs in the ring

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kKPanel = BK * 128;      // 16 KB: 128 rows x 128 B
  static constexpr int kKTile = kPanels * kKPanel;
  static constexpr int kQPanel = BQ * 128;      // 16 KB: 128 rows x 128 B
  static constexpr int kQTile = kPanels * kQPanel;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kKTile;
  static constexpr int kRingOff = kVOff + kKTile;  // slot s: Q at +0, dO at +kQTile
  static constexpr int kVecOff = kRingOff + kQStages * 2 * kQTile;  // per slot: lse2, D
  static constexpr int kListOff = kVecOff + kQStages * 2 * BQ * 4;
  static constexpr int kCtrlOff = kListOff + kListBufs * kListChunk * 4;
  static constexpr int kSmemBytes = kCtrlOff + 512 + 1024;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kColDK + D <= kTmemCols, "tensor memory budget");
};

struct Ctrl {
  uint64_t kv_full, kv_free;
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t s_full, dp_free, pds_full;
  uint64_t acc_full, acc_free;
  uint64_t list_full[kListBufs], list_empty[kListBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Ctrl) <= 512, "control block");

struct Maps {
  CUtensorMap k, v, q, dout;
};

// entries: (query head within the group << 24) | (query tile << 2) | class
__device__ __forceinline__ int entry_g(int e) { return e >> 24; }
__device__ __forceinline__ int entry_qt(int e) { return (e >> 2) & 0x3fffff; }
__device__ __forceinline__ int entry_cls(int e) { return e & 3; }

// S^T-like product: A (128 key rows, K-major, panels kKPanel apart) x B
// (128 query rows, K-major, panels kQPanel apart): M = N = 128, K = D.
template <int D>
__device__ __forceinline__ void issue_kq(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc) {
  using C = Cfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t ao = (uint64_t)((kk >> 2) * (C::kKPanel >> 4) + (kk & 3) * 2);
    const uint64_t bo = (uint64_t)((kk >> 2) * (C::kQPanel >> 4) + (kk & 3) * 2);
    umma_ss(d_tmem, adesc + ao, bdesc + bo, idesc, kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A B with A (128 keys x 128 queries, 16-bit pairs) in tensor
// memory -- queries 32 c .. 32 c + 31 in columns [a + 32 c, a + 32 c + 16)
// -- and B a 128-query tile MN-major (N = D in panels kQPanel apart).  P^T
// sits at a = the score columns, dS^T at a + 16.  Step kk covers 16 queries.
__device__ __forceinline__ void issue_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < BQ / 16; ++kk)
    umma_ts(d_tmem, a_tmem + (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8),
            bdesc + (uint64_t)(kk * 128), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

template <int D, int kFmt>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const Params bp, const __grid_constant__ Maps maps, int n_items) {
  using C = Cfg<D>;
  const FwdParams& p = bp.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + C::kCtrlOff);
  volatile int* abort_flag = &ctrl->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int* list = reinterpret_cast<int*>(smem + C::kListOff);

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->kv_full, 1);
    mbar_init(&ctrl->kv_free, 1);
    for (int s = 0; s < kQStages; ++s) {
      // two arrivals: the copies' expect_tx and the producer once the
      // slot's lse / D vectors are written
      mbar_init(&ctrl->q_full[s], 2);
      mbar_init(&ctrl->q_empty[s], 1);
    }
    mbar_init(&ctrl->s_full, 1);
    mbar_init(&ctrl->dp_free, 256);
    mbar_init(&ctrl->pds_full, 256);
    mbar_init(&ctrl->acc_full, 1);
    mbar_init(&ctrl->acc_free, 256);
    mbar_init(&ctrl->drain, 1);
    for (int b = 0; b < kListBufs; ++b) {
      mbar_init(&ctrl->list_full[b], 1);
      mbar_init(&ctrl->list_empty[b], kKvConsumers);
    }
    ctrl->abort = 0;
    mbar_fence_init();
  }
  if (warp == kMma) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  ListReader rd;
  rd.list = smem_u32(list);
  rd.full = ctrl->list_full;
  rd.empty = ctrl->list_empty;

  if (warp >= 8) {
    regs_dec<kRegsControl>();
    if (warp == kBuilder) {
      // ---------------------------------------------------------- schedule
      // Per item: its header, then for every query head of the key/value
      // head's group every query tile that sees the key tile, with its
      // class.  The CTAs take the items in waves of one per CTA, every other
      // wave in reverse CTA order (one wave when the grid has a CTA per item).
      ListWriter wr;
      wr.list = smem_u32(list);
      wr.full = ctrl->list_full;
      wr.empty = ctrl->list_empty;
      wr.abort = abort_flag;
      bool ok = true;
      int claims = 0;
      while (ok) {
        const int wave_pos =
            (claims & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x;
        const int item = claims * (int)gridDim.x + wave_pos;
        ++claims;
        if (item >= n_items) break;
        const SeqWork it = find_work_item(p, BK, item);
        if (lane == 0) {
          if (it.live) {
            const int k_lo = it.qr * BK, k_hi = min(k_lo + BK, it.L);
            const RingGeom g = make_geom(it.L, p.n_ring, p.layout, p.causal, p.passes);
            ok = put_item(wr, item, it);
            const int nqt = (it.L + BQ - 1) / BQ;
            // contiguous causal: the query tiles that end before the first key
            // see none of it (query and key positions are the stored rows), so
            // the walk starts at the tile that holds row k_lo; every other
            // tile is classified exactly (a few divisions per call, which the
            // leading empty tiles would otherwise spend before the first entry)
            const int qt0 = (g.causal && g.layout == LAYOUT_CONTIGUOUS) ? k_lo / BQ : 0;
            for (int gq = 0; ok && gq < p.kv_group; ++gq)
              for (int qt = qt0; ok && qt < nqt; ++qt) {
                const int q_lo = qt * BQ, q_hi = min(q_lo + BQ, it.L);
                const int cls = classify(g, q_lo, q_hi, k_lo, k_hi);
                if (cls != CLS_EMPTY) ok = wr.put((gq << 24) | (qt << 2) | cls);
              }
            if (ok) ok = wr.put(kItemEnd);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (lane == 0) {
        if (ok) ok = wr.put(kAllDone);
        if (ok) ok = wr.flush();
        if (!ok) {
          *abort_flag = 1;
          latch_status(p.status, ST_TIMEOUT);
        }
      }
      __syncwarp();
    } else if (warp == kProducer) {
      // ---------------------------------------------------------- producer
      // The whole warp reads the list.  Per query tile lane 0 issues the Q
      // and dO copies, then the lanes stage the tile's lse (log2 units) and
      // D into the slot's vectors and lane 0 arrives once more.
      if (lane == 0) {
        tma_prefetch_desc(&maps.k);
        tma_prefetch_desc(&maps.v);
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.dout);
      }
      int n = 0, k = 0, nkv = 0;
      bool ok = true;
      bool dq_done = false;  // the dq kernel (which writes D) has completed
      while (ok) {
        int h = 0;
        ok = rd.next_warp(&h, abort_flag);
        if (!ok || h == kAllDone) break;
        SeqWork it;
        ok = read_item<true>(rd, &it, abort_flag);
        if (ok && k > 0) ok = warp_wait(&ctrl->kv_free, (k - 1) & 1, abort_flag);
        if (!ok) break;
        if (lane == 0) {
          const int k_row = it.base + it.qr * BK;
          mbar_arrive_expect_tx(&ctrl->kv_full, 2 * C::kKTile);
          for (int pn = 0; pn < C::kPanels; ++pn) {
            tma_load_3d(smem + C::kKOff + pn * C::kKPanel, &maps.k, &ctrl->kv_full, pn * 64,
                        it.h, k_row);
            tma_load_3d(smem + C::kVOff + pn * C::kKPanel, &maps.v, &ctrl->kv_full, pn * 64,
                        it.h, k_row);
          }
        }
        ++nkv;
        while (ok) {
          int e = 0;
          ok = rd.next_warp(&e, abort_flag);
          if (!ok || e < 0) break;
          const int slot = n % kQStages;
          if (n >= kQStages) {
            ok = warp_wait(&ctrl->q_empty[slot], ((n / kQStages) - 1) & 1, abort_flag);
            if (!ok) break;
          }
          const int q_lo = entry_qt(e) * BQ;
          const int hq = it.h * p.kv_group + entry_g(e);  // query head
          // the copies first, so their latency overlaps the vector loads
          if (lane == 0) {
            uint8_t* dst = smem + C::kRingOff + slot * 2 * C::kQTile;
            const int q_row = it.base + q_lo;
            mbar_arrive_expect_tx(&ctrl->q_full[slot], 2 * C::kQTile);
            for (int pn = 0; pn < C::kPanels; ++pn) {
              tma_load_3d(dst + pn * C::kQPanel, &maps.q, &ctrl->q_full[slot], pn * 64, hq,
                          q_row);
              tma_load_3d(dst + C::kQTile + pn * C::kQPanel, &maps.dout, &ctrl->q_full[slot],
                          pn * 64, hq, q_row);
            }
          }
          float* vec = reinterpret_cast<float*>(smem + C::kVecOff) + slot * 2 * BQ;
          // this launch may have started before the dq kernel finished (a
          // programmatic dependent): D is read only after it has completed
          // (returns at once when the launch is not a dependent)
          if (!dq_done) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            dq_done = true;
          }
#pragma unroll
          for (int u = 0; u < BQ / 32; ++u) {
            const int j = lane + 32 * u;
            const int qi = q_lo + j;
            float l2 = 0.f, dd = 0.f;
            if (qi < it.L) {
              const int64_t li = (int64_t)it.b * p.lse_seq_stride +
                                 (int64_t)hq * p.lse_head_stride +
                                 (p.cu_seqlens ? it.base : 0) + qi;
              l2 = p.lse[li] * 1.4426950408889634f;
              dd = bp.dsum[li];
            }
            // stored negated: the gradient warps add them
            vec[j] = -l2;
            vec[BQ + j] = -dd;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctrl->q_full[slot]);
          ++n;
        }
        ++k;
      }
      if (lane == 0 && !ok) {
        *abort_flag = 1;
        latch_status(p.status, ST_TIMEOUT);
        for (int u = (n > kQStages ? n - kQStages : 0); u < n; ++u)
          mbar_wait(&ctrl->q_full[u % kQStages], (u / kQStages) & 1, nullptr);
        if (nkv > 0) mbar_wait(&ctrl->kv_full, (nkv - 1) & 1, nullptr);
      }
      __syncwarp();
    } else if (warp == kMma) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc_s = idesc_f16kind_f32(BK, BQ, 0, kFmt);
      constexpr uint32_t idesc_a = idesc_f16kind_f32(BK, D, 1, kFmt);
      const uint64_t kdesc = smem_desc_sw128(smem_u32(smem + C::kKOff), 16, 1024);
      const uint64_t vdesc = smem_desc_sw128(smem_u32(smem + C::kVOff), 16, 1024);
      const uint64_t qk0 = smem_desc_sw128(smem_u32(smem + C::kRingOff), 16, 1024);
      const uint64_t dok0 = smem_desc_sw128(smem_u32(smem + C::kRingOff + C::kQTile), 16, 1024);
      const uint64_t qmn0 = smem_desc_sw128(smem_u32(smem + C::kRingOff), C::kQPanel, 1024);
      const uint64_t domn0 =
          smem_desc_sw128(smem_u32(smem + C::kRingOff + C::kQTile), C::kQPanel, 1024);
      constexpr uint64_t kSlotStep = (uint64_t)((2 * C::kQTile) >> 4);
      const uint32_t tS = tmem + C::kColS, tDP = tmem + C::kColDP;
      const uint32_t tDV = tmem + C::kColDV, tDK = tmem + C::kColDK;
      uint32_t npd = 0;
      int n = 0, k = 0;
      bool ok = true, issued_any = false;
      auto take = [&]() -> int {
        const int slot = n % kQStages;
        ok = mbar_wait(&ctrl->q_full[slot], (n / kQStages) & 1, abort_flag);
        ++n;
        if (ok) tc_fence_after();
        return slot;
      };
      // an item's first step: its dP^T once the previous step's has been
      // read (its S^T follows that step's dV and dK in issue order)
      auto issue_first = [&](int slot) {
        if (npd > 0) {
          ok = mbar_wait(&ctrl->dp_free, (npd - 1) & 1, abort_flag);
          if (!ok) return;
          tc_fence_after();
        }
        issue_kq<D>(tDP, vdesc, dok0 + slot * kSlotStep, idesc_s);
        issue_kq<D>(tS, kdesc, qk0 + slot * kSlotStep, idesc_s);
        umma_commit(&ctrl->s_full);
        issued_any = true;
      };
      while (ok) {
        int h = 0;
        if (lane == 0) ok = rd.next(&h, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        h = __shfl_sync(0xffffffffu, h, 0);
        if (!ok || h == kAllDone) break;
        if (lane == 0) {
          SeqWork skip;
          ok = read_item<false>(rd, &skip, abort_flag);
          if (ok) ok = mbar_wait(&ctrl->kv_full, k & 1, abort_flag);
          tc_fence_after();
          bool started = false;
          int e = -1;
          if (ok) ok = rd.next(&e, abort_flag);
          if (ok && e >= 0) {
            int slot = take();
            if (ok) issue_first(slot);
            while (ok) {
              int en = -1;
              ok = rd.next(&en, abort_flag);
              if (!ok) break;
              const int slot_n = en >= 0 ? take() : -1;
              if (!ok) break;
              if (en >= 0) {
                // dP^T(t+1) as soon as the gradient warps have read dP^T(t)
                ok = mbar_wait(&ctrl->dp_free, npd & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_kq<D>(tDP, vdesc, dok0 + slot_n * kSlotStep, idesc_s);
              }
              ok = mbar_wait(&ctrl->pds_full, npd & 1, abort_flag);
              if (!ok) break;
              tc_fence_after();
              if (!started && k > 0) {
                ok = mbar_wait(&ctrl->acc_free, (k - 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
              }
              issue_acc(tDV, tS, domn0 + slot * kSlotStep, idesc_a, started);
              issue_acc(tDK, tS + 16, qmn0 + slot * kSlotStep, idesc_a, started);
              umma_commit(&ctrl->q_empty[slot]);
              ++npd;
              started = true;
              if (en < 0) {
                umma_commit(&ctrl->kv_free);  // every use of K, V is issued
                break;
              }
              // in issue order after dV and dK, which read P^T and dS^T
              issue_kq<D>(tS, kdesc, qk0 + slot_n * kSlotStep, idesc_s);
              umma_commit(&ctrl->s_full);
              slot = slot_n;
            }
          } else if (ok) {
            umma_commit(&ctrl->kv_free);
          }
          if (ok) {
            if (!started && k > 0) {
              ok = mbar_wait(&ctrl->acc_free, (k - 1) & 1, abort_flag);
              tc_fence_after();
            }
            if (ok) umma_commit(&ctrl->acc_full);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        ++k;
      }
      if (lane == 0 && !ok) {
        *abort_flag = 1;
        latch_status(p.status, ST_TIMEOUT);
        if (issued_any) {
          umma_commit(&ctrl->drain);
          mbar_wait(&ctrl->drain, 0, nullptr);
        }
      }
      __syncwarp();
    }
  } else {
    regs_inc<kRegsGrad>();
    // ---------------------------------------------------------- gradient warps
    const int half = warp >> 2;           // query columns [64 half, 64 half + 64)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;       // key row of the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + half * 64;
    const uint32_t tDP = tmem + lane_off + C::kColDP + half * 64;
    uint32_t sphase = 0;
    int k = 0, nstep = 0;
    bool ok = true;
    while (true) {
      int h;
      ok = rd.next_warp(&h, abort_flag);
      if (!ok || h == kAllDone) break;
      SeqWork it;
      ok = read_item<true>(rd, &it, abort_flag);
      if (!ok) break;
      const int L = it.L;
      const int sk = it.qr * BK + r;
      const bool kvalid = sk < L;
      const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
      bool any = false;
      while (true) {
        int e;
        ok = rd.next_warp(&e, abort_flag);
        if (!ok || e < 0) break;
        const int cls = entry_cls(e);
        const int q_lo = entry_qt(e) * BQ;
        const int slot = nstep % kQStages;
        // the slot's lse / D vectors were written before its second arrival
        ok = warp_wait(&ctrl->q_full[slot], (nstep / kQStages) & 1, abort_flag);
        if (!ok) break;
        const float* vec = reinterpret_cast<const float*>(smem + C::kVecOff) + slot * 2 * BQ;
        ++nstep;
        // S^T(t), dP^T(t) computed; dV and dK of the previous step done
        ok = warp_wait(&ctrl->s_full, sphase, abort_flag);
        sphase ^= 1;
        if (!ok) break;
        tc_fence_after();
        // dP^T of this warp's 64 queries first (with the first 32 scores):
        // its columns then take the next step's dP^T while this step is
        // computed
        float dp[64], s[32];
        {
          uint32_t* dr = reinterpret_cast<uint32_t*>(dp);
          uint32_t* sr = reinterpret_cast<uint32_t*>(s);
          RA_TMEM_LD32(tDP, dr);
          RA_TMEM_LD32(tDP + 32, (dr + 32));
          RA_TMEM_LD32(tS, sr);
          tmem_wait_ld();
        }
        tc_fence_before();
        mbar_arrive(&ctrl->dp_free);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c > 0) {
            uint32_t* sr = reinterpret_cast<uint32_t*>(s);
            RA_TMEM_LD32(tS + c * 32, sr);
            tmem_wait_ld();
          }
          // allowed query columns of this key row as a bit word
          const int qc = q_lo + half * 64 + c * 32;
          uint32_t am = 0u;
          if (kvalid) {
            const int nq = min(max(L - qc, 0), 32);
            am = nq >= 32 ? 0xffffffffu : ((1u << nq) - 1u);
            if (cls == CLS_PARTIAL) {
              uint32_t bits = 0u;
              if (p.causal && p.layout == LAYOUT_CONTIGUOUS && p.passes >= p.n_ring) {
                // contiguous causal, no pass limit: the queries at or after
                // the key's own position
                const int lo = sk - qc;
                bits = lo <= 0 ? 0xffffffffu : (lo >= 32 ? 0u : ~((1u << lo) - 1u));
              } else {
                for (int j = 0; j < nq; ++j) {
                  const int qi = qc + j;
                  const int rq = block_of(g, qi);
                  if (allowed(g, qi, rq, token_of(g, qi, rq), sk)) bits |= 1u << j;
                }
              }
              am &= bits;
            }
          }
          uint32_t pp[16], pd[16];
          const int q0 = half * 64 + c * 32;
#pragma unroll
          for (int sb = 0; sb < 2; ++sb) {
            // -lse (log2 units) and -D of 16 query columns
            float nl[16], nd[16];
            const uint32_t va = smem_u32(vec + q0 + 16 * sb), vb = smem_u32(vec + BQ + q0 + 16 * sb);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              ld_shared_f4(va + 16u * u, nl[4 * u], nl[4 * u + 1], nl[4 * u + 2], nl[4 * u + 3]);
              ld_shared_f4(vb + 16u * u, nd[4 * u], nd[4 * u + 1], nd[4 * u + 2], nd[4 * u + 3]);
            }
            // P = ex2(S scale - lse) and dS = P (dP - D) in paired fp32
            // instructions (the same roundings as the scalar forms); masked
            // entries are selected to zero after the products
            const uint64_t sc2 = f32x2_pack(p.scale_log2, p.scale_log2);
#pragma unroll
            for (int j2 = 0; j2 < 8; ++j2) {
              const int jl = 2 * j2, j = 16 * sb + jl;
              float y0, y1;
              ffma2(s[j], s[j + 1], sc2, f32x2_pack(nl[jl], nl[jl + 1]), y0, y1);
              const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
              const uint64_t r2 = mul2(f32x2_pack(p0, p1),
                                       add2(f32x2_pack(dp[32 * c + j], dp[32 * c + j + 1]),
                                            f32x2_pack(nd[jl], nd[jl + 1])));
              const bool a0 = (am >> j) & 1u, a1 = (am >> (j + 1)) & 1u;
              pp[8 * sb + j2] = pack_x2<kFmt>(a0 ? p0 : 0.f, a1 ? p1 : 0.f);
              pd[8 * sb + j2] = pack_x2<kFmt>(a0 ? f32x2_lo(r2) : 0.f, a1 ? f32x2_hi(r2) : 0.f);
            }
          }
          // P^T and dS^T over the 32 score columns just read
          RA_TMEM_ST16(tS + c * 32, pp);
          RA_TMEM_ST16(tS + c * 32 + 16, pd);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctrl->pds_full);
        any = true;
      }
      if (!ok) break;
      // epilogue: warps 0-3 write dV, warps 4-7 dK (scaled), one key row each
      ok = warp_wait(&ctrl->acc_full, k & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tA = tmem + lane_off + (half == 0 ? C::kColDV : C::kColDK);
      const float mul = half == 0 ? 1.f : p.scale;
      const int64_t goff = ((int64_t)(it.base + sk) * p.heads + it.h) * D;
      uint16_t* dst16 = static_cast<uint16_t*>(half == 0 ? bp.dv : bp.dk);
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (any) {
          RA_TMEM_LD32(tA + c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pk[j] = pack_x2<kFmt>(__uint_as_float(o[2 * j]) * mul,
                                __uint_as_float(o[2 * j + 1]) * mul);
        if (kvalid) {
          uint4* dst = reinterpret_cast<uint4*>(dst16 + goff + c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&ctrl->acc_free);
      ++k;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) latch_status(p.status, ST_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int kFmt>
static cudaError_t launch_t(const Params& bp_in, cudaStream_t stream, int num_sms) {
  using C = Cfg<D>;
  Params bp = bp_in;
  FwdParams& p = bp.f;
  p.order = 0;
  p.n_qranges = (p.seqlen + BK - 1) / BK;
  const int64_t items = work_grid(p, BK);
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  Maps maps;
  if (!make_map(&maps.k, p.k, p.total_rows, p.heads, D, p.kv_tok_stride, kFmt, BK) ||
      !make_map(&maps.v, p.v, p.total_rows, p.heads, D, p.kv_tok_stride, kFmt, BK) ||
      !make_map(&maps.q, p.q, p.total_rows, bp.heads_q, D, p.tok_stride, kFmt, BQ) ||
      !make_map(&maps.dout, bp.dout, p.total_rows, bp.heads_q, D, (int64_t)bp.heads_q * D,
                kFmt, BQ))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, kFmt>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // Dense causal items differ in length: one CTA per item, balanced by the
  // hardware block scheduler (persistent CTAs measured 11 % slower there).
  // Otherwise persistent CTAs, one per SM (1.6-2.3 % faster non-causal).
  const bool per_item = p.causal && !p.cu_seqlens;
  const int64_t grid = per_item ? items : (items < num_sms ? items : num_sms);
  if (per_item) {
    bwd_dkdv_kernel<D, kFmt><<<(unsigned)grid, kThreads, C::kSmemBytes, stream>>>(
        bp, maps, (int)items);
    return cudaGetLastError();
  }
  // Persistent CTAs: a programmatic dependent of the dq kernel launched just
  // before it on the stream.  Its CTAs start on the SMs that kernel's last
  // CTAs leave, and read D (the one input that kernel writes) after
  // griddepcontrol.wait (2.5-3 % faster non-causal; with one CTA per item,
  // dense causal, it measured 1 % slower, so those launch plainly).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bwd_dkdv_kernel<D, kFmt>, bp, maps, (int)items);
}

}  // namespace kv

template <int D, int kFmt>
static cudaError_t launch_both(const Params& bp, int num_sms, cudaStream_t stream) {
  cudaError_t e = launch_t<D, kFmt>(bp, stream, num_sms);
  if (e != cudaSuccess) return e;
  // dK/dV: the work decode runs over the key/value heads
  Params kvp = bp;
  kvp.f.heads = bp.f.heads_kv;
  return kv::launch_t<D, kFmt>(kvp, stream, num_sms);
}

}  // namespace tcb

// dq (and D into dsum), then dk and dv, on `stream`.  f: the forward's
// parameters (q/k/v, lse, geometry, status word, a zeroed work counter);
// dsum: float scratch in lse layout.  16-bit inputs, d_head 64 or 128.
cudaError_t launch_bwd_tc(const FwdParams& f, const void* o, const void* dout, void* dq,
                          void* dk, void* dv, float* dsum, int fmt, int num_sms,
                          cudaStream_t stream) {
  tcb::Params bp;
  bp.f = f;
  bp.heads_q = f.heads;
  bp.o = o;
  bp.dout = dout;
  bp.dq = dq;
  bp.dk = dk;
  bp.dv = dv;
  bp.dsum = dsum;
  if (fmt == kFmtBF16) {
    if (f.d_head == 128) return tcb::launch_both<128, kFmtBF16>(bp, num_sms, stream);
    if (f.d_head == 64) return tcb::launch_both<64, kFmtBF16>(bp, num_sms, stream);
  } else if (fmt == kFmtF16) {
    if (f.d_head == 128) return tcb::launch_both<128, kFmtF16>(bp, num_sms, stream);
    if (f.d_head == 64) return tcb::launch_both<64, kFmtF16>(bp, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ra

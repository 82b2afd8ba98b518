// ra_fwd_tc.cu -- ring-ordered blockwise attention forward on the sm_100a
// tensor cores (tcgen05 + TMEM), bf16 or fp16 inputs, fp32 accumulation.
//
// The method: the sequence is split into N ring blocks; a query block keeps
// its queries in place and meets the key/value blocks in ring order, folding
// each block into its output with the running softmax ("Ring Attention"
// glossary, "Come funziona la ring attention"; "Ring Attention simulation"
// gist, flashattention() update: running row max, running denominator,
// output rescaled by exp(m_old - m_new)).  Production kernels subtract the
// running maximum before exponentiating (same glossary page).  The blockwise
// evaluation inside one device is the flash-attention tiling of the
// "Attention的分块计算" blog (local softmax of a block in fast on-chip memory,
// combined into the global softmax through per-block max and sum).
//
// Persistent CTAs (one per SM, 384 threads) claim work items (two query
// tiles of one (sequence, head)) from a per-launch counter, in item order
// (heaviest causal ranges first); the pipelines run across item boundaries:
// the next item's Q is loaded as soon as the last S MMA of the current one is
// done (q_free), and its first PV MMA waits only until the softmax warps have
// read O out (o_free).  Dense causal launches run one CTA per item instead;
// key/value-outer ring steps take items by a static stride and split the
// items of a mostly empty last wave into halves of their key tiles, the
// second halves folded in afterwards by step_merge_kernel.
// Warp roles:
//   warps 0-3  softmax for query tile 0 (one TMEM lane = one query row each)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q once per item; K and V tiles into one ring of
//              shared-memory slots in the order K(0), V(0), K(1), V(1), ...
//              (the issuer takes V(t) and K(t+1) for PV(t) and S(t+1))
//   warp  9    MMA issuer for both query tiles: S_i = Q_i K^T into tensor
//              memory and O_i += P_i V with P_i read from tensor memory, as
//              tcgen05.mma; completion signalled with tcgen05.commit.  (With
//              kTcIssuers = 2, warps 9 and 11 issue one query tile each; one
//              issuer measured faster: the two tiles then stay out of phase.)
//   warp  10   schedule builder: runs the ring-order tile walk (ra_sched.h)
//              and publishes the visited kv tiles with their per-query-tile
//              class into a shared-memory ring of small list chunks
// The control warpgroup (warps 8-11) hands registers to the softmax
// warpgroups with setmaxnreg.
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1, with P_i (16-bit,
// two keys per column) written over the first half of S_i once S_i is in
// registers.  Shared memory: Q_0, Q_1, the K/V ring, the list.
//
// Per kv tile t issuer i waits until softmax i has written P_i(t) (p_full),
// then issues PV_i(t) followed by S_i(t+1).  The tensor core runs the MMAs
// of one thread in issue order, so S_i(t+1) overwrites the P_i(t) columns
// only after PV_i(t) has read them, and the commit that announces S_i(t+1)
// (s_full) also covers PV_i(t): when softmax i sees S_i(t+1), P_i(t) is free
// and O_i is stable for a rescale.  While softmax i works on its tile the
// tensor core runs the other query tile's PV and S, so the two softmax
// warpgroups take turns on the exponential unit.
//
// The running max is only moved when it grows by more than kRescaleLog2
// (in log2 units); until then exponentials are taken against the stale max
// (values <= 2^kRescaleLog2), which is exact up to rounding because the same
// reference is used for O and l.
#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ra_common.cuh"
#include "ra_list.cuh"
#include "ra_params.h"
#include "ra_sched.h"
#include "ra_work.cuh"

namespace ra {

constexpr int kTcBM = 128;          // rows per query tile (TMEM lanes)
constexpr int kTcQT = 2;            // query tiles per CTA
constexpr int kTcBN = 128;          // keys per kv tile
constexpr int kTcThreads = 384;     // 2 softmax warpgroups + 1 control warpgroup
constexpr int kTcProducerWarp = 8;
constexpr int kTcMmaWarp = 9;      // MMA issuer (allocates TMEM)
constexpr int kTcMmaWarp1 = 11;    // second MMA issuer when kTcIssuers == 2
constexpr int kTcListWarp = 10;
// MMA issuer warps: 2 = one per query tile, 1 = warp 9 issues for both tiles
constexpr int kTcIssuers = 1;
constexpr int kListConsumers = 9 + kTcIssuers;  // producer, issuers, 8 softmax warps
// Register split.  Launch: 384 threads x 168 = 64512 registers.  After the
// split: 256 softmax threads x 176 + 128 control threads x 152 = 64512.
constexpr int kRegsSoftmax = 176;
constexpr int kRegsControl = 152;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

// Element format traits: 16-bit (f16 / bf16, kind::f16 MMAs, K = 16 per
// instruction) or 8-bit e4m3 (kind::f8f6f4, K = 32).
template <int kFmt>
struct TcFmt {
  static constexpr bool kF8 = kFmt == kFmtE4M3;
  static constexpr int kBytes = kF8 ? 1 : 2;       // bytes per element
  static constexpr int kK = kF8 ? 32 : 16;         // K per MMA instruction
  static constexpr int kPanelElems = 128 / kBytes; // elements per 128-byte row panel
  // MMA format field: e4m3 is 0 under kind::f8f6f4; f16 0 and bf16 1 under kind::f16
  static constexpr int kMmaFmt = kF8 ? 0 : kFmt;
};

template <int D, int kFmt = kFmtBF16>
struct TcCfg {
  static constexpr int kPanels = D * TcFmt<kFmt>::kBytes / 128;  // 128-byte swizzle panels
  static constexpr int kPanelBytes = kTcBM * 128;           // 128 rows x 128 B
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // one Q/K/V tile
  static constexpr int kStages = kTileBytes >= 32768 ? 5 : 10;  // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kTcQT * kTileBytes;
  static constexpr int kListOff = kKVOff + kStages * kTileBytes;
  static constexpr int kCtrlOff = kListOff + kListBufs * kListChunk * 4;
  static constexpr int kCtrlBytes = 1024;
  static constexpr int kSmemBytes = kCtrlOff + kCtrlBytes + 1024;  // + align slack
  static constexpr uint32_t kColS = 0;                      // S_i at i * 128
  static constexpr uint32_t kColO = 256;                    // O_i at 256 + i * D
  static constexpr int kSlots = 10;                         // ring slots the barriers allow
  static_assert(kStages <= kSlots, "K/V ring barriers");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct TcCtrl {
  uint64_t q_full;
  uint64_t q_free;
  uint64_t kv_full[10];
  uint64_t kv_empty[10];
  uint64_t s_full[kTcQT];
  uint64_t p_full[kTcQT];
  uint64_t o_full[kTcQT];
  uint64_t o_free[kTcQT];
  uint64_t list_full[kListBufs];
  uint64_t list_empty[kListBufs];
  uint64_t drain[kTcQT];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(TcCtrl) <= 1024, "control block");

struct TcMaps {
  CUtensorMap q, k, v;
};

// Number of leading columns of kv tile [k0, k0 + nk) allowed for query (rq,
// tq) when the whole tile lies in ring block rk (the allowed keys of one
// block always form a prefix in stored order).
__device__ __forceinline__ int single_block_limit(const RingGeom& g, int rq, int tq, int rk,
                                                  int k0, int nk) {
  if (!pass_ok(g, rq, rk)) return 0;
  if (!g.causal) return nk;
  int last;  // last allowed stored key of block rk
  if (g.layout == LAYOUT_CONTIGUOUS) {
    last = tq;
  } else {
    if (tq < rk) return 0;
    last = block_start(g, rk) + (tq - rk) / g.N;
  }
  const int lim = last - k0 + 1;
  return lim < 0 ? 0 : (lim > nk ? nk : lim);
}

// S = Q K^T for one query tile: M = 128 rows, N = 128 keys, K = D in steps of
// 32 bytes (16 16-bit or 32 8-bit elements).  Both operands K-major in
// 128-byte-swizzled panels; the descriptors of step kk are the tile's base
// descriptors plus a constant (start address field, in 16-byte units: panel
// * 1024 + 2 * (kk % 4)).
template <int D, int kFmt>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t qdesc, uint64_t kdesc,
                                         uint32_t idesc) {
  using C = TcCfg<D, kFmt>;
  using F = TcFmt<kFmt>;
#pragma unroll
  for (int kk = 0; kk < D / F::kK; ++kk) {
    const uint64_t off = (uint64_t)((kk >> 2) * (C::kPanelBytes >> 4) + (kk & 3) * 2);
    if (F::kF8)
      umma_ss_f8(d_tmem, qdesc + off, kdesc + off, idesc, kk > 0 ? 1u : 0u);
    else
      umma_ss(d_tmem, qdesc + off, kdesc + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V for one query tile: A = P from tensor memory (128 lanes, two
// 16-bit or four 8-bit keys per column; one step's K keys are 8 columns), B
// = V tile MN-major (N = D split in 128-byte panels, LBO = panel stride;
// 8-key groups 1024 bytes apart).  Step kk covers K keys (16 or 32).
template <int D, int kFmt>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t vdesc,
                                         uint32_t idesc, bool accumulate) {
  using F = TcFmt<kFmt>;
#pragma unroll
  for (int kk = 0; kk < kTcBN / F::kK; ++kk) {
    const uint64_t voff = (uint64_t)(kk * F::kK * 8);  // K rows of 128 B, 16-byte units
    if (F::kF8)
      umma_ts_f8(d_tmem, p_tmem + (uint32_t)(kk * 8), vdesc + voff, idesc,
                 (accumulate || kk > 0) ? 1u : 0u);
    else
      umma_ts(d_tmem, p_tmem + (uint32_t)(kk * 8), vdesc + voff, idesc,
              (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Bits [lo, hi) of a 32-bit word, 0 <= lo < hi <= 32.
__device__ __forceinline__ uint32_t bit_range(int lo, int hi) {
  const uint32_t upto = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}

// Replace the scores of disallowed keys by -inf.  Keys at or beyond L (the
// next sequence, or rows past the tensor) are always disallowed; on PARTIAL
// tiles the ring mask is applied too.  In stored order the keys of one ring
// block are consecutive and a query's allowed keys among them form a prefix
// (single_block_limit), so the allowed columns of a tile are the union of one
// interval per ring block the tile meets.
__device__ __forceinline__ void apply_mask(float* x, const FwdParams& p, int L, bool valid,
                                           int cls, int rq, int tq, int k0, int nk) {
  uint32_t mw[kTcBN / 32];  // allowed columns as 4 x 32-bit masks (indices stay compile-time)
  if (!valid || cls == CLS_FULL) {
#pragma unroll
    for (int w = 0; w < kTcBN / 32; ++w) {
      const int n = min(max(nk - 32 * w, 0), 32);
      mw[w] = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
    }
  } else {
    const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
#pragma unroll
    for (int w = 0; w < kTcBN / 32; ++w) mw[w] = 0u;
    const int kend = k0 + nk;
    int c = k0;
    // at most one pass per ring block (empty blocks advance rk only)
    for (int rk = block_of(g, k0); c < kend && rk < g.N; ++rk) {
      const int be = min(block_start(g, rk + 1), kend);
      if (be <= c) continue;
      const int a = c - k0, bnd = a + single_block_limit(g, rq, tq, rk, c, be - c);
#pragma unroll
      for (int w = 0; w < kTcBN / 32; ++w) {
        const int lo = max(a - 32 * w, 0), hi = min(bnd - 32 * w, 32);
        if (hi > lo) mw[w] |= bit_range(lo, hi);
      }
      c = be;
    }
  }
#pragma unroll
  for (int c = 0; c < kTcBN; ++c) x[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? x[c] : -INFINITY;
}

// Is the item announced by list header h the second half of a split ring
// step item (launch items n_items - 2 * split .. n_items - 1 come in halves)?
__device__ __forceinline__ bool split_half(int h, int n_items, int split) {
  const int d = -h - 8 - (n_items - 2 * split);  // launch item from the header
  return d >= 0 && (d & 1);
}

// Schedule-list entries of an item (ra_list.cuh): (kt << 4) | (class of
// query tile 1 << 2) | class of query tile 0 for a visited kv tile.
__device__ __forceinline__ int entry_tile(int e) { return e >> 4; }
__device__ __forceinline__ int entry_cls(int e, int i) { return (e >> (2 * i)) & 3; }

template <int D, int kFmt>
__global__ void __launch_bounds__(kTcThreads, 1)
    fwd_tc_kernel(const FwdParams p, const __grid_constant__ TcMaps maps, int n_items,
                  int claim_limit) {
  using C = TcCfg<D, kFmt>;
  using F = TcFmt<kFmt>;
  constexpr int kRows = kTcBM * kTcQT;  // query rows per work item
  constexpr int KVS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcCtrl* ctrl = reinterpret_cast<TcCtrl*>(smem + C::kCtrlOff);
  volatile int* abort_flag = &ctrl->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ------------------------------------------------------------ set-up
  int* list = reinterpret_cast<int*>(smem + C::kListOff);
  if (threadIdx.x == 0) {
    mbar_init(&ctrl->q_full, 1);
    mbar_init(&ctrl->q_free, kTcIssuers);  // one commit per issuer
    for (int s = 0; s < KVS; ++s) {
      mbar_init(&ctrl->kv_full[s], 1);
      mbar_init(&ctrl->kv_empty[s], kTcIssuers);
    }
    for (int i = 0; i < kTcQT; ++i) {
      mbar_init(&ctrl->s_full[i], 1);
      mbar_init(&ctrl->p_full[i], kTcBM);
      mbar_init(&ctrl->o_full[i], 1);
      mbar_init(&ctrl->o_free[i], kTcBM);
      mbar_init(&ctrl->drain[i], 1);
    }
    for (int b = 0; b < kListBufs; ++b) {
      mbar_init(&ctrl->list_full[b], 1);
      mbar_init(&ctrl->list_empty[b], kListConsumers);
    }
    ctrl->abort = 0;
    mbar_fence_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Ring steps are launched as programmatic dependents of the previous
  // launch on the stream: the next step's CTAs may be placed on SMs this
  // launch has finished with and run their set-up (barriers, tensor memory)
  // while its last CTAs finish.  The launch before may have written any of
  // the inputs (q, k, v, cu_seqlens, the running out and lse), so no thread
  // reads global memory before griddepcontrol.wait has returned, which is
  // after that launch has completed and its writes are visible.
  if (p.step) {
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
  }
  const uint32_t tmem = ctrl->tmem_base;
  ListReader rd;
  rd.list = smem_u32(list);
  rd.full = ctrl->list_full;
  rd.empty = ctrl->list_empty;

  if (warp >= 8) {
   regs_dec<kRegsControl>();
   if (warp == kTcListWarp) {
    // ---------------------------------------------------------- schedule
    // Claims work items from the launch's counter (dynamic balance; heavy
    // items come first in the item order), at most one item ahead of the
    // producer, and streams each item's header, ring-order visit list and
    // end marker, in chunks of kListChunk entries.
    ListWriter wr;
    wr.list = smem_u32(list);
    wr.full = ctrl->list_full;
    wr.empty = ctrl->list_empty;
    wr.abort = abort_flag;
    bool ok = true;
    auto put = [&](int v) -> bool { return wr.put(v); };
    auto flush = [&]() -> bool { return wr.flush(); };
    int j = 0;       // items emitted
    int claims = 0;  // items claimed (emitted or skipped)
    while (ok) {
      if (claim_limit > 0 && j >= claim_limit) {
        if (lane == 0) ok = put(kAllDone) && flush();
        break;
      }
      if (lane == 0 && j > 0) {
        ok = flush();
        // item j-1 has started (its Q landed) before another item is claimed
        if (ok) ok = mbar_wait(&ctrl->q_full, (j - 1) & 1, abort_flag);
      }
      // the launch's counter hands out items; without one (ring steps,
      // whose items are all alike) CTA c takes items c, c + grid, ...
      int item = blockIdx.x + claims * (int)gridDim.x;
      ++claims;
      if (lane == 0 && ok && p.work_counter) item = atomicAdd(p.work_counter, 1);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      item = __shfl_sync(0xffffffffu, item, 0);
      if (!ok) break;
      if (item >= n_items) {
        if (lane == 0) ok = put(kAllDone) && flush();
        break;
      }
      // the halves of a split ring-step item share the item's description
      const int n_whole = n_items - 2 * p.step_split;
      const bool split = item >= n_whole;
      const SeqWork it =
          find_work_item(p, kRows, split ? n_whole + ((item - n_whole) >> 1) : item);
      if (!it.live) continue;
      if (lane == 0) {
        // query rows of this sequence held in q: the sequence, or one ring block
        const int nrows = p.step ? p.step_rows : it.L;
        const int q0 = it.qr * kRows;
        const int qm = min(q0 + kTcBM, nrows), q1 = min(q0 + kRows, nrows);
        const RingGeom g = make_geom(it.L, p.n_ring, p.layout, p.causal, p.passes);
        ok = put_item(wr, item, it);
        int kt, c0, c1;
        // test hook: a record of each visited kv tile
        auto dump = [&](int entry) {
          if (!p.sched_dump) return;
          const int i = atomicAdd(p.sched_dump, 1);
          if (i < p.sched_dump_cap) {
            int* r = p.sched_dump + 4 + 4 * (int64_t)i;
            r[0] = it.b;
            r[1] = it.h;
            r[2] = it.qr;
            r[3] = entry;
          }
        };
        if (!p.step) {
          TileWalk walk;
          walk.init(g, q0, qm, q1, kTcBN);
          while (ok && walk.next(&kt, &c0, &c1)) {
            dump((kt << 4) | (c1 << 2) | c0);
            ok = put((kt << 4) | (c1 << 2) | c0);
          }
        } else {
          // one ring step: the tiles of key/value block kv_block (tile-aligned
          // blocks; kt counts tiles inside the block).  The item's query rows
          // all lie in ring block q_block and every key tile in kv_block, so
          // a tile's class is that of one segment pair: no block lookups (the
          // general classify() divides by the block geometry several times
          // per call, which at one thread paced the whole step).
          const int qo = p.q_block * p.step_rows, ko = p.kv_block * p.step_rows;
          // a split item's half walks half of the block's tiles
          const int nkt = p.step_rows / kTcBN;
          const int kt_lo = split ? (((item - n_whole) & 1) ? nkt / 2 : 0) : 0;
          const int kt_hi = split ? (((item - n_whole) & 1) ? nkt : nkt / 2) : nkt;
          auto seg_class = [&](int a, int b, int c) -> int {
            if (a >= b) return CLS_EMPTY;
            bool any = false, all = true;
            classify_segment(g, p.q_block, a, b, p.kv_block, c, c + kTcBN, &any, &all);
            return any ? (all ? CLS_FULL : CLS_PARTIAL) : CLS_EMPTY;
          };
          for (kt = kt_lo; ok && kt < kt_hi; ++kt) {
            const int k0 = ko + kt * kTcBN;
            c0 = seg_class(qo + q0, qo + qm, k0);
            c1 = seg_class(qo + qm, qo + q1, k0);
            if (c0 != CLS_EMPTY || c1 != CLS_EMPTY) {
              dump((kt << 4) | (c1 << 2) | c0);
              ok = put((kt << 4) | (c1 << 2) | c0);
            }
          }
        }
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
   } else if (warp == kTcProducerWarp) {
    // ---------------------------------------------------------- producer
    // Ring order K(0), V(0), K(1), V(1), ...: the order in which the issuers
    // consume the tiles (PV(t) comes before S(t+1)).
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
    }
    int n = 0, k = 0, nq = 0;  // K/V tiles, items and query loads issued
    bool ok = true;
    auto load = [&](const CUtensorMap* map, int h, int row) -> bool {
      const int slot = n % KVS;
      if (n >= KVS && !mbar_wait(&ctrl->kv_empty[slot], ((n / KVS) - 1) & 1, abort_flag))
        return false;
      uint8_t* dst = smem + C::kKVOff + slot * C::kTileBytes;
      mbar_arrive_expect_tx(&ctrl->kv_full[slot], C::kTileBytes);
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_3d(dst + pn * C::kPanelBytes, map, &ctrl->kv_full[slot], pn * F::kPanelElems,
                    h, row);
      ++n;
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
        // the item's first K enters the ring before Q waits for the previous
        // item's last S MMAs (q_free)
        int e = -1;
        if (ok) ok = rd.next(&e, abort_flag);
        const int hk = it.h / p.kv_group;  // key/value head of this query head
        if (ok && e >= 0) ok = load(&maps.k, hk, it.base + entry_tile(e) * kTcBN);
        if (ok && k > 0) ok = mbar_wait(&ctrl->q_free, (k - 1) & 1, abort_flag);
        if (ok && !p.withhold_q) {
          uint8_t* qs = smem + C::kQOff;
          const int q0 = it.qr * kRows;
          mbar_arrive_expect_tx(&ctrl->q_full, kTcQT * C::kTileBytes);
          for (int i = 0; i < kTcQT; ++i)
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d(qs + i * C::kTileBytes + pn * C::kPanelBytes, &maps.q,
                          &ctrl->q_full, pn * F::kPanelElems, it.h, it.base + q0 + i * kTcBM);
          ++nq;
        }
        if (ok && e >= 0) ok = load(&maps.v, hk, it.base + entry_tile(e) * kTcBN);
        while (ok && e >= 0) {
          ok = rd.next(&e, abort_flag);
          if (!ok || e < 0) break;
          ok = load(&maps.k, hk, it.base + entry_tile(e) * kTcBN);
          if (ok) ok = load(&maps.v, hk, it.base + entry_tile(e) * kTcBN);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ++k;
    }
    if (lane == 0 && !ok) {
      *abort_flag = 1;
      latch_status(p.status, ST_TIMEOUT);
      // let the copies already issued land before the CTA can exit
      for (int u = (n > KVS ? n - KVS : 0); u < n; ++u)
        mbar_wait(&ctrl->kv_full[u % KVS], (u / KVS) & 1, nullptr);
      if (nq > 0) mbar_wait(&ctrl->q_full, (nq - 1) & 1, nullptr);
    }
    __syncwarp();
   } else if (warp == kTcMmaWarp || kTcIssuers == 2) {
    // ---------------------------------------------------------- MMA issuers
    // Issuer of query tiles [i0, i1): S_i(0), then per kv tile t, once
    // softmax i has written P_i(t) into tensor memory (p_full), PV_i(t) and
    // S_i(t+1).  Both are issued by this thread, so they run in that order:
    // S_i(t+1) overwrites the P_i(t) columns after PV_i(t) has read them.
    // Every issuer walks the K/V ring in load order; a slot is released by
    // one commit of each issuer.
    const int i0 = (kTcIssuers == 2 && warp == kTcMmaWarp1) ? 1 : 0;
    const int i1 = kTcIssuers == 2 ? i0 + 1 : kTcQT;
    // a negative softmax scale is applied as S = (-Q) K^T times |scale|
    const uint32_t idesc_s =
        idesc_f16kind_f32(kTcBM, kTcBN, 0, F::kMmaFmt) | (p.scale_log2 < 0.f ? (1u << 13) : 0u);
    constexpr uint32_t idesc_o = idesc_f16kind_f32(kTcBM, D, 1, F::kMmaFmt);
    // base descriptors: K-major tiles (Q, K) and MN-major tiles (V)
    const uint64_t qdesc0 = smem_desc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
    const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + C::kKVOff), 16, 1024);
    const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + C::kKVOff), C::kPanelBytes, 1024);
    constexpr uint64_t kSlotStep = (uint64_t)(C::kTileBytes >> 4);
    constexpr uint64_t kQStep = (uint64_t)(C::kTileBytes >> 4);
    uint32_t pphase[kTcQT] = {0, 0};
    int n = 0, k = 0;
    bool ok = true, issued_any = false;
    // next ring slot, once its tile has landed
    auto take = [&]() -> int {
      const int slot = n % KVS;
      ok = mbar_wait(&ctrl->kv_full[slot], (n / KVS) & 1, abort_flag);
      ++n;
      if (ok) tc_fence_after();
      return slot;
    };
    auto issue_s_tile = [&](int e, int i, int slot) {
      if (entry_cls(e, i) == CLS_EMPTY) return;
      issue_qk<D, kFmt>(tmem + C::kColS + i * kTcBN, qdesc0 + i * kQStep, kdesc0 + slot * kSlotStep,
                  idesc_s);
      umma_commit(&ctrl->s_full[i]);
      issued_any = true;
    };
    while (ok) {
      int h = 0;
      if (lane == 0) ok = rd.next(&h, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      h = __shfl_sync(0xffffffffu, h, 0);
      if (!ok || h == kAllDone) break;
      // the second half of a split ring-step item starts from the empty state
      const bool acc = p.accumulate && !split_half(h, n_items, p.step_split);
      if (lane == 0) {
        SeqWork skip;  // the item's description is not needed here
        ok = read_item<false>(rd, &skip, abort_flag);
        if (ok) ok = mbar_wait(&ctrl->q_full, k & 1, abort_flag);
        tc_fence_after();
        bool started[kTcQT] = {false, false};
        // the previous item's O_i must have been read out before it is overwritten
        bool ofree_pending[kTcQT] = {k > 0, k > 0};
        auto wait_ofree = [&](int i) {
          if (ok && ofree_pending[i]) {
            ok = mbar_wait(&ctrl->o_free[i], (k - 1) & 1, abort_flag);
            ofree_pending[i] = false;
            tc_fence_after();
          }
        };
        int e = -1;
        if (ok) ok = rd.next(&e, abort_flag);
        if (ok && e >= 0) {
          // S_i(0) for every tile of this issuer, tile 0 first
          const int slot_k0 = take();
          if (ok) {
            for (int i = i0; i < i1; ++i) issue_s_tile(e, i, slot_k0);
            umma_commit(&ctrl->kv_empty[slot_k0]);
          }
          int ep = e;  // entry of kv tile t
          while (ok) {
            ok = rd.next(&e, abort_flag);  // kv tile t + 1, or the item's end
            if (!ok) break;
            const bool has = e >= 0;
            // every S of this item is issued: Q may be replaced once they finish
            if (!has) umma_commit(&ctrl->q_free);
            const int slot_v = take();             // V(t)
            const int slot_k = ok && has ? take() : 0;  // K(t + 1)
            if (!ok) break;
            // per tile, PV_i(t) then S_i(t + 1): with one issuer the tensor
            // core runs PV_0 S_0 PV_1 S_1, so while softmax 0 works on S_0(t+1)
            // the tensor core computes tile 1's products, and the other way round
            for (int i = i0; i < i1 && ok; ++i) {
              if (entry_cls(ep, i) != CLS_EMPTY) {
                ok = mbar_wait(&ctrl->p_full[i], pphase[i], abort_flag);
                pphase[i] ^= 1;
                if (!ok) break;
                tc_fence_after();
                if (!started[i]) wait_ofree(i);
                if (!ok) break;
                // an accumulating ring step adds to the O loaded from the state
                issue_pv<D, kFmt>(tmem + C::kColO + i * D, tmem + C::kColS + i * kTcBN,
                            vdesc0 + slot_v * kSlotStep, idesc_o, started[i] || acc);
                started[i] = true;
              }
              if (has) issue_s_tile(e, i, slot_k);
            }
            if (!ok) break;
            umma_commit(&ctrl->kv_empty[slot_v]);
            if (!has) break;
            umma_commit(&ctrl->kv_empty[slot_k]);
            ep = e;
          }
        } else if (ok) {
          umma_commit(&ctrl->q_free);  // an item without tiles
        }
        if (ok) {
          for (int i = i0; i < i1; ++i) wait_ofree(i);
          if (ok)
            for (int i = i0; i < i1; ++i) umma_commit(&ctrl->o_full[i]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ++k;
    }
    if (lane == 0 && !ok) {
      *abort_flag = 1;
      latch_status(p.status, ST_TIMEOUT);
      if (issued_any) {
        // wait (bounded) for the MMAs already issued before TMEM is freed
        umma_commit(&ctrl->drain[i0]);
        mbar_wait(&ctrl->drain[i0], 0, nullptr);
      }
    }
    __syncwarp();
   }
  } else {
    regs_inc<kRegsSoftmax>();
    // ---------------------------------------------------------- softmax
    const int tile = warp >> 2;          // query tile handled by this warp
    const int quad = warp & 3;           // TMEM lane quadrant
    const int r = quad * 32 + lane;      // row within the query tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + tile * kTcBN;
    const uint32_t tO = tmem + lane_off + C::kColO + tile * D;
    // P_tile goes over the first kTcBN / 2 columns of S_tile (two keys per column)
    const uint32_t tP = tS;
    const float sl2 = fabsf(p.scale_log2);  // > 0; the sign is folded into the MMA
    uint32_t sphase = 0;
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
      // sq: row in q/out; sqg: its stored index in the sequence (they differ
      // in a ring step, where q holds one block); kvo: same offset for keys
      const int sq = it.qr * kRows + tile * kTcBM + r;
      const int qo = p.step ? p.q_block * p.step_rows : 0;
      const int kvo = p.step ? p.kv_block * p.step_rows : 0;
      const bool valid = sq < (p.step ? p.step_rows : L);
      int rq = 0, tq = 0;
      if (valid) {
        const RingGeom g = make_geom(L, p.n_ring, p.layout, p.causal, p.passes);
        rq = block_of(g, qo + sq);
        tq = token_of(g, qo + sq, rq);
      }
      const int64_t li = (int64_t)it.b * p.lse_seq_stride + (int64_t)it.h * p.lse_head_stride +
                         (p.cu_seqlens ? it.base : 0) + sq;
      float m_ref = -INFINITY;  // reference max, log2 domain
      float l = 0.f;
      bool first = true;
      // A ring step that accumulates starts from the running state: m = lse
      // (log2 units) with l = 1 and O = the normalised output (O = 0 where
      // nothing was folded yet); the first PV then adds to O.  The second
      // half of a split item (split_half) starts from the empty state.
      const bool from_state = p.step && p.accumulate && !split_half(h, n_items, p.step_split);
      if (from_state) {
        const float lp = valid ? p.lse[li] : -INFINITY;
        const bool has = lp > -INFINITY;
        if (has) {
          m_ref = lp * 1.4426950408889634f;
          l = 1.f;
        }
        // The warp's 32 rows are loaded together in the 16x256b fragment
        // shape: four threads read 32 contiguous bytes of one row (whole
        // sectors), where a thread per row would touch a line per thread.
        // Every load is issued before the first tensor-memory store.
        const float* obase = static_cast<const float*>(p.out) +
                             ((int64_t)(it.base + sq - lane) * p.heads + it.h) * D;
        const int64_t rstride = (int64_t)p.heads * D;
        uint32_t o[2][D / 2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int ra = 16 * hf + (lane >> 2), rb = ra + 8;  // rows of the warp
          const bool ha = __shfl_sync(0xffffffffu, has ? 1 : 0, ra) != 0;
          const bool hb = __shfl_sync(0xffffffffu, has ? 1 : 0, rb) != 0;
#pragma unroll
          for (int g = 0; g < D / 8; ++g) {
            const int col = 8 * g + 2 * (lane & 3);
            const float2 fa = ha ? *reinterpret_cast<const float2*>(obase + ra * rstride + col)
                                 : make_float2(0.f, 0.f);
            const float2 fb = hb ? *reinterpret_cast<const float2*>(obase + rb * rstride + col)
                                 : make_float2(0.f, 0.f);
            o[hf][4 * g] = __float_as_uint(fa.x);
            o[hf][4 * g + 1] = __float_as_uint(fa.y);
            o[hf][4 * g + 2] = __float_as_uint(fb.x);
            o[hf][4 * g + 3] = __float_as_uint(fb.y);
          }
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t th = tO + ((uint32_t)(16 * hf) << 16);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) RA_TMEM_ST256X8(th + 64 * c, (o[hf] + 32 * c));
        }
        tmem_wait_st();
      }

      while (true) {
        int e;
        ok = rd.next_warp(&e, abort_flag);
        if (!ok || e < 0) break;
        const int cls = entry_cls(e, tile);
        if (cls == CLS_EMPTY) continue;
        ok = warp_wait(&ctrl->s_full[tile], sphase, abort_flag);
        sphase ^= 1;
        if (!ok) break;
        tc_fence_after();

        float x[kTcBN];
        {
          uint32_t* xr = reinterpret_cast<uint32_t*>(x);
#pragma unroll
          for (int c = 0; c < kTcBN; c += 32) RA_TMEM_LD32(tS + c, (xr + c));
          tmem_wait_ld();
        }
        const int k0 = kvo + entry_tile(e) * kTcBN;  // stored index of the tile's first key
        const int nk = min(kTcBN, L - k0);
        if (cls == CLS_PARTIAL || nk < kTcBN) {
          apply_mask(x, p, L, valid, cls, rq, tq, k0, nk);
        }
        // row max as a tree of independent maxima (short dependency chains)
        float mx8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) mx8[j] = x[j];
#pragma unroll
        for (int c = 8; c < kTcBN; c += 2)
          mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], x[c], x[c + 1]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_tile = mx * sl2;  // -inf stays -inf (sl2 > 0)
        const bool need = m_tile > m_ref + kRescaleLog2;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_ref - m_tile);  // 0 when m_ref == -inf
          m_ref = m_tile;
        }
        const float msub = m_ref == -INFINITY ? 0.f : m_ref;
        // P row in registers (16-bit pairs); scale-and-subtract and the row
        // sums in paired fp32 instructions
        const uint64_t sc2 = f32x2_pack(sl2, sl2), ms2 = f32x2_pack(-msub, -msub);
        uint64_t sum2[2] = {0ull, 0ull};  // two independent (even, odd) partial sums
        // P packed 2 (16-bit) or 4 (e4m3) keys per 32-bit column
        constexpr int kPCols = kTcBN * F::kBytes / 4;
        uint32_t pk[kPCols];
        float pa = 0.f, pb = 0.f;  // e4m3: the even pair, packed with the odd one
#pragma unroll
        for (int j = 0; j < kTcBN / 2; ++j) {
          float ya, yb;
          ffma2(x[2 * j], x[2 * j + 1], sc2, ms2, ya, yb);
          const float a = ex2_approx(ya);
          const float b = ex2_approx(yb);
          sum2[j & 1] = fadd2(sum2[j & 1], a, b);
          if (F::kF8) {
            if (j & 1)
              pk[j >> 1] = pack_e4m3x4(pa, pb, a, b);
            else
              pa = a, pb = b;
          } else {
            pk[j] = pack_x2<kFmt>(a, b);
          }
        }
        // P into tensor memory, over the scores just read (the previous PV of
        // this tile finished before this S was announced)
#pragma unroll
        for (int c = 0; c < kPCols; c += 32) RA_TMEM_ST32(tP + c, (pk + c));
        l = l * alpha + ((f32x2_lo(sum2[0]) + f32x2_hi(sum2[0])) +
                         (f32x2_lo(sum2[1]) + f32x2_hi(sum2[1])));
        if ((!first || from_state) && __any_sync(0xffffffffu, need)) {
          // O_row *= alpha (exactly 1.0 for rows that keep their reference)
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            RA_TMEM_LD32(tO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            RA_TMEM_ST32(tO + c, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctrl->p_full[tile]);
        first = false;
      }
      if (!ok) break;

      // epilogue: O is read out of tensor memory, handed back, then stored
      ok = warp_wait(&ctrl->o_full[tile], k & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const int64_t orow_off = ((int64_t)(it.base + sq) * p.heads + it.h) * D;
      // a ring step writes fp32: the running output, or (second half of a
      // split item) the partial at row sp_row of the split buffers
      const bool to_split = split_half(h, n_items, p.step_split);
      const bool acc = p.accumulate && !to_split;
      const int64_t sp_row =
          (int64_t)((-h - 8 - (n_items - 2 * p.step_split)) >> 1) * kRows + tile * kTcBM + r;
      float* const srow = to_split ? p.split_out + sp_row * D
                                   : static_cast<float*>(p.out) + orow_off;
      const int64_t sstride = to_split ? D : (int64_t)p.heads * D;
      if (!first && p.step) {
        // ring step: the running output stays fp32, written by the warp's
        // threads together in the 16x256b fragment shape (32 contiguous
        // bytes of a row per four threads, as the state was loaded)
        const float inv_l = valid ? p.out_scale / l : 0.f;
        float* obase = srow - (int64_t)lane * sstride;
        const int64_t rstride = sstride;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int ra = 16 * hf + (lane >> 2), rb = ra + 8;  // rows of the warp
          const float ia = __shfl_sync(0xffffffffu, inv_l, ra);
          const float ib = __shfl_sync(0xffffffffu, inv_l, rb);
          const bool va = __shfl_sync(0xffffffffu, valid ? 1 : 0, ra) != 0;
          const bool vb = __shfl_sync(0xffffffffu, valid ? 1 : 0, rb) != 0;
          const uint32_t th = tO + ((uint32_t)(16 * hf) << 16);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            RA_TMEM_LD256X8(th + 64 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const int col = 64 * c + 8 * g + 2 * (lane & 3);
              if (va)
                *reinterpret_cast<float2*>(obase + ra * rstride + col) = make_float2(
                    __uint_as_float(o[4 * g]) * ia, __uint_as_float(o[4 * g + 1]) * ia);
              if (vb)
                *reinterpret_cast<float2*>(obase + rb * rstride + col) = make_float2(
                    __uint_as_float(o[4 * g + 2]) * ib, __uint_as_float(o[4 * g + 3]) * ib);
            }
          }
        }
      } else if (!first) {
        const float inv_l = valid ? p.out_scale / l : 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          RA_TMEM_LD32(tO + c, o);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[j] = pack_x2<F::kF8 ? kFmtBF16 : kFmt>(__uint_as_float(o[2 * j]) * inv_l,
                                                     __uint_as_float(o[2 * j + 1]) * inv_l);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow_off + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      } else if (p.step && !acc && valid) {
        // no key of this block is visible to the row: the empty result
        float4* dst = reinterpret_cast<float4*>(srow);
#pragma unroll
        for (int j = 0; j < D / 4; ++j) dst[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      tc_fence_before();
      mbar_arrive(&ctrl->o_free[tile]);
      if (valid) {
        float* const lse_dst = to_split ? p.split_lse + sp_row : p.lse + li;
        if (!first) {
          *lse_dst = (m_ref + __log2f(l)) * 0.69314718055994530942f;
        } else if (p.step && !acc) {
          *lse_dst = -INFINITY;
        }
        // (an accumulating step without new keys leaves the state as it was)
      }
      ++k;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) latch_status(p.status, ST_TIMEOUT);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
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

static EncodeTiledFn get_encode_fn() {
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

// [rows, heads, D] view of 16-bit elements (bf16 or fp16) with the given row
// stride; box 64 x 1 x 128.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int heads, int D,
                     int64_t tok_stride, int fmt) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const int esz = fmt == kFmtE4M3 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)tok_stride * esz};
  cuuint32_t box[3] = {(cuuint32_t)(128 / esz), 1, (cuuint32_t)kTcBM};  // one 128-byte panel
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = fmt == kFmtE4M3   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : fmt == kFmtBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, dt, 3, const_cast<void*>(ptr), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Folds the second-half partials of a split ring step into the running
// state (one warp per query row): with a = the state after the first half and
// b = the partial, O = (w_a O_a + w_b O_b) / (w_a + w_b) and lse = m + ln(w_a
// + w_b), w = exp(lse - m), m = max(lse_a, lse_b) -- the same fold as
// ring_attn_merge.  Rows whose partial saw no key keep the state; rows whose
// state is empty take the partial (their O is not read).
template <int D>
__global__ void __launch_bounds__(256) step_merge_kernel(const FwdParams p, int first_item) {
  constexpr int kRows = kTcBM * kTcQT;
  const int wg = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int s = wg / kRows, t = wg - s * kRows;
  if (s >= p.step_split) return;
  const WorkItem it = decode_work(p, first_item + s);
  const int sq = it.qr * kRows + t;
  if (sq >= p.step_rows) return;
  const float lb = p.split_lse[(int64_t)s * kRows + t];
  if (lb == -INFINITY) return;
  const int64_t li = (int64_t)it.b * p.lse_seq_stride + (int64_t)it.h * p.lse_head_stride + sq;
  float* o = static_cast<float*>(p.out) +
             ((int64_t)(it.b * p.step_rows + sq) * p.heads + it.h) * D;
  const float* ob = p.split_out + ((int64_t)s * kRows + t) * D;
  const float la = p.lse[li];
  constexpr int kPer = D / 32;  // elements per lane
  if (la == -INFINITY) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) o[lane * kPer + j] = ob[lane * kPer + j];
    if (lane == 0) p.lse[li] = lb;
    return;
  }
  const float m = fmaxf(la, lb);
  const float wa = expf(la - m), wb = expf(lb - m);
  const float inv = 1.f / (wa + wb);
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int c = lane * kPer + j;
    o[c] = (wa * o[c] + wb * ob[c]) * inv;
  }
  if (lane == 0) p.lse[li] = m + logf(wa + wb);
}

template <int D, int kFmt>
static cudaError_t launch_tc_t(const FwdParams& p, cudaStream_t stream) {
  using C = TcCfg<D, kFmt>;
  FwdParams pp = p;
  pp.n_qranges = (q_rows_per_seq(p) + kTcBM * kTcQT - 1) / (kTcBM * kTcQT);
  set_striped_order(pp, kTcBM * kTcQT);
  const int64_t items = work_grid(pp, kTcBM * kTcQT);
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  // persistent: one CTA per SM (shared memory and tensor memory allow one).
  // The SM count is cached per device; host threads may launch concurrently,
  // so the cache is atomic (a racing first lookup stores the same value).
  static std::atomic<int> sms_cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int num_sms = sms_cache[dev].load(std::memory_order_relaxed);
  if (!num_sms) {
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        num_sms < 1)
      return cudaErrorInvalidDevice;
    sms_cache[dev].store(num_sms, std::memory_order_relaxed);
  }
  // Dense causal work varies per item: one CTA per item, balanced by the
  // hardware block scheduler, measured faster than persistent CTAs there.
  // Otherwise persistent CTAs (one per SM) claim items until none is left:
  // from the launch's counter, or for ring steps (launched as programmatic
  // dependents of the previous launch, with no counter reset between) by a
  // static stride over the CTAs.
  const bool per_item = p.causal && !p.cu_seqlens && !p.step;
  // A ring step whose items leave the last wave of CTAs at most half full
  // splits those items in halves of their key tiles, so the last wave takes
  // half as long; a merge kernel folds the second halves in afterwards.  The
  // partials live in stream-ordered scratch (without it the step runs
  // unsplit).
  int split = 0;
  float* scratch = nullptr;
  if (p.step && p.step_rows / kTcBN >= 2) {
    const int64_t r = items % num_sms;
    if (r > 0 && 2 * r <= num_sms) {
      const size_t bytes = (size_t)r * (kTcBM * kTcQT) * (D + 1) * sizeof(float);
      if (cudaMallocAsync(reinterpret_cast<void**>(&scratch), bytes, stream) == cudaSuccess) {
        split = (int)r;
      } else {
        (void)cudaGetLastError();
        scratch = nullptr;
      }
    }
  }
  pp.step_split = split;
  pp.split_out = scratch;
  pp.split_lse = scratch ? scratch + (size_t)split * (kTcBM * kTcQT) * D : nullptr;
  const int64_t launch_items = items + split;
  const int64_t grid =
      per_item ? items : (launch_items < num_sms ? launch_items : num_sms);
  const int claim_limit = per_item ? 1 : 0;
  // the scratch goes back to the pool on every exit path below
  auto release = [&](cudaError_t err) -> cudaError_t {
    if (scratch) {
      const cudaError_t f = cudaFreeAsync(scratch, stream);
      if (err == cudaSuccess) err = f;
    }
    return err;
  };
  TcMaps maps;
  if (!make_map(&maps.q, p.q, p.total_rows, p.heads, D, p.tok_stride, kFmt) ||
      !make_map(&maps.k, p.k, p.total_rows, p.heads_kv, D, p.kv_tok_stride, kFmt) ||
      !make_map(&maps.v, p.v, p.total_rows, p.heads_kv, D, p.kv_tok_stride, kFmt))
    return release(cudaErrorInvalidValue);
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D, kFmt>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return release(e);
  if (p.step) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fwd_tc_kernel<D, kFmt>, pp, maps, (int)launch_items,
                           claim_limit);
    if (e == cudaSuccess && split > 0) {
      const int warps = split * kTcBM * kTcQT;
      step_merge_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(
          pp, (int)(items - split));
      e = cudaGetLastError();
    }
    return release(e);
  }
  fwd_tc_kernel<D, kFmt><<<(unsigned)grid, kTcThreads, C::kSmemBytes, stream>>>(
      pp, maps, (int)items, claim_limit);
  return cudaGetLastError();
}

// 16-bit inputs (fmt kFmtBF16 or kFmtF16), d_head 64 or 128; e4m3 inputs
// (kFmtE4M3) with d_head 128, not in ring-step mode.
cudaError_t launch_fwd_tc(const FwdParams& p, int fmt, cudaStream_t stream) {
  if (fmt == kFmtBF16) {
    switch (p.d_head) {
      case 64: return launch_tc_t<64, kFmtBF16>(p, stream);
      case 128: return launch_tc_t<128, kFmtBF16>(p, stream);
    }
  } else if (fmt == kFmtF16) {
    switch (p.d_head) {
      case 64: return launch_tc_t<64, kFmtF16>(p, stream);
      case 128: return launch_tc_t<128, kFmtF16>(p, stream);
    }
  } else if (fmt == kFmtE4M3 && p.d_head == 128 && !p.step) {
    return launch_tc_t<128, kFmtE4M3>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ra

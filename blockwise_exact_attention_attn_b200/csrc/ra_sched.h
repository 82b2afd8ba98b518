// ra_sched.h -- ring-step scheduler: ring geometry, (q-tile, kv-tile) pair
// classification and the ring-order tile walk.  Pure integer code, compiled
// for the host (schedule inspection) and the device (every kernel).
//
// Ring order: query block r meets key/value block (r - step) mod N at ring
// step step = 0, 1, ..., N - 1 ("Ring Attention" glossary, "Come funziona la
// ring attention", four-device simulation: j = (i - step) % n_devices; "Ring
// Attention simulation" gist, Device.run: step 0 uses the device's own block,
// later steps the block received from the previous device).  max ring passes
// P keeps steps 0 .. P-1 (issue thread "A ring attention with flash attention
// kernel implementation": a configurable cap on ring passes).  Causal blocks
// that lie entirely after every query are skipped ("Ring Attention" glossary:
// under a causal mask the devices holding the first query blocks skip most key
// blocks), and the striped layout puts token t in block t mod N (same page,
// Striped Attention).
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

enum : int { CLS_EMPTY = 0, CLS_FULL = 1, CLS_PARTIAL = 2 };
enum : int { LAYOUT_CONTIGUOUS = 0, LAYOUT_STRIPED = 1 };

// Pairs of (q-block, kv-block) segments examined exactly per tile pair; above
// this the classification falls back to PARTIAL (always safe: the element
// mask is then applied).
constexpr int kExactSegmentPairs = 64;

// Geometry of one sequence of length L split into N ring blocks.
struct RingGeom {
  int L;        // tokens in the sequence (>= 1)
  int N;        // ring blocks (>= 1)
  int layout;   // LAYOUT_CONTIGUOUS or LAYOUT_STRIPED
  int causal;   // 0 / 1
  int passes;   // min(max_ring_passes, N), >= 1
  int q;        // striped: L / N
  int rem;      // striped: L % N
};

RA_HD RingGeom make_geom(int L, int N, int layout, int causal, int P) {
  RingGeom g;
  g.L = L;
  g.N = N;
  g.layout = layout;
  g.causal = causal;
  g.passes = P < N ? P : N;
  g.q = L / N;
  g.rem = L % N;
  return g;
}

// floor((a * b + c) / d) for non-negative a, b, c and positive d; 32-bit
// arithmetic whenever the numerator fits (64-bit division is slow on the GPU).
RA_HD int muladd_div(int a, int b, int c, int d) {
  const uint64_t num = (uint64_t)(uint32_t)a * (uint32_t)b + (uint32_t)c;
  if (num <= 0xffffffffull) return (int)((uint32_t)num / (uint32_t)d);
  return (int)(num / (uint64_t)d);
}

// First stored row of ring block r (r in [0, N]; r == N gives L).
//   contiguous: block r = rows t with floor(t*N/L) == r, i.e. [ceil(rL/N), ..)
//   striped   : blocks hold ceil((L - r)/N) rows each, stored in order.
RA_HD int block_start(const RingGeom& g, int r) {
  if (g.layout == LAYOUT_CONTIGUOUS) return muladd_div(r, g.L, g.N - 1, g.N);
  return r * g.q + (r < g.rem ? r : g.rem);
}

// Ring block of stored row s (0 <= s < L).
RA_HD int block_of(const RingGeom& g, int s) {
  if (g.layout == LAYOUT_CONTIGUOUS) return muladd_div(s, g.N, 0, g.L);
  const int big = g.rem * (g.q + 1);  // rows held by the blocks of q+1 rows
  if (s < big) return s / (g.q + 1);
  return g.rem + (s - big) / g.q;     // here q >= 1 because s < L
}

// Original token position of stored row s that lies in ring block r.
RA_HD int token_of(const RingGeom& g, int s, int r) {
  if (g.layout == LAYOUT_CONTIGUOUS) return s;
  return (s - block_start(g, r)) * g.N + r;
}

// Is ring step (rq - rk) mod N within the pass limit?
RA_HD bool pass_ok(const RingGeom& g, int rq, int rk) {
  int d = rq - rk;
  if (d < 0) d += g.N;
  return d < g.passes;
}

// Classify the pair of stored row ranges q in [a, b) of block rq and
// k in [c, d) of block rk (both non-empty and inside their blocks).
// Sets *any when some pair is allowed and clears *all when some is not.
RA_HD void classify_segment(const RingGeom& g, int rq, int a, int b, int rk,
                            int c, int d, bool* any, bool* all) {
  if (!pass_ok(g, rq, rk)) { *all = false; return; }
  if (!g.causal) { *any = true; return; }
  if (g.layout == LAYOUT_CONTIGUOUS) {
    // tokens are stored rows: allowed iff key <= query
    if (c <= b - 1) *any = true;
    if (!(d - 1 <= a)) *all = false;
    return;
  }
  // striped: query token i*N + rq, key token j*N + rk (local i, j);
  // key <= query  iff  j <= i - [rk > rq]
  const int sq = block_start(g, rq), sk = block_start(g, rk);
  const int delta = rk > rq ? 1 : 0;
  const int ia = a - sq, ib = b - sq, ja = c - sk, jb = d - sk;
  if (ja <= ib - 1 - delta) *any = true;
  if (!(jb - 1 <= ia - delta)) *all = false;
}

// Exact class of the tile pair q rows [q0, q1), key rows [k0, k1) of one
// sequence (ranges clipped to [0, L) by the caller).
RA_HD int classify(const RingGeom& g, int q0, int q1, int k0, int k1) {
  if (q0 >= q1 || k0 >= k1) return CLS_EMPTY;
  const int rq0 = block_of(g, q0), rq1 = block_of(g, q1 - 1);
  const int rk0 = block_of(g, k0), rk1 = block_of(g, k1 - 1);
  if ((int64_t)(rq1 - rq0 + 1) * (rk1 - rk0 + 1) > kExactSegmentPairs) {
    // many tiny blocks: only the cheap causal bound is used
    if (g.causal && g.layout == LAYOUT_CONTIGUOUS && k0 > q1 - 1) return CLS_EMPTY;
    return CLS_PARTIAL;
  }
  bool any = false, all = true;
  for (int rq = rq0; rq <= rq1; ++rq) {
    const int bs = block_start(g, rq), be = block_start(g, rq + 1);
    const int a = q0 > bs ? q0 : bs, b = q1 < be ? q1 : be;
    if (a >= b) continue;
    for (int rk = rk0; rk <= rk1; ++rk) {
      const int cs = block_start(g, rk), ce = block_start(g, rk + 1);
      const int c = k0 > cs ? k0 : cs, d = k1 < ce ? k1 : ce;
      if (c >= d) continue;
      classify_segment(g, rq, a, b, rk, c, d, &any, &all);
    }
  }
  if (!any) return CLS_EMPTY;
  return all ? CLS_FULL : CLS_PARTIAL;
}

// Element mask: is stored key s_k allowed for stored query s_q (same
// sequence, both in [0, L))?  Used on PARTIAL tiles.
RA_HD bool allowed(const RingGeom& g, int sq, int rq, int tq, int sk) {
  const int rk = block_of(g, sk);
  if (!pass_ok(g, rq, rk)) return false;
  if (!g.causal) return true;
  return token_of(g, sk, rk) <= tq;
}

// Walk over the kv-tiles (kv_tile rows each, tile kt = rows [kt*BN, ..)) that
// a query row range [q0, q1) visits, in ring order: ring steps 0, 1, ...,
// N - 1 relative to the ring block of row q0; inside one block the tiles whose
// first row lies in that block, ascending.  Every kv-tile of the sequence is
// therefore considered exactly once.  Up to two query sub-ranges (the halves
// [q0, qm) and [qm, q1)) are classified per tile, so a CTA that owns two
// q-tiles can share one walk; a tile is emitted when it is non-EMPTY for at
// least one sub-range.
// Query segments (one per ring block) of a query sub-range, cached by the
// walk so that the tiles lying inside one key block are classified without
// any division.  Slot k holds ring block r0 + k (empty when a >= b); all
// loops over slots are unrolled so the arrays stay in registers.
constexpr int kMaxQSegs = 4;
struct QSegs {
  int n;                      // slots in use, or -1 when there are too many blocks
  int r[kMaxQSegs];           // ring block
  int a[kMaxQSegs], b[kMaxQSegs];  // stored rows [a, b)
  int start[kMaxQSegs];       // first stored row of block r
};

RA_HD void make_qsegs(const RingGeom& g, int lo, int hi, QSegs* s) {
  s->n = 0;
#pragma unroll
  for (int k = 0; k < kMaxQSegs; ++k) {
    s->r[k] = 0;
    s->a[k] = 0;
    s->b[k] = 0;
    s->start[k] = 0;
  }
  if (lo >= hi) return;
  const int r0 = block_of(g, lo), r1 = block_of(g, hi - 1);
  if (r1 - r0 + 1 > kMaxQSegs) { s->n = -1; return; }
  s->n = r1 - r0 + 1;
#pragma unroll
  for (int k = 0; k < kMaxQSegs; ++k) {
    const int r = r0 + k;
    if (k < s->n) {
      const int bs = block_start(g, r), be = block_start(g, r + 1);
      s->r[k] = r;
      s->a[k] = lo > bs ? lo : bs;
      s->b[k] = hi < be ? hi : be;
      s->start[k] = bs;
    }
  }
}

// Class of query segments `s` against key rows [c, d) that lie inside key
// block rk starting at row ks (same rules as classify_segment).
RA_HD int classify_in_block(const RingGeom& g, const QSegs& s, int rk, int ks, int c, int d) {
  bool any = false, all = true;
#pragma unroll
  for (int i = 0; i < kMaxQSegs; ++i) {
    if (i >= s.n || s.a[i] >= s.b[i]) continue;
    const int rq = s.r[i];
    if (!pass_ok(g, rq, rk)) { all = false; continue; }
    if (!g.causal) { any = true; continue; }
    if (g.layout == LAYOUT_CONTIGUOUS) {
      if (c <= s.b[i] - 1) any = true;
      if (!(d - 1 <= s.a[i])) all = false;
    } else {
      const int delta = rk > rq ? 1 : 0;
      const int ia = s.a[i] - s.start[i], ib = s.b[i] - s.start[i];
      const int ja = c - ks, jb = d - ks;
      if (ja <= ib - 1 - delta) any = true;
      if (!(jb - 1 <= ia - delta)) all = false;
    }
  }
  if (!any) return CLS_EMPTY;
  return all ? CLS_FULL : CLS_PARTIAL;
}

struct TileWalk {
  RingGeom g;
  int q0, qm, q1;   // sub-range 0 = [q0, qm), sub-range 1 = [qm, q1)
  QSegs seg0, seg1; // their per-block segments
  int kbs, kbe;     // stored rows of the current key block
  int BN;
  int rq_ref;       // ring block of q0
  int rqa, rqb;     // ring blocks spanned by [q0, q1)
  int tmax;         // largest original token among rows [q0, q1)
  int step;         // current ring step
  int rk;           // current key block
  int kt, kt_end;   // remaining tiles lying wholly inside the current block
  int kt_cross;     // tile starting in this block and ending in a later one, or -1

  RA_HD void init(const RingGeom& geom, int q_begin, int q_mid, int q_end,
                  int kv_tile) {
    g = geom;
    q0 = q_begin; qm = q_mid; q1 = q_end;
    BN = kv_tile;
    make_qsegs(g, q0, qm, &seg0);
    make_qsegs(g, qm, q1, &seg1);
    kbs = kbe = 0;
    rq_ref = block_of(g, q0);
    rqa = rq_ref;
    rqb = block_of(g, q1 - 1);
    // largest token of the query range
    if (g.layout == LAYOUT_CONTIGUOUS) {
      tmax = q1 - 1;
    } else {
      tmax = 0;
      for (int r = rqa; r <= rqb; ++r) {
        const int be = block_start(g, r + 1);
        const int last = (q1 < be ? q1 : be) - 1;
        if (last >= block_start(g, r)) {
          const int t = token_of(g, last, r);
          if (t > tmax) tmax = t;
        }
      }
    }
    step = -1;
    kt = 0;
    kt_end = 0;
    kt_cross = -1;
  }

  // Is key block rk reachable by any query block of [rqa, rqb] within the
  // pass limit?
  RA_HD bool block_passes(int r) const {
    if (g.passes >= g.N) return true;
    if (rqb - rqa + 1 >= g.N) return true;
    for (int x = rqa; x <= rqb; ++x)
      if (pass_ok(g, x, r)) return true;
    return false;
  }

  // Advance to the next block with candidate tiles; false when done.
  // The tiles of block rk are those whose first row lies in it.  The last of
  // them may reach into later blocks; that one is always classified exactly.
  // The others lie wholly inside block rk, so the block-level pass test and
  // the causal frontier of block rk may drop them without looking.
  RA_HD bool next_block() {
    while (true) {
      ++step;
      if (step >= g.N) return false;
      rk = rq_ref - step;
      if (rk < 0) rk += g.N;
      const int bs = block_start(g, rk), be = block_start(g, rk + 1);
      if (bs >= be) continue;
      kbs = bs;
      kbe = be;
      kt = (bs + BN - 1) / BN;
      const int kt_all = (be + BN - 1) / BN;  // tiles starting in [bs, be)
      if (kt >= kt_all) continue;
      kt_cross = -1;
      kt_end = kt_all;
      if ((int64_t)kt_all * BN > be && kt_all * BN - BN < be && be < g.L) {
        kt_cross = kt_all - 1;
        kt_end = kt_all - 1;
      }
      if (!block_passes(rk)) {
        kt_end = kt;  // whole-block tiles all fail the pass limit
      } else if (g.causal) {
        // keys of block rk with token <= tmax form a prefix of the block
        int lim;
        if (g.layout == LAYOUT_CONTIGUOUS) {
          lim = tmax;
        } else {
          lim = tmax < rk ? -1 : bs + (tmax - rk) / g.N;
        }
        const int kt_lim = lim < bs ? kt : lim / BN + 1;
        if (kt_lim < kt_end) kt_end = kt_lim;
        if (kt_end < kt) kt_end = kt;
      }
      if (kt >= kt_end && kt_cross < 0) continue;
      return true;
    }
  }

  // Next visited tile: returns false when the walk is over, else sets the
  // tile index and the class for each query sub-range (CLS_EMPTY for an empty
  // sub-range).
  RA_HD bool next(int* tile, int* cls0, int* cls1) {
    while (true) {
      int t;
      bool inner;
      if (kt < kt_end) {
        t = kt++;
        inner = true;
      } else if (kt_cross >= 0) {
        t = kt_cross;
        kt_cross = -1;
        inner = false;
      } else {
        if (!next_block()) return false;
        continue;
      }
      const int k0 = t * BN;
      const int k1 = (k0 + BN < g.L) ? k0 + BN : g.L;
      int c0, c1;
      if (inner && seg0.n >= 0 && seg1.n >= 0) {
        // tile inside key block rk: division-free classification
        c0 = classify_in_block(g, seg0, rk, kbs, k0, k1);
        c1 = classify_in_block(g, seg1, rk, kbs, k0, k1);
      } else {
        c0 = classify(g, q0, qm, k0, k1);
        c1 = classify(g, qm, q1, k0, k1);
      }
      if (c0 == CLS_EMPTY && c1 == CLS_EMPTY) continue;
      *tile = t;
      *cls0 = c0;
      *cls1 = c1;
      return true;
    }
  }
};

}  // namespace ra

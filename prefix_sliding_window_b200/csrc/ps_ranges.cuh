// Integer geometry of the Prefix Sliding mask, shared by host and device code of libps:
// visible ranges of a decode query, their split into TMA tiles, and the prefill tile plan.
//
// Mask ("Prefix Sliding 完全拆解", §核心机制, eq. A(i), 0-indexed): the query at position
// p sees k iff k <= p and (k < Lp or k > p - W).  With n = p + 1 this is the prefix rows
// [0, min(n, Lp)) plus the window positions [max(Lp, n - W), n), i.e. at most Lp + W keys
// (eq. L_total).
#pragma once

#include <stdint.h>

#include "../../include/ps.h"

#ifdef __CUDACC__
#define PS_HD __host__ __device__ __forceinline__
#else
#define PS_HD inline
#endif

namespace ps {

// Keys per decode tile (one TMA box height).
constexpr int kDecodeTile = 64;

struct VisibleRanges {
  int32_t pre_len;     // prefix rows [0, pre_len)
  int32_t seg0_start;  // ring slots [seg0_start, seg0_start + seg0_len)
  int32_t seg0_len;
  int32_t seg1_len;    // ring slots [0, seg1_len) after the wrap
};

// Visible ranges of the query at position p (p >= 0).  Ring slot of position q >= Lp is
// (q - Lp) mod W.  The window positions [wstart, n) are contiguous, so their slots form
// at most two runs: [s0, W) and [0, ...).
// x mod w for x >= 0, w > 0: a 32-bit remainder when x fits (the case in practice), which
// on the GPU is a few instructions against a long emulated 64-bit division.
PS_HD int64_t mod_nonneg(int64_t x, int32_t w) {
  if (x < (int64_t(1) << 32)) return int64_t(uint32_t(x) % uint32_t(w));
  return x % w;
}

PS_HD VisibleRanges visible_ranges(int64_t p, int32_t lp, int32_t w) {
  VisibleRanges r;
  const int64_t n = p + 1;
  r.pre_len = static_cast<int32_t>(n < lp ? n : lp);
  const int64_t wstart = (n - w > lp) ? (n - w) : lp;
  const int64_t win = n - wstart > 0 ? n - wstart : 0;
  if (win == 0) {
    r.seg0_start = 0;
    r.seg0_len = 0;
    r.seg1_len = 0;
    return r;
  }
  const int64_t s0 = mod_nonneg(wstart - lp, w);
  const int64_t room = w - s0;
  r.seg0_start = static_cast<int32_t>(s0);
  r.seg0_len = static_cast<int32_t>(win < room ? win : room);
  r.seg1_len = static_cast<int32_t>(win - r.seg0_len);
  return r;
}

PS_HD int32_t ceil_div_i32(int32_t a, int32_t b) { return (a + b - 1) / b; }

// One TMA tile of the visible key sequence: `rows` box rows starting at `row0` of map
// `map_id` (0 = prefix / linear cache, 1 = ring); rows [lo, hi) of the box are visible.
// Rows outside [lo, hi) are outside the tensor (TMA fills them with zeros).
struct DecodeTile {
  int32_t map_id;
  int32_t row0;
  int32_t lo;
  int32_t hi;
};

// Tiling of the (up to three) segments.  A segment that ends at the end of its tensor
// dimension is tiled forward from its start, so the last box runs past the end of the
// tensor; every other segment starts at row 0 and is tiled backward from its end, so the
// first box starts at a negative row.  Either way no box reads a row that is inside the
// tensor but outside the segment, so no invisible key is ever loaded.
struct DecodeTiling {
  int32_t nt[3];       // tiles per segment
  int32_t begin[3];    // first row of the segment
  int32_t end[3];      // one past the last row
  int32_t forward[3];  // 1: tiled forward from begin; 0: backward from end; 2: tiles on
                       // 64-row block boundaries (paged stores), rows outside masked
  int32_t map_id[3];
  int32_t total;
};

// dim_prefix: rows of the prefix (or linear) tensor dimension; w: ring rows.
PS_HD DecodeTiling make_tiling(const VisibleRanges& r, int32_t dim_prefix, int32_t w) {
  DecodeTiling t;
  // segment 0: prefix rows [0, pre_len)
  t.begin[0] = 0;
  t.end[0] = r.pre_len;
  t.forward[0] = (r.pre_len == dim_prefix) ? 1 : 0;
  t.map_id[0] = 0;
  // segment 1: ring [s0, s0 + l0); either it ends at W or it starts at slot 0
  t.begin[1] = r.seg0_start;
  t.end[1] = r.seg0_start + r.seg0_len;
  t.forward[1] = (t.end[1] == w) ? 1 : 0;
  t.map_id[1] = 1;
  // segment 2: ring [0, l1)
  t.begin[2] = 0;
  t.end[2] = r.seg1_len;
  t.forward[2] = (r.seg1_len == w) ? 1 : 0;
  t.map_id[2] = 1;
  t.total = 0;
  for (int s = 0; s < 3; ++s) {
    t.nt[s] = ceil_div_i32(t.end[s] - t.begin[s], kDecodeTile);
    t.total += t.nt[s];
  }
  return t;
}

// Tiling of a paged store: every segment cut on 64-row block boundaries (a tile is one block;
// rows outside the segment are masked by the tile's [lo, hi)).
PS_HD DecodeTiling make_tiling_paged(const VisibleRanges& r) {
  DecodeTiling t;
  t.begin[0] = 0;
  t.end[0] = r.pre_len;
  t.map_id[0] = 0;
  t.begin[1] = r.seg0_start;
  t.end[1] = r.seg0_start + r.seg0_len;
  t.map_id[1] = 1;
  t.begin[2] = 0;
  t.end[2] = r.seg1_len;
  t.map_id[2] = 1;
  t.total = 0;
  for (int s = 0; s < 3; ++s) {
    t.forward[s] = 2;
    t.nt[s] = t.end[s] > t.begin[s]
                  ? ceil_div_i32(t.end[s], kDecodeTile) - t.begin[s] / kDecodeTile
                  : 0;
    t.total += t.nt[s];
  }
  return t;
}

PS_HD DecodeTile tiling_tile(const DecodeTiling& t, int32_t idx) {
  // segment selection with constant indices only (keeps the tiling in registers)
  int32_t begin, end, fwd, map_id, nt;
  if (idx < t.nt[0]) {
    begin = t.begin[0]; end = t.end[0]; fwd = t.forward[0]; map_id = t.map_id[0]; nt = t.nt[0];
  } else if (idx < t.nt[0] + t.nt[1]) {
    idx -= t.nt[0];
    begin = t.begin[1]; end = t.end[1]; fwd = t.forward[1]; map_id = t.map_id[1]; nt = t.nt[1];
  } else {
    idx -= t.nt[0] + t.nt[1];
    begin = t.begin[2]; end = t.end[2]; fwd = t.forward[2]; map_id = t.map_id[2]; nt = t.nt[2];
  }
  DecodeTile d;
  d.map_id = map_id;
  if (fwd == 2) {
    d.row0 = (begin / kDecodeTile + idx) * kDecodeTile;
    d.lo = begin > d.row0 ? begin - d.row0 : 0;
    const int32_t left = end - d.row0;
    d.hi = left < kDecodeTile ? left : kDecodeTile;
  } else if (fwd) {
    d.row0 = begin + idx * kDecodeTile;
    d.lo = 0;
    const int32_t left = end - d.row0;
    d.hi = left < kDecodeTile ? left : kDecodeTile;
  } else {
    d.row0 = end - (nt - idx) * kDecodeTile;
    d.lo = d.row0 < begin ? begin - d.row0 : 0;
    d.hi = kDecodeTile;
  }
  return d;
}

// ----------------------------------------------------------- prefill tile plan
// Query tile qt covers rows [qt*bq, qt*bq + bq); key tile kt covers [kt*bk, kt*bk + bk).
// Closed-form classification ("Prefix Sliding 完全拆解", §Kernel 实现):
//   SKIP    - no row/column pair of the tile is visible (never loaded, never computed);
//   FULL    - every one of the bq*bk pairs is in range (< seq) and visible;
//   PARTIAL - otherwise (element-wise mask).
// Returns 0 for SKIP, 1 (PS_TILE_FULL) or 2 (PS_TILE_PARTIAL).
PS_HD int32_t classify_tile(int64_t qt, int64_t kt, int64_t seq, int32_t lp, int32_t w,
                            int32_t bq, int32_t bk) {
  const int64_t q0 = qt * bq, k0 = kt * bk;
  if (q0 >= seq || k0 >= seq) return 0;
  const int64_t imax = (q0 + bq < seq ? q0 + bq : seq) - 1;  // last in-range row
  const int64_t k1 = (k0 + bk < seq ? k0 + bk : seq);        // one past last in-range col
  // any visible pair?  prefix part: column k0 < Lp with k0 <= some row.
  bool any = (k0 < lp) && (k0 <= imax);
  if (!any && lp < k1) {
    // window part: a row i in [max(q0,k0,lp), min(imax, k1+w-2)] exists
    int64_t lo = q0 > k0 ? q0 : k0;
    if (lp > lo) lo = lp;
    const int64_t hi = imax < k1 + w - 2 ? imax : k1 + w - 2;
    any = lo <= hi;
  }
  if (!any) return 0;
  const bool in_range = (q0 + bq <= seq) && (k0 + bk <= seq);
  const int64_t kmax = k0 + bk - 1;
  const int64_t qmax = q0 + bq - 1;
  const bool causal_ok = kmax <= q0;
  const int64_t kwin = k0 > lp ? k0 : lp;  // smallest column that must be in the window
  const bool mask_ok = (kmax < lp) || (kwin > qmax - w);
  return (in_range && causal_ok && mask_ok) ? PS_TILE_FULL : PS_TILE_PARTIAL;
}

// Candidate key-tile ranges of query tile qt: prefix tiles [0, pe) and window tiles
// [ws, we]; the plan is their union in ascending order, SKIP tiles dropped.
PS_HD void qtile_candidates(int64_t qt, int64_t seq, int32_t lp, int32_t w, int32_t bq,
                            int32_t bk, int64_t* pe, int64_t* ws, int64_t* we) {
  const int64_t q0 = qt * bq;
  const int64_t imax = (q0 + bq < seq ? q0 + bq : seq) - 1;
  *pe = (lp + bk - 1) / bk;
  int64_t first_win_col = q0 - w + 1;
  if (first_win_col < lp) first_win_col = lp;
  *ws = first_win_col / bk;
  *we = imax / bk;
  if (*ws < *pe) *ws = *pe;  // union: do not list a tile twice
}

// Position of key tile kt in query tile qt's plan, for a (qt, kt) pair that is in it (square
// tiles, b = Bq = Bk).  A prefix tile (kt < pe) is visible to qt iff kt <= qt, and every
// window candidate in [ws, we] is non-SKIP (its first key is within W - 1 of the tile's
// first row, its last key is at most the tile's last row), so the plan is [0, min(pe,
// qt + 1)) followed by [ws, we].
PS_HD int64_t plan_index(int64_t qt, int64_t kt, int32_t lp, int32_t w, int32_t b) {
  const int64_t pe = (lp + b - 1) / b;
  if (kt < pe) return kt;
  int64_t first_win_col = qt * b - w + 1;
  if (first_win_col < lp) first_win_col = lp;
  int64_t ws = first_win_col / b;
  if (ws < pe) ws = pe;
  return (pe < qt + 1 ? pe : qt + 1) + (kt - ws);
}

// Number of non-SKIP tiles of query tile qt.
PS_HD int64_t qtile_count(int64_t qt, int64_t seq, int32_t lp, int32_t w, int32_t bq,
                          int32_t bk) {
  int64_t pe, ws, we;
  qtile_candidates(qt, seq, lp, w, bq, bk, &pe, &ws, &we);
  int64_t c = 0;
  const int64_t kt_last = (seq - 1) / bk;
  for (int64_t kt = 0; kt < pe && kt <= kt_last; ++kt)
    if (classify_tile(qt, kt, seq, lp, w, bq, bk)) ++c;
  for (int64_t kt = ws; kt <= we; ++kt)
    if (classify_tile(qt, kt, seq, lp, w, bq, bk)) ++c;
  return c;
}

// Query tiles that hold a visible pair with key tile kt (square tiles, b = Bq = Bk):
// key k is seen by the queries [k, seq) when k < lp and [k, min(seq, k + w)) otherwise; over
// the keys of the tile these intervals overlap, so their union [k0, last] is contiguous and
// every query tile in [k0 / b, last / b] is non-SKIP.  Returns false if the tile is empty.
PS_HD bool ktile_qrange(int64_t kt, int64_t seq, int32_t lp, int32_t w, int32_t b, int64_t* qlo,
                        int64_t* qhi) {
  const int64_t k0 = kt * b;
  if (k0 >= seq) return false;
  const int64_t k1 = (k0 + b < seq ? k0 + b : seq);  // one past the last in-range key
  int64_t last = seq - 1;
  if (k0 >= lp) {
    const int64_t l = k1 - 1 + w - 1;  // last query that sees the tile's last key
    if (l < last) last = l;
  }
  *qlo = k0 / b;
  *qhi = last / b;
  return true;
}

}  // namespace ps

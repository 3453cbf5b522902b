// dca_plan.cuh -- tile classification of Dual Chunk Attention, shared by the
// host code and the kernels of the CUDA path.
//
// "Qwen2.5-1M 不重训外推 1M", section 核心思想, splits the causal L x L score
// matrix into intra-chunk, successive-chunk and inter-chunk parts.  With
// n_x = x / s, a (query i, key j) pair has chunk distance n_i - n_j:
//   0 -> INTRA  (query rotated by r_i)
//   1 -> SUCC   (query rotated by s + r_i when r_i < w, else by c - 1)
//  >=2 -> INTER (query rotated by c - 1)
// and every key is rotated by j mod s.  The query rotation therefore depends
// only on the row and the class, so a (q-tile, k-tile) pair whose pairs all
// share one class is one plain MMA with that class's rotated Q.
//
// For a q-tile with rows [i0, i_last] the keys of each class form one
// contiguous range (a superset under reading B's diagonal window), so the
// k-tiles carrying a class are one contiguous range too.  A q-tile's work list is: INTER k-tiles, then SUCC k-tiles, then INTRA
// k-tiles (one Q rotation per phase).  A k-tile that holds keys of several
// classes appears once per class and is masked per element to that class;
// tiles crossing the causal diagonal are masked to j <= i.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define DCA_HD __host__ __device__ __forceinline__
#else
#define DCA_HD inline
#endif

namespace dca {

enum : int { CLS_INTRA = 0, CLS_SUCC = 1, CLS_INTER = 2 };

struct TilePlan {
  int lo[3];  // first k-tile of each class (indexed by CLS_*)
  int hi[3];  // one past the last k-tile
  int n_items;
};

DCA_HD int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

DCA_HD int class_of_distance(int64_t chunk_dist) {
  return chunk_dist <= 0 ? CLS_INTRA : (chunk_dist == 1 ? CLS_SUCC : CLS_INTER);
}

// Window readings of section "Successive-Chunk Attention":
//   READING_A: an adjacent-chunk pair keeps its true distance when the query's
//              offset in its chunk r_i < w (the query rotation depends on the
//              row only: s + r_i, or c - 1 when r_i >= w);
//   READING_B: an adjacent-chunk pair keeps its true distance when i - j < w;
//              the other adjacent-chunk pairs take the inter-chunk rule and are
//              processed with the INTER rotation (c - 1).
enum : int { READING_A = 0, READING_B = 1 };

// Work-list class of pair (i, j), j <= i, with chunk distance dn.
DCA_HD int pair_class(int64_t dn, int64_t i_minus_j, int64_t w, int reading) {
  if (dn <= 0) return CLS_INTRA;
  if (dn == 1 && (reading == READING_A || i_minus_j < w)) return CLS_SUCC;
  return CLS_INTER;
}

// Work list of the q-tile whose real rows are [i0, i_last] (absolute indices),
// for key tiles of `bn` keys.
DCA_HD TilePlan make_plan(int64_t i0, int64_t i_last, int64_t s, int64_t w, int bn,
                          int reading) {
  TilePlan P;
  const int64_t n0 = i0 / s, n1 = i_last / s;
  // INTER: keys with n_j <= n1 - 2, i.e. j < s*(n1-1); under reading B also the
  // adjacent-chunk keys j <= i - w of some row (j < min(s*n1, i_last - w + 1))
  int64_t inter_end = (n1 >= 2) ? s * (n1 - 1) : 0;
  if (reading == READING_B && n1 >= 1) {
    const int64_t far_end = (s * n1 < i_last - w + 1) ? s * n1 : i_last - w + 1;
    if (far_end > inter_end) inter_end = far_end;
  }
  P.lo[CLS_INTER] = 0;
  P.hi[CLS_INTER] = static_cast<int>(cdiv64(inter_end, bn));
  // SUCC: keys with n_j in [n0-1, n1-1]; under reading B only those with
  // i - j < w for some row (j > i0 - w)
  if (n1 >= 1 && (reading == READING_A || w > 0)) {
    int64_t a = s * (n0 >= 1 ? n0 - 1 : 0);
    const int64_t b = s * n1;
    if (reading == READING_B && i0 - w + 1 > a) a = i0 - w + 1;
    P.lo[CLS_SUCC] = static_cast<int>(a / bn);
    P.hi[CLS_SUCC] = a < b ? static_cast<int>(cdiv64(b, bn)) : P.lo[CLS_SUCC];
  } else {
    P.lo[CLS_SUCC] = P.hi[CLS_SUCC] = 0;
  }
  // INTRA: keys with n_j in [n0, n1] and j <= i_last
  P.lo[CLS_INTRA] = static_cast<int>((s * n0) / bn);
  P.hi[CLS_INTRA] = static_cast<int>(i_last / bn) + 1;
  P.n_items = (P.hi[CLS_INTER] - P.lo[CLS_INTER]) + (P.hi[CLS_SUCC] - P.lo[CLS_SUCC]) +
              (P.hi[CLS_INTRA] - P.lo[CLS_INTRA]);
  return P;
}

// Key ranges [lo, hi) of the three classes for the query rows [i0, i_last]
// (the unions over the rows; the k-tile ranges of make_plan are these ranges
// rounded out to tiles).  A pair (i, j) of class c has j inside range c.
DCA_HD void class_key_ranges(int64_t i0, int64_t i_last, int64_t s, int64_t w, int reading,
                             int64_t lo[3], int64_t hi[3]) {
  const int64_t n0 = i0 / s, n1 = i_last / s;
  int64_t inter_end = (n1 >= 2) ? s * (n1 - 1) : 0;
  if (reading == READING_B && n1 >= 1) {
    const int64_t far_end = (s * n1 < i_last - w + 1) ? s * n1 : i_last - w + 1;
    if (far_end > inter_end) inter_end = far_end;
  }
  lo[CLS_INTER] = 0;
  hi[CLS_INTER] = inter_end;
  if (n1 >= 1 && (reading == READING_A || w > 0)) {
    int64_t a = s * (n0 >= 1 ? n0 - 1 : 0);
    const int64_t b = s * n1;
    if (reading == READING_B && i0 - w + 1 > a) a = i0 - w + 1;
    lo[CLS_SUCC] = a;
    hi[CLS_SUCC] = a < b ? b : a;
  } else {
    lo[CLS_SUCC] = hi[CLS_SUCC] = 0;
  }
  lo[CLS_INTRA] = s * n0;
  hi[CLS_INTRA] = i_last + 1;
}

// Keys [lo, hi) that pair with query row i in work-list class `cls` (causal
// j <= i included): one contiguous range per row and class.  INTRA: the
// row's own chunk up to i; SUCC: chunk n_i - 1 (reading B: only i - j < w);
// INTER: chunks up to n_i - 2 (reading B: also chunk n_i - 1 where
// i - j >= w).  Works in any signed integer type holding i, s and w.
template <class I>
DCA_HD void row_key_range(I i, int cls, I s, I w, int reading, I& lo, I& hi) {
  const I ni = i / s;
  if (cls == CLS_INTRA) {
    lo = s * ni;
    hi = i + 1;
    return;
  }
  if (ni == 0) {
    lo = hi = 0;
    return;
  }
  const I a = s * (ni - 1), b = s * ni;
  if (cls == CLS_SUCC) {
    lo = a;
    hi = b;
    if (reading == READING_B && i - w + 1 > lo) lo = i - w + 1;
    if (hi < lo) hi = lo;
    return;
  }
  lo = 0;
  hi = a;
  if (reading == READING_B) {
    const I f = (i - w + 1 < b) ? i - w + 1 : b;
    if (f > hi) hi = f;
  }
}

// Item n of the work list -> (k-tile, class).  Order: INTER, SUCC, INTRA.
DCA_HD void plan_item(const TilePlan& P, int n, int& kt, int& cls) {
  const int c2 = P.hi[CLS_INTER] - P.lo[CLS_INTER];
  const int c1 = P.hi[CLS_SUCC] - P.lo[CLS_SUCC];
  if (n < c2) {
    cls = CLS_INTER;
    kt = P.lo[CLS_INTER] + n;
  } else if (n < c2 + c1) {
    cls = CLS_SUCC;
    kt = P.lo[CLS_SUCC] + (n - c2);
  } else {
    cls = CLS_INTRA;
    kt = P.lo[CLS_INTRA] + (n - c2 - c1);
  }
}

// True when every (i, j) with i in [i0, i_hi], j in [j0, j_hi] is causal
// (j <= i) and of class `cls`: the tile needs no per-element mask.
DCA_HD bool item_is_full(int64_t i0, int64_t i_hi, int64_t j0, int64_t j_hi, int64_t s,
                         int64_t w, int cls, int reading) {
  const int64_t ni0 = i0 / s, ni1 = i_hi / s, nj0 = j0 / s, nj1 = j_hi / s;
  if (cls == CLS_INTER)
    return ni0 - nj1 >= 2 || (reading == READING_B && ni0 - nj1 >= 1 && i0 - j_hi >= w);
  if (cls == CLS_SUCC)
    return (ni0 - nj1 >= 1) && (ni1 - nj0 <= 1) && (reading == READING_A || i_hi - j0 < w);
  return ni0 == ni1 && nj0 == nj1 && ni0 == nj0 && j_hi <= i0;
}

// Per class, the k-tiles [lo, hi) that need no mask for the query tile whose
// rows are [i0, i_hi] (same predicate as item_is_full, solved for kt once per
// tile so the kernels avoid per-item 64-bit divisions).
struct FullRanges {
  int lo[3];
  int hi[3];
};

DCA_HD int64_t floor_div64(int64_t a, int64_t b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

DCA_HD FullRanges make_full_ranges(int64_t i0, int64_t i_hi, int64_t s, int64_t w, int bn,
                                   int reading) {
  FullRanges F;
  const int64_t ni0 = i0 / s, ni1 = i_hi / s;
  // INTER: j_hi < s*(ni0-1)  <=>  (kt+1)*bn <= s*(ni0-1); under reading B also
  // j_hi < s*ni0 with j_hi <= i0 - w
  F.lo[CLS_INTER] = 0;
  {
    int64_t hi = ni0 >= 1 ? floor_div64(s * (ni0 - 1), bn) : 0;
    if (reading == READING_B && ni0 >= 1) {
      const int64_t end = (s * ni0 < i0 - w + 1) ? s * ni0 : i0 - w + 1;
      const int64_t hb = floor_div64(end, bn);
      if (hb > hi) hi = hb;
    }
    F.hi[CLS_INTER] = static_cast<int>(hi > 0 ? hi : 0);
  }
  // SUCC: j_hi < s*ni0 and j0 >= s*(ni1-1); under reading B also j0 > i_hi - w
  {
    int64_t lo = ni1 >= 1 ? cdiv64(s * (ni1 - 1), bn) : 0;
    if (reading == READING_B) {
      const int64_t lb = (i_hi - w + 1) > 0 ? cdiv64(i_hi - w + 1, bn) : 0;
      if (lb > lo) lo = lb;
    }
    const int64_t hi = floor_div64(s * ni0, bn);
    F.lo[CLS_SUCC] = static_cast<int>(lo);
    F.hi[CLS_SUCC] = static_cast<int>(hi > lo ? hi : lo);
  }
  // INTRA: one chunk for all rows, j0 >= s*ni0, j_hi < s*(ni0+1), j_hi <= i0
  if (ni0 == ni1) {
    const int64_t lo = cdiv64(s * ni0, bn);
    const int64_t end = (s * (ni0 + 1) < i0 + 1) ? s * (ni0 + 1) : i0 + 1;
    const int64_t hi = floor_div64(end, bn);
    F.lo[CLS_INTRA] = static_cast<int>(lo);
    F.hi[CLS_INTRA] = static_cast<int>(hi > lo ? hi : lo);
  } else {
    F.lo[CLS_INTRA] = F.hi[CLS_INTRA] = 0;
  }
  return F;
}

DCA_HD bool is_full(const FullRanges& F, int kt, int cls) {
  return kt >= F.lo[cls] && kt < F.hi[cls];
}

// Position (row of the RoPE table) by which query row i is rotated in class
// `cls`.  The table stores positions [0, min(s, cap)) directly, positions
// [s, s + w) directly when cap > s, and position c - 1 at row `tab_c1`.
DCA_HD int64_t query_table_row(int64_t i, int cls, int64_t s, int64_t w, int64_t tab_c1) {
  const int64_t r = i % s;
  if (cls == CLS_INTRA) return r;
  if (cls == CLS_SUCC && r < w) return s + r;
  return tab_c1;
}

// Number of table rows for key capacity `cap`: direct rows plus one for c - 1.
DCA_HD int64_t table_rows(int64_t cap, int64_t s, int64_t w) {
  const int64_t direct = (cap < s ? cap : s) + (cap > s ? w : 0);
  return direct + 1;
}

}  // namespace dca

// dca_sparse_plan.cuh -- the work list of one (128-row query tile, query
// head) of the vertical-slash sparse attention, shared by the kernel (which
// keeps the plan in shared memory) and the host introspection entry point.
//
// Items are windows of 128 keys, visited class by class (INTER, SUCC, INTRA;
// see dca_plan.cuh); within a class first the 128-position tiles of the
// head's gathered vertical keys whose positions fall in the class's key
// range, then windows of cache keys covering what the slash diagonals (and
// the diagonal j = i) reach from the rows of the tile: each run of slash
// offsets reaches one contiguous key range, the ranges are merged, and each
// merged range, clipped to the class's key range, is covered by windows that
// start at its first key (not at a tile boundary: a lone far diagonal reaches
// 128 keys, one window).  Ranges closer than 128 keys are merged, so a
// window that runs past the end of its range never reaches the next one.  A
// key shared by two classes is visited once per class; the kernel masks each
// item to its class and its member pairs.
#pragma once
#include <stdint.h>
#include <vector_types.h>

#include "dca_plan.cuh"

namespace dca {

constexpr int SPARSE_IV_MAX = 1024;  // slash runs per head (1023) + the diagonal j = i

struct SparsePlan {
  int n_items;
  int n_iv;            // merged slash key-tile intervals
  int nv_eff;          // vertical keys <= the tile's last row
  int vt[3][2];        // vertical (gathered) tile range per class (indexed by CLS_*)
  int kr[3][2];        // cache key range [lo, hi) per class
  int2 iv[SPARSE_IV_MAX];  // [x, y) key ranges reached by the slashes, ascending
};

DCA_HD int sparse_class_at(int ci) {  // visiting order INTER, SUCC, INTRA
  return ci == 0 ? CLS_INTER : (ci == 1 ? CLS_SUCC : CLS_INTRA);
}

struct SparseIter {
  int ci, phase;  // class index in visiting order; -1 start, 0 vertical, 1 slash
  int t, t_end;   // start of the next item and the end of the current range
  int iv;         // slash range index
};

DCA_HD void sparse_iter_init(SparseIter& it) {
  it.ci = 0;
  it.phase = -1;
  it.t = it.t_end = 0;
  it.iv = 0;
}

// Next item: src 0 = vertical, `start` = first position in the gathered
// keys (a multiple of 128); src 1 = slash, `start` = first cache key of the
// 128-key window.
DCA_HD bool sparse_iter_next(SparseIter& it, const SparsePlan& P, int& src, int& start, int& cls) {
  for (;;) {
    if (it.phase >= 0 && it.t < it.t_end) {
      src = it.phase;
      start = it.t;
      it.t += 128;
      cls = sparse_class_at(it.ci);
      return true;
    }
    if (it.phase == 1) {
      const int c = sparse_class_at(it.ci);
      const int clo = P.kr[c][0], chi = P.kr[c][1];
      while (it.iv < P.n_iv) {
        const int2 r = P.iv[it.iv];
        if (r.x >= chi) break;
        ++it.iv;
        const int a = r.x > clo ? r.x : clo;
        const int b = r.y < chi ? r.y : chi;
        if (a < b) {
          it.t = a;
          it.t_end = b;
          break;
        }
      }
      if (it.t < it.t_end) continue;
      ++it.ci;
      it.phase = -1;
    }
    if (it.ci >= 3) return false;
    const int c = sparse_class_at(it.ci);
    if (it.phase == -1) {
      it.phase = 0;
      it.t = P.vt[c][0] * 128;
      it.t_end = P.vt[c][1] * 128;
      continue;
    }
    // vertical tiles done: slash ranges from the first that reaches the class
    it.phase = 1;
    it.iv = 0;
    while (it.iv < P.n_iv && P.iv[it.iv].y <= P.kr[c][0]) ++it.iv;
    it.t = it.t_end = 0;
  }
}

// The plan is built in stages that the host and the kernel share; only the
// lookups differ (the kernel loads the runs and searches the vertical list
// with a whole warp).
//
// Stage 1: the class key ranges of the tile's rows.
DCA_HD void sparse_plan_ranges(SparsePlan& P, int64_t i0, int64_t i_last, int64_t s, int64_t w,
                               int reading, int64_t klo[3], int64_t khi[3]) {
  class_key_ranges(i0, i_last, s, w, reading, klo, khi);
  for (int c = 0; c < 3; ++c) {
    P.kr[c][0] = static_cast<int>(klo[c]);
    P.kr[c][1] = static_cast<int>(khi[c] > klo[c] ? khi[c] : klo[c]);
  }
}

// The keys whose position in the sorted vertical list the plan needs:
// SPARSE_NKEYS lower bounds (i_last + 1, then lo and hi of each class).
constexpr int SPARSE_NKEYS = 7;
DCA_HD void sparse_plan_keys(int64_t i_last, const int64_t klo[3], const int64_t khi[3],
                             int64_t key[SPARSE_NKEYS]) {
  key[0] = i_last + 1;
  for (int c = 0; c < 3; ++c) {
    key[1 + 2 * c] = klo[c];
    key[2 + 2 * c] = khi[c];
  }
}

// Stage 2: vertical tile ranges per class from those lower bounds.
DCA_HD void sparse_plan_vertical(SparsePlan& P, const int64_t klo[3], const int64_t khi[3],
                                 const int pos[SPARSE_NKEYS], int bn) {
  P.nv_eff = pos[0];
  for (int c = 0; c < 3; ++c) {
    int a = 0, b = 0;
    if (khi[c] > klo[c]) {
      a = pos[1 + 2 * c];
      b = pos[2 + 2 * c];
      if (b > P.nv_eff) b = P.nv_eff;
    }
    P.vt[c][0] = a / bn;
    P.vt[c][1] = b > a ? (b + bn - 1) / bn : a / bn;
  }
}

// Stage 3: slash key ranges.  run_at(k) is the k-th run from the largest
// offsets down (keys ascending), k < nr; the diagonal j = i comes last.
// Ranges closer than bn keys are merged.  The output index never passes the
// input index, so the runs may be staged in P.iv itself (run_at(k) reading
// P.iv[k]).
template <class RunAt>
DCA_HD void sparse_plan_slash(SparsePlan& P, RunAt run_at, int nr, int64_t i0_, int64_t i_last_,
                              int bn) {
  const int i0 = static_cast<int>(i0_), i_last = static_cast<int>(i_last_);
  int n_iv = 0, cx = 0, cy = 0;
  bool open = false;  // a range [cx, cy) is being merged
  for (int k = 0; k <= nr; ++k) {
    int oa = 0, ob = 1;
    if (k < nr) {
      const int2 r = run_at(k);
      oa = r.x;
      ob = r.y;
    }
    if (oa > i_last) continue;
    const int ta = i0 - (ob - 1) > 0 ? i0 - (ob - 1) : 0;
    const int tb = i_last - oa + 1;
    if (open && ta < cy + bn) {
      if (tb > cy) cy = tb;
      if (ta < cx) cx = ta;
    } else {
      if (open) {  // index <= k: run k is already read
        P.iv[n_iv].x = cx;
        P.iv[n_iv].y = cy;
        ++n_iv;
      }
      cx = ta;
      cy = tb;
      open = true;
    }
  }
  if (open) {
    P.iv[n_iv].x = cx;
    P.iv[n_iv].y = cy;
    ++n_iv;
  }
  P.n_iv = n_iv;
}

// Stage 4: the item count, range by range (the iterator's windows: per
// class, the vertical tiles, then each slash range clipped to the class's
// key range, ceil(length / 128) windows).
DCA_HD int sparse_range_items(int2 r, const int kr[3][2]) {
  int n = 0;
  for (int c = 0; c < 3; ++c) {
    const int a = r.x > kr[c][0] ? r.x : kr[c][0];
    const int b = r.y < kr[c][1] ? r.y : kr[c][1];
    if (a < b) n += (b - a + 127) / 128;
  }
  return n;
}
DCA_HD int sparse_vertical_items(const SparsePlan& P) {
  return (P.vt[0][1] - P.vt[0][0]) + (P.vt[1][1] - P.vt[1][0]) + (P.vt[2][1] - P.vt[2][0]);
}
DCA_HD void sparse_plan_count(SparsePlan& P) {
  int n = sparse_vertical_items(P);
  for (int r = 0; r < P.n_iv; ++r) n += sparse_range_items(P.iv[r], P.kr);
  P.n_items = n;
}

// Builds the plan of the query rows [i0, i_last] for a head with nvh sorted
// vertical keys vk and nr slash runs (offset ranges [x, y), ascending, at most
// SPARSE_IV_MAX - 1), one lookup at a time.  bn = 128.
DCA_HD void sparse_plan_build(SparsePlan& P, const int32_t* vk, int nvh, const int2* runs, int nr,
                              int64_t i0, int64_t i_last, int64_t s, int64_t w, int reading,
                              int bn) {
  int64_t klo[3], khi[3], key[SPARSE_NKEYS];
  sparse_plan_ranges(P, i0, i_last, s, w, reading, klo, khi);
  sparse_plan_keys(i_last, klo, khi, key);
  int pos[SPARSE_NKEYS];
  for (int e = 0; e < SPARSE_NKEYS; ++e) {
    int lo = 0, hi = nvh;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (vk[mid] < key[e]) lo = mid + 1; else hi = mid;
    }
    pos[e] = lo;
  }
  sparse_plan_vertical(P, klo, khi, pos, bn);
  sparse_plan_slash(P, [&](int k) { return runs[nr - 1 - k]; }, nr, i0, i_last, bn);
  sparse_plan_count(P);
}

}  // namespace dca

// dca_select_rows.cuh -- the per-key row masks of the key selection (its
// score passes and the host introspection entry dca_class_rows).
#pragma once
#include <stdint.h>

#include "dca_plan.cuh"

namespace dca {

// Rows [*ra, *rb) of a block of estimate rows (positions i_first + r,
// r < n_last) that pair with key j: causal (j <= i), j < Lk, and either of
// pair class `cls` (cls >= 0) or, with cls < 0, a key of chunk `chunk`.
// For a fixed key the class is non-decreasing in i -- INTRA while
// i < t1 = s (n_j + 1), INTER from t2 on, SUCC between, where t2 = s (n_j + 2),
// or under reading B the smaller of that and max(t1, j + w) -- so the rows of
// one class are one contiguous range.
// Needs 0 <= j < 2^32 and 1 <= s < 2^32 (the one division is 32-bit).
DCA_HD void class_row_range(int64_t j, int64_t i_first, int n_last, int64_t Lk, int64_t s,
                            int64_t w, int reading, int cls, int64_t chunk, int* ra, int* rb) {
  int64_t lo = j - i_first, hi = n_last;
  const int64_t nj = static_cast<int64_t>(static_cast<uint32_t>(j) / static_cast<uint32_t>(s));
  if (j >= Lk) hi = 0;
  if (cls < 0) {
    if (nj != chunk) hi = 0;
  } else {
    const int64_t t1 = s * (nj + 1);
    int64_t t2 = s * (nj + 2);
    if (reading == READING_B) {
      const int64_t b = t1 > j + w ? t1 : j + w;
      if (b < t2) t2 = b;
    }
    if (cls == CLS_INTRA) {
      if (t1 - i_first < hi) hi = t1 - i_first;
    } else if (cls == CLS_SUCC) {
      if (t1 - i_first > lo) lo = t1 - i_first;
      if (t2 - i_first < hi) hi = t2 - i_first;
    } else {
      if (t2 - i_first > lo) lo = t2 - i_first;
    }
  }
  if (lo < 0) lo = 0;
  if (lo > n_last) lo = n_last;
  if (hi < lo) hi = lo;
  *ra = static_cast<int>(lo);
  *rb = static_cast<int>(hi);
}

}  // namespace dca

// fill_map.cuh -- the row -> sequence search shared by pkv_fill's kernel and
// its race check.
#pragma once

#include <stdint.h>

namespace pkv {

// The last b in [0, batch) with cu[b] <= t, for cu non-decreasing (global or
// shared memory).
__device__ __forceinline__ int32_t fill_seq_of(const int32_t* cu, int32_t batch, int32_t t) {
  int32_t lo = 0, hi = batch;   // cu[lo] <= t < cu[hi] when cu is non-decreasing
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

}  // namespace pkv

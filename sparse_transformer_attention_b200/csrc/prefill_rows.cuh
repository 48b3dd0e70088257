// Shared prologue of the prefill score passes (internal).
#pragma once

#include "common.cuh"
#include "prefill.cuh"

namespace ca {

constexpr int kPrefillTileRows = 128;  // query rows per CTA of a score pass

// Window and last candidate position of each row of the tile (query rows
// r0 .. r0+127 of head h, at positions p0 + r, written to s_hi[0..127]);
// *s_maxhi is the largest last-candidate position over the tile's rows (-1
// if none).  Every thread of the CTA must call it.
__device__ __forceinline__ void tile_rows(const PrefillArgs& a, int b, int h,
                                          int r0, int* s_hi, int* s_maxhi) {
  const int tid = threadIdx.x;
  if (tid == 0) *s_maxhi = -1;
  __syncthreads();
  if (tid < kPrefillTileRows) {
    const int r = r0 + tid;
    int hi = -1;
    if (r < a.nq) {
      const int w = row_window(a.W_i, (int64_t)b * a.nq + r, a.W_h, h, a.W,
                               a.L, a.status, true);
      hi = a.p0 + r - w;
    }
    s_hi[tid] = hi;
    atomicMax(s_maxhi, hi);
  }
  __syncthreads();
}

}  // namespace ca

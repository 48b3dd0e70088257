// Per-row streaming Top-k for the prefill score pass.
//
// One thread owns one query row (the TMEM lane layout of a 128-row MMA
// accumulator, and the thread-per-row FFMA path use the same layout).  The
// row's current best k keys live in a shared-memory min-heap whose root is
// the admission threshold; the heap starts full of key 0, which sorts below
// every real key.  Scores arrive 32 columns at a time in registers:
//   1. a max over the chunk decides whether any column can beat the
//      threshold (most chunks stop here once the heap is warm);
//   2. otherwise the columns at or above the threshold are appended to a
//      small per-row staging list (predicated stores, no divergence);
//   3. when any row of the warp could overflow its staging list, every lane
//      drains its own list into its heap (replace-root and sift down for each
//      staged key that still beats the root).
// Shared-memory layouts interleave the 128 rows (slot * 128 + row), so the
// 32 lanes of a warp touching the same slot hit distinct banks.
// Order: larger key wins (higher fp32 score, then lower index), as in
// §2.2.3 of the Condensate Theorem page with the tie rule of the library.
#pragma once

#include "common.cuh"

namespace ca {

constexpr int kTileRows = 128;

struct RowTopk {
  uint64_t* heap;   // [k][128]
  uint2* stage;     // [S][128]: {fp32 score bits, key position}
  int r;            // row within the tile (0..127)
  int k;
  int S;            // staging capacity per row
  int scnt;
  uint64_t root;
  float thr;        // score of the root, -inf while the heap has room

  __device__ __forceinline__ void init(uint64_t* heap_, uint2* stage_, int r_,
                                       int k_, int S_) {
    heap = heap_;
    stage = stage_;
    r = r_;
    k = k_;
    S = S_;
    scnt = 0;
    root = 0ull;
    thr = -INFINITY;
    for (int e = 0; e < k; ++e) heap[e * kTileRows + r] = 0ull;
  }

  __device__ __forceinline__ uint64_t& H(int e) { return heap[e * kTileRows + r]; }

  // Precondition: key > root.  Replace the root and restore the heap.
  __device__ __forceinline__ void replace_root(uint64_t key) {
    int p = 0;
#pragma unroll 1
    while (true) {
      int c = 2 * p + 1;
      if (c >= k) break;
      uint64_t cv = H(c);
      if (c + 1 < k) {
        uint64_t c2 = H(c + 1);
        if (c2 < cv) {
          cv = c2;
          c = c + 1;
        }
      }
      if (cv >= key) break;
      H(p) = cv;
      p = c;
    }
    H(p) = key;
    root = H(0);
  }

  __device__ __forceinline__ void drain() {
    int rounds = __reduce_max_sync(0xFFFFFFFFu, (unsigned)scnt);
#pragma unroll 1
    for (int t = 0; t < rounds; ++t) {
      if (t < scnt) {
        uint2 e = stage[t * kTileRows + r];
        uint64_t key = make_key(__uint_as_float(e.x), e.y);
        if (key > root) replace_root(key);
      }
    }
    scnt = 0;
    thr = root ? key_score(root) : -INFINITY;
  }

  // Offer 32 consecutive scores (fp32 bits) for key positions j0..j0+31.
  // When MASKED, only positions in [jlo, jhi] are candidates.
  template <bool MASKED>
  __device__ __forceinline__ void offer(const uint32_t (&raw)[32], int j0,
                                        int jlo, int jhi) {
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float s = __uint_as_float(raw[c]);
      if (!MASKED || (j0 + c >= jlo && j0 + c <= jhi)) mx = fmaxf(mx, s);
    }
    const bool hit = (mx >= thr) && (mx != -INFINITY);
    if (!__any_sync(0xFFFFFFFFu, hit)) return;
    if (__any_sync(0xFFFFFFFFu, scnt + 32 > S)) drain();
    uint2* dst = stage + scnt * kTileRows + r;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float s = __uint_as_float(raw[c]);
      bool p = hit && (s >= thr);
      if (MASKED) p = p && (j0 + c >= jlo) && (j0 + c <= jhi);
      if (p) {
        *dst = make_uint2(raw[c], (uint32_t)(j0 + c));
        dst += kTileRows;
        ++scnt;
      }
    }
  }

  // Write the row's k keys (heap order, 0 = empty slot).
  __device__ __forceinline__ void store(uint64_t* out) {
    for (int e = 0; e < k; ++e) out[e] = H(e);
  }
};

}  // namespace ca

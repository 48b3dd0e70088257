// Register-resident sorts by one warp (no shared-memory barriers).
#pragma once

#include <stdint.h>

namespace ca {

// Ascending bitonic sort of 32*NPL values held by one warp (element
// e = t*32 + lane in v[t]); pairs closer than 32 are exchanged by shuffles.
template <int NPL>
__device__ __forceinline__ void warp_bitonic(uint32_t (&v)[NPL], int lane) {
#pragma unroll
  for (int size = 2; size <= 32 * NPL; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      uint32_t nv[NPL];
#pragma unroll
      for (int t = 0; t < NPL; ++t) {
        const int e = t * 32 + lane;
        const uint32_t other = (stride >= 32)
            ? v[t ^ (stride >> 5)]
            : __shfl_xor_sync(0xFFFFFFFFu, v[t], stride);
        const bool up = (e & size) == 0, lower = (e & stride) == 0;
        nv[t] = (lower == up) ? min(v[t], other) : max(v[t], other);
      }
#pragma unroll
      for (int t = 0; t < NPL; ++t) v[t] = nv[t];
    }
  }
}

template <int NPL>
__device__ __forceinline__ void warp_sort_n(uint32_t* a, int n, int lane) {
  uint32_t v[NPL];
#pragma unroll
  for (int t = 0; t < NPL; ++t) {
    const int e = t * 32 + lane;
    v[t] = e < n ? a[e] : 0xFFFFFFFFu;
  }
  warp_bitonic<NPL>(v, lane);
#pragma unroll
  for (int t = 0; t < NPL; ++t) a[t * 32 + lane] = v[t];
}

// Sort a[0..n) ascending with one warp; a has room for kpow2 >= n entries
// (kpow2 a power of two <= 1024); entries n..kpow2 become 0xFFFFFFFF.
__device__ __forceinline__ void warp_sort_prefix(uint32_t* a, int n, int kpow2,
                                                 int lane) {
  if (kpow2 <= 32) warp_sort_n<1>(a, n, lane);
  else if (kpow2 <= 64) warp_sort_n<2>(a, n, lane);
  else if (kpow2 <= 128) warp_sort_n<4>(a, n, lane);
  else if (kpow2 <= 256) warp_sort_n<8>(a, n, lane);
  else if (kpow2 <= 512) warp_sort_n<16>(a, n, lane);
  else warp_sort_n<32>(a, n, lane);
}

}  // namespace ca

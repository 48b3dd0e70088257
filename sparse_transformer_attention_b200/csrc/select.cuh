// CTA-wide exact selection on 64-bit keys (see make_key in common.cuh).
//
// Radix select, most significant byte first: each pass histograms the keys
// that still match the chosen prefix and picks the byte whose bucket holds
// the kk-th largest key.  A list stops early once its chosen bucket holds
// exactly the keys still needed: every key of the bucket is then selected,
// and the bucket's lower bound (prefix followed by zero bytes) separates the
// selected keys from the others.  Several independent lists share passes and
// barriers.
#pragma once

#include "common.cuh"

namespace ca {

// Barrier policies: the whole CTA, or a named barrier over the N threads of
// one warp group (the other warps of the CTA keep running).
struct CtaBarrier {
  __device__ static __forceinline__ void sync() { __syncthreads(); }
};
template <int ID, int N>
struct GroupBarrier {
  __device__ static __forceinline__ void sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory");
  }
};

template <int NL>
struct SelectState {
  uint64_t prefix[NL];
  uint32_t need[NL];
  uint32_t done[NL];
  uint32_t hist[NL * 256];
};

// For each list l < NL (keys[l*stride .. l*stride + n[l])), compute T[l] such
// that exactly kk[l] keys are >= T[l] (keys unique, kk[l] >= 1).  A list
// with n[l] <= kk[l] gets T[l] = 0 (keep all).  n, kk and T live in shared
// memory.  Every one of the NT threads synchronised by Bar must call this
// with its index tid in [0, NT); on return all of them may read T.
template <int NT, int NL, class Bar = CtaBarrier>
__device__ void cta_select_thresholds(const uint64_t* keys, int stride,
                                      const int* n, const int* kk, uint64_t* T,
                                      SelectState<NL>* st, int tid) {
  static_assert(NL * 32 <= NT, "one warp per list for the bucket scan");
  const int warp = tid >> 5, lane = tid & 31;
  if (tid < NL) {
    st->prefix[tid] = 0;
    st->need[tid] = (uint32_t)kk[tid];
    st->done[tid] = n[tid] <= kk[tid];
  }
  Bar::sync();
#pragma unroll 1
  for (int shift = 56; shift >= 0; shift -= 8) {
    bool all_done = true;
#pragma unroll
    for (int l = 0; l < NL; ++l) all_done = all_done && st->done[l];
    if (all_done) break;  // uniform: every thread reads the same state
    const uint64_t hmask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
    for (int b = tid; b < NL * 256; b += NT) st->hist[b] = 0;
    Bar::sync();
#pragma unroll
    for (int l = 0; l < NL; ++l) {
      if (st->done[l]) continue;
      const uint64_t* kl = keys + (size_t)l * stride;
      const uint64_t pf = st->prefix[l];
      const int nl = n[l];
      for (int e = tid; e < nl; e += NT) {
        const uint64_t key = kl[e];
        if ((key & hmask) == pf)
          atomicAdd(&st->hist[l * 256 + ((uint32_t)(key >> shift) & 255u)], 1u);
      }
    }
    Bar::sync();
    if (warp < NL && !st->done[warp]) {
      const uint32_t* h = st->hist + warp * 256;
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        c[t] = h[255 - 8 * lane - t];
        sum += c[t];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t excl = incl - sum;
      const uint32_t nd = st->need[warp];
      __syncwarp();
      if (excl < nd && nd <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (acc + c[t] >= nd) {
            const uint32_t digit = 255u - 8u * lane - t;
            st->prefix[warp] |= (uint64_t)digit << shift;
            st->need[warp] = nd - acc;
            if (c[t] == nd - acc) st->done[warp] = 1u;
            break;
          }
          acc += c[t];
        }
      }
    }
    Bar::sync();
  }
  if (tid < NL) T[tid] = (n[tid] <= kk[tid]) ? 0ull : st->prefix[tid];
  Bar::sync();
}

// One warp cuts the list lst[0..n) of unique keys down to its best kk keys
// (n > kk >= 1), in place and in no particular order, and returns the
// threshold T with exactly kk keys >= T.  Radix select from the most
// significant byte, stopping as soon as the chosen byte's bucket holds
// exactly the keys still needed (its lower bound then separates the sets).
__device__ __forceinline__ uint64_t warp_cut(uint64_t* lst, int n, int kk, uint32_t* hist,
                             int lane) {
  uint64_t prefix = 0ull;
  uint32_t need = (uint32_t)kk;
#pragma unroll 1
  for (int shift = 56; shift >= 0; shift -= 8) {
    const uint64_t hmask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
#pragma unroll
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int e = lane; e < n; e += 32) {
      const uint64_t key = lst[e];
      if ((key & hmask) == prefix)
        atomicAdd(&hist[(uint32_t)(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      c[t] = hist[255 - 8 * lane - t];
      sum += c[t];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += v;
    }
    const uint32_t excl = incl - sum;
    const bool mine = excl < need && need <= incl;
    uint32_t digit = 0, nd = 0, bucket = 0;
    if (mine) {
      uint32_t acc = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (acc + c[t] >= need) {
          digit = 255u - 8u * lane - t;
          nd = need - acc;
          bucket = c[t];
          break;
        }
        acc += c[t];
      }
    }
    const int src = __ffs(__ballot_sync(0xFFFFFFFFu, mine)) - 1;
    digit = __shfl_sync(0xFFFFFFFFu, digit, src);
    nd = __shfl_sync(0xFFFFFFFFu, nd, src);
    bucket = __shfl_sync(0xFFFFFFFFu, bucket, src);
    prefix |= (uint64_t)digit << shift;
    need = nd;
    __syncwarp();  // the histogram is cleared again next pass
    if (bucket == nd) break;
  }
  // keep the keys >= prefix, packed to the front in reading order; a slot
  // is only written after the whole group of 32 that covers it was read
  int wr = 0;
  for (int base = 0; base < n; base += 32) {
    const int e = base + lane;
    const uint64_t key = e < n ? lst[e] : 0ull;
    const bool keep = e < n && key >= prefix;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) lst[wr + __popc(bal & ((1u << lane) - 1u))] = key;
    wr += __popc(bal);
    __syncwarp();
  }
  return prefix;
}

}  // namespace ca

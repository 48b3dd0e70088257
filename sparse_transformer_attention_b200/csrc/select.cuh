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

// ---------------------------------------------------------------- one warp,
// keys in registers (element e = t * 32 + lane in v[t]; key 0 marks an
// absent element and is never counted or kept; the nonzero keys are unique)

// Largest of the 64-bit values held by a warp (every lane gets it).
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  return v;
}

// Load n keys from src (shared or global memory) into registers, 0 past n.
template <int NPL>
__device__ __forceinline__ void warp_load_keys(const uint64_t* src, int n,
                                               uint64_t (&v)[NPL], int lane) {
#pragma unroll
  for (int t = 0; t < NPL; ++t) {
    const int e = t * 32 + lane;
    v[t] = e < n ? src[e] : 0ull;
  }
}

// The kk-th largest nonzero key (kk >= 1), or 1 when at most kk keys are
// nonzero: in both cases exactly min(kk, nonzero) keys are >= the result.
// Bisection on the high words, from the common prefix of the smallest and
// the largest, then on the low words of the keys whose high word is the
// chosen one; each count is one warp reduction, and the search stops at the
// first probe that leaves exactly kk keys above it.
template <int NPL>
__device__ __forceinline__ uint64_t warp_kth(const uint64_t (&v)[NPL], int kk) {
  constexpr unsigned kAll = 0xFFFFFFFFu;
  uint32_t hw[NPL];
  uint32_t nz = 0u, mx = 0u, mn = 0xFFFFFFFFu;
#pragma unroll
  for (int t = 0; t < NPL; ++t) {
    hw[t] = (uint32_t)(v[t] >> 32);
    const bool real = v[t] != 0ull;
    nz += real;
    mx = real ? max(mx, hw[t]) : mx;
    mn = real ? min(mn, hw[t]) : mn;
  }
  nz = __reduce_add_sync(kAll, nz);
  if (nz <= (uint32_t)kk) return 1ull;
  mx = __reduce_max_sync(kAll, mx);
  mn = __reduce_min_sync(kAll, mn);
  // Real scores have ord codes of at least 0x007FFFFF in the high word, so
  // every probe below (>= 1) leaves the absent keys out.
  const uint32_t diff = mn ^ mx;
  const int nb = diff ? 32 - __clz(diff) : 0;
  uint32_t th = nb == 32 ? 0u : (mn >> nb) << nb;
#pragma unroll 1
  for (int bit = nb - 1; bit >= 0; --bit) {
    const uint32_t c = th | (1u << bit);
    uint32_t m = 0u;
#pragma unroll
    for (int t = 0; t < NPL; ++t) m += hw[t] >= c;
    m = __reduce_add_sync(kAll, m);
    if (m >= (uint32_t)kk) {
      th = c;
      if (m == (uint32_t)kk) return (uint64_t)th << 32;
    }
  }
  // th is the kk-th largest high word; fewer than kk keys lie above it
  uint32_t above = 0u;
#pragma unroll
  for (int t = 0; t < NPL; ++t) above += hw[t] > th;
  above = __reduce_add_sync(kAll, above);
  const uint32_t need = (uint32_t)kk - above;
  uint32_t tl = 0u;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t c = tl | (1u << bit);
    uint32_t m = 0u;
#pragma unroll
    for (int t = 0; t < NPL; ++t)
      m += hw[t] == th && (uint32_t)v[t] >= c;
    m = __reduce_add_sync(kAll, m);
    if (m >= need) {
      tl = c;
      if (m == need) break;
    }
  }
  return ((uint64_t)th << 32) | tl;
}

// Write the keys >= T (T >= 1) to out[0..), in element order; returns how
// many.  out may alias the source of v: every lane has its keys in
// registers before the first ballot.
template <int NPL>
__device__ __forceinline__ int warp_keep(const uint64_t (&v)[NPL], uint64_t T,
                                         uint64_t* out, int lane) {
  int w = 0;
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int t = 0; t < NPL; ++t) {
    const bool keep = v[t] >= T;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) out[w + __popc(bal & below)] = v[t];
    w += __popc(bal);
  }
  return w;
}

// One warp cuts lst[0..n) (n <= 32 * NPL, kk >= 1, nonzero keys unique)
// to its best kk keys in place, dropping the absent (0) keys; returns the
// kk-th largest key (or 1 when at most kk keys are nonzero, which are then
// all kept) and sets *kept to the number of keys left.
template <int NPL>
__device__ __forceinline__ uint64_t warp_cut_regs(uint64_t* lst, int n, int kk,
                                                  int lane, int* kept) {
  uint64_t v[NPL];
  warp_load_keys<NPL>(lst, n, v, lane);
  const uint64_t T = warp_kth<NPL>(v, kk);
  __syncwarp();
  *kept = warp_keep<NPL>(v, T, lst, lane);
  __syncwarp();
  return T;
}

}  // namespace ca

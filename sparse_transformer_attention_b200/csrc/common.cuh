// Shared device helpers for the Condensate attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ca {

// Bits of the device status word (first 4 bytes of the workspace).
constexpr uint32_t kErrWindow = 1u;    // a window below 1 or k_h outside [0, k]
constexpr uint32_t kErrTimeout = 2u;   // a bounded wait ran out
constexpr uint32_t kErrCmax = 4u;      // |C_i| larger than C_max
constexpr uint32_t kErrInternal = 8u;  // internal capacity check failed
constexpr uint32_t kErrBounds = 16u;   // (debug builds) an index check failed

constexpr int kStatusBytes = 256;      // status area at the workspace start

// Limits of the bounded waits.  A pipeline wait (a consumer waiting for its
// producer) gives up after kPipelineWaitNs and aborts the CTA; a drain wait
// (a thread waiting for copies or MMAs it issued itself, before exit) is
// always given kDrainWaitNs.
constexpr uint64_t kPipelineWaitNs = 2000000000ull;  // 2 s
constexpr uint64_t kDrainWaitNs = 2000000000ull;     // 2 s

__device__ __forceinline__ void raise_flag(uint32_t* status, uint32_t bit) {
  atomicOr(status, bit);
}

// Index checks of the debug build.  Built with CA_DEBUG, the kernels check
// the indexes that the release build keeps in range by construction (the
// cursors of the prefill selector's shared-memory segments, the slots of the
// decode score pass's per-head lists, the merge's survivor slots, the rows
// listed for the exact fallback): a failed check raises kErrBounds and the
// access is skipped, so a bug shows as a status code instead of a memory
// fault.  The release build compiles every check to `true`.
#ifdef CA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t* status) {
  if constexpr (kDebugChecks) {
    if (!ok) raise_flag(status, kErrBounds);
    return ok;
  } else {
    return true;
  }
}

// Order-preserving map of an fp32 score to uint32: a > b (as reals) iff
// ord(a) > ord(b).  -0 is folded onto +0 first so equal reals map equally.
__device__ __forceinline__ uint32_t ord_f32(float s) {
  uint32_t b = __float_as_uint(__fadd_rn(s, 0.0f));
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float unord_f32(uint32_t o) {
  uint32_t b = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  return __uint_as_float(b);
}

// Selection key: larger key = higher score, and on equal scores the lower
// index (the tie rule of the Top-k).  Key 0 never encodes a real candidate
// (every finite score maps to ord >= 0x00800000), so it marks empty slots.
__device__ __forceinline__ uint64_t make_key(float s, uint32_t j) {
  return ((uint64_t)ord_f32(s) << 32) | (uint64_t)(0xFFFFFFFFu - j);
}
__device__ __forceinline__ uint32_t key_index(uint64_t key) {
  return 0xFFFFFFFFu - (uint32_t)key;
}
__device__ __forceinline__ float key_score(uint64_t key) {
  return unord_f32((uint32_t)(key >> 32));
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) {
  return __uint_as_float(w << 16);
}
__device__ __forceinline__ float bf16hi(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// Element type traits: T in {float, __nv_bfloat16}.
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPer16B = 4;
  // unpack 16 bytes into 4 floats
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static __forceinline__ float load1(const float* p) { return *p; }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kPer16B = 8;
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
  }
  __device__ static __forceinline__ float load1(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
};

// Load N consecutive elements (N in {2, 4}, naturally aligned) as floats.
template <typename T, int N>
__device__ __forceinline__ void load_f32(const T* p, float* f);
template <>
__device__ __forceinline__ void load_f32<float, 2>(const float* p, float* f) {
  float2 v = *reinterpret_cast<const float2*>(p);
  f[0] = v.x; f[1] = v.y;
}
template <>
__device__ __forceinline__ void load_f32<float, 4>(const float* p, float* f) {
  float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load_f32<__nv_bfloat16, 2>(const __nv_bfloat16* p, float* f) {
  uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  f[0] = bf16lo(w); f[1] = bf16hi(w);
}
template <>
__device__ __forceinline__ void load_f32<__nv_bfloat16, 4>(const __nv_bfloat16* p, float* f) {
  uint2 w = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
}

template <typename T> __device__ __forceinline__ void store_out(T* p, float v);
template <> __device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// Window of a query row: W_i[wi] when given, else W_h[h] when given, else
// W.  A window below 1 raises kErrWindow (when `report`) and is read as 1;
// a window beyond `limit` (the cache length) covers every causal position
// and is read as `limit`.
__device__ __forceinline__ int row_window(const int32_t* W_i, int64_t wi,
                                          const int32_t* W_h, int h, int W,
                                          int limit, uint32_t* status,
                                          bool report) {
  int w = W_i ? W_i[wi] : (W_h ? W_h[h] : W);
  if (w < 1) {
    if (report) raise_flag(status, kErrWindow);
    w = 1;
  }
  return w > limit ? limit : w;
}

// Top-k size of q-head h: k_h[h] when given (clamped to [0, k], a value
// outside raising kErrWindow when `report`), else k.
__device__ __forceinline__ int head_k(const int32_t* k_h, int h, int k,
                                      uint32_t* status, bool report) {
  if (!k_h) return k;
  int kh = k_h[h];
  if (kh < 0 || kh > k) {
    if (report) raise_flag(status, kErrWindow);
    kh = kh < 0 ? 0 : k;
  }
  return kh;
}

// Online log-sum-exp state in log2 units: the sum of 2^(x - m) over the
// values x folded in, with m their maximum (m = -inf, l = 0 when empty).
struct Lse2 {
  float m = -INFINITY, l = 0.f;
  __device__ __forceinline__ void add(float x) {
    if (x > m) {
      l = l * exp2f(m - x) + 1.f;
      m = x;
    } else {
      l += exp2f(x - m);
    }
  }
  __device__ __forceinline__ void merge(float m2, float l2) {
    if (l2 == 0.f) return;
    if (l == 0.f) {
      m = m2;
      l = l2;
      return;
    }
    const float mn = fmaxf(m, m2);
    l = l * exp2f(m - mn) + l2 * exp2f(m2 - mn);
    m = mn;
  }
};

// Mass report of one query row over the full causal softmax, from three
// log2-domain (max, sum) states of scaled scores: C_i (m_c, l_c), the
// window together with the anchor (m_wa, l_wa), and every candidate
// [1, i-W_i] (m_cand, l_cand; the Top-k members are among them), plus the
// anchor's own scaled score s0 (`anc`: the anchor lies outside the window).
// Writes anchor, window, Top-k and excluded mass and the natural-log
// log-sum-exp ("Condensate Theorem" page 1 §2.2.1, §2.2.2, §3.2.2).
__device__ __forceinline__ void mass_report(float* mass, float* lse,
                                            size_t row, float m_c, float l_c,
                                            float m_wa, float l_wa,
                                            float m_cand, float l_cand,
                                            float s0, bool anc) {
  const float F = l_cand > 0.f ? fmaxf(m_c, m_cand) : m_c;
  const float lC = l_c * exp2f(m_c - F);
  const float lwa = l_wa > 0.f ? l_wa * exp2f(m_wa - F) : 0.f;
  const float lcand = l_cand > 0.f ? l_cand * exp2f(m_cand - F) : 0.f;
  const float p0 = exp2f(s0 - F);
  const float all = lwa + lcand;
  const float ltop = fmaxf(lC - lwa, 0.f);
  if (mass) {
    mass[row * 4 + 0] = p0 / all;
    mass[row * 4 + 1] = fmaxf(lwa - (anc ? p0 : 0.f), 0.f) / all;
    mass[row * 4 + 2] = ltop / all;
    mass[row * 4 + 3] = fmaxf(lcand - ltop, 0.f) / all;
  }
  if (lse) lse[row] = (F + log2f(all)) * 0.6931471805599453f;
}

}  // namespace ca

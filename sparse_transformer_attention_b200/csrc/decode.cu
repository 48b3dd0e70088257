// Decode path: one query per (batch, q-head) at position L-1 against an
// L-long KV cache.  "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质",
// §2.1 Definition 1 (C_i for the last row), §2.2.3 (Dynamic Top-k), §2.4
// Corollary 3 (per-query window), §5.2.2 (select, then attend on the subset).
//
// Launch 1, decode_score_topk: grid (chunks, Hkv, B).  Each CTA streams one
// chunk of K rows of one kv-head once, with 16-byte coalesced loads (8 lanes
// per 256-byte row), scores all G = Hq/Hkv q-heads of the group from the same
// bytes, and keeps a per-head candidate buffer in shared memory behind a
// threshold that only rises.  Buffers are cut back to exactly the best k
// keys by a CTA radix select; the chunk's best k keys per q-head go to the
// workspace.  The union of the chunks' best-k lists contains the global
// Top-k, since every global Top-k member is among the best k of its chunk.
//
// Launch 2, decode_merge_attend: grid (Hq, B).  Each CTA merges its q-head's
// chunk lists into the exact Top-k, writes C_i in ascending order, then runs
// an fp32 online softmax over the gathered K/V rows of C_i.
#include "common.cuh"
#include "decode.cuh"
#include "profile.cuh"
#include "select.cuh"

namespace ca {

namespace {

constexpr int kThreads = 256;
constexpr int kSub = 1024;     // keys per sub-chunk between buffer checks
constexpr int kSlack = 512;    // insert room kept after a cut
constexpr int kMergeThreads = 512;

// Transposing butterfly over the 8 lanes of one key.  On entry v[h] is this
// lane's partial dot product for q-head h of the group; every step halves
// the list, sending one half to the partner lane and adding the other half's
// copy received from it.  On exit v[0] is the full dot product for q-head
// reduce_head(l8); lanes that share a head hold the same value.
template <int NV>
__device__ __forceinline__ void halve(float* v, int lane, int dist) {
  const bool b = (lane & dist) != 0;
#pragma unroll
  for (int p = 0; p < NV / 2; ++p) {
    const float send = b ? v[p] : v[p + NV / 2];
    const float keep = b ? v[p + NV / 2] : v[p];
    v[p] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, dist);
  }
}

template <int G>
__device__ __forceinline__ float group_reduce(float (&v)[G], int lane) {
  if constexpr (G >= 2) halve<G>(v, lane, 4);
  else v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 4);
  if constexpr (G >= 4) halve<G / 2>(v, lane, 2);
  else v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 2);
  if constexpr (G >= 8) halve<G / 4>(v, lane, 1);
  else v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 1);
  return v[0];
}

// q-head (within the group) held by lane l8 after group_reduce, and whether
// this lane is the one that reports it.
template <int G>
__device__ __forceinline__ int reduce_head(int l8) {
  if constexpr (G == 8) return l8;
  else if constexpr (G == 4) return ((l8 >> 2) & 1) * 2 + ((l8 >> 1) & 1);
  else if constexpr (G == 2) return (l8 >> 2) & 1;
  else return 0;
}
template <int G>
__device__ __forceinline__ bool reduce_owner(int l8) {
  if constexpr (G == 8) return true;
  else if constexpr (G == 4) return (l8 & 1) == 0;
  else if constexpr (G == 2) return (l8 & 3) == 0;
  else return l8 == 0;
}

template <int G>
struct TopkShared {
  int cnt[G];
  int kk[G];
  uint64_t thr[G];
  uint64_t T[G];
  int out_pos;
  SelectState<G> sel;
};

// Cut every list whose count exceeds `limit` down to its best k keys.
template <int G>
__device__ void cut_lists(uint64_t* buf, int cap, uint64_t* tmp, int k,
                          int limit, TopkShared<G>* sh) {
  __shared__ int s_n[G];
  bool any = false;
#pragma unroll
  for (int h = 0; h < G; ++h) any = any || (sh->cnt[h] > limit);
  if (!any) return;  // uniform decision
  if (threadIdx.x < G) {
    s_n[threadIdx.x] = sh->cnt[threadIdx.x] > limit ? sh->cnt[threadIdx.x] : 0;
    sh->kk[threadIdx.x] = k;
  }
  __syncthreads();
  cta_select_thresholds<kThreads, G>(buf, cap, s_n, sh->kk, sh->T, &sh->sel);
#pragma unroll 1
  for (int h = 0; h < G; ++h) {
    if (s_n[h] == 0) continue;
    const uint64_t T = sh->T[h];
    if (threadIdx.x == 0) sh->out_pos = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < s_n[h]; e += kThreads) {
      uint64_t key = buf[h * cap + e];
      if (key >= T) tmp[atomicAdd(&sh->out_pos, 1)] = key;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < k; e += kThreads) buf[h * cap + e] = tmp[e];
    if (threadIdx.x == 0) {
      sh->cnt[h] = k;
      sh->thr[h] = T;
    }
    __syncthreads();
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, G >= 8 ? 1 : 2)
decode_score_topk(DecodeArgs a) {
  constexpr int VEC = Elem<T>::kPer16B;
  constexpr int CPL = D / VEC / 8;  // 16-byte pieces per lane
  constexpr int DPL = CPL * VEC;    // head dims per lane
  constexpr int U = 4;              // keys in flight per lane
  static_assert(CPL >= 1, "row too short for 8 lanes");

  extern __shared__ __align__(16) unsigned char smem[];
  const int k = a.k;
  const int cap = k + kSub + kSlack;
  uint64_t* buf = reinterpret_cast<uint64_t*>(smem);  // [G][cap]
  uint64_t* tmp = buf + (size_t)G * cap;               // [k]
  TopkShared<G>* sh = reinterpret_cast<TopkShared<G>*>(tmp + k);

  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int l8 = lane & 7, ks = lane >> 3;
  const int64_t L = a.L;
  const int Wb = row_window(a.W_i, b, a.W, (int)L, a.status,
                            chunk == 0 && g == 0 && tid == 0);
  const int64_t hi = (L - 1) - Wb;  // last candidate position

  // this lane's slice of the G queries, as fp32
  float qf[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const T* qh = reinterpret_cast<const T*>(a.q) +
                  ((size_t)b * a.Hq + (size_t)g * G + h) * D;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      uint4 v = *reinterpret_cast<const uint4*>(qh + (l8 + 8 * c) * VEC);
      Elem<T>::unpack(v, &qf[h][c * VEC]);
    }
  }
  if (tid < G) {
    sh->cnt[tid] = 0;
    sh->thr[tid] = 0ull;
  }
  __syncthreads();

  const int myh = reduce_head<G>(l8);
  const bool owner = reduce_owner<G>(l8);
  const T* Kg = reinterpret_cast<const T*>(a.K) + ((size_t)b * a.Hkv + g) * L * D;
  const int64_t j0 = (int64_t)chunk * a.chunk_len;
  const int64_t c0 = j0 < 1 ? 1 : j0;
  int64_t c1 = j0 + a.chunk_len;
  if (c1 > hi + 1) c1 = hi + 1;
  bool first_cut = true;

#pragma unroll 1
  for (int64_t sub = c0; sub < c1; sub += kSub) {
    const uint64_t thr = sh->thr[myh];
    const int64_t wbase = sub + warp * (kSub / 8);
#pragma unroll 1
    for (int it = 0; it < kSub / 8; it += 4 * U) {
      uint4 raw[U][CPL];
      int64_t jj[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        jj[u] = wbase + it + u * 4 + ks;
        int64_t jr = jj[u] < c1 ? jj[u] : c0;  // stay inside the row range
        const T* row = Kg + (size_t)jr * D;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          raw[u][c] = ld_stream_v4(row + (l8 + 8 * c) * VEC);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          float f[VEC];
          Elem<T>::unpack(raw[u][c], f);
#pragma unroll
          for (int e = 0; e < VEC; ++e)
#pragma unroll
            for (int h = 0; h < G; ++h)
              part[h] = fmaf(qf[h][c * VEC + e], f[e], part[h]);
        }
        const float s = group_reduce<G>(part, lane);
        if (owner && jj[u] < c1) {
          const uint64_t key = make_key(s, (uint32_t)jj[u]);
          if (key > thr) {
            int pos = atomicAdd(&sh->cnt[myh], 1);
            buf[(size_t)myh * cap + pos] = key;
          }
        }
      }
    }
    __syncthreads();
    // The first cut sets a useful threshold; later cuts only keep room for
    // the next sub-chunk.
    cut_lists<G>(buf, cap, tmp, k, first_cut ? k : cap - kSub, sh);
    first_cut = false;
  }
  __syncthreads();
  cut_lists<G>(buf, cap, tmp, k, k, sh);

  // write this chunk's best keys per q-head; empty slots get key 0
#pragma unroll 1
  for (int h = 0; h < G; ++h) {
    uint64_t* out = a.cand +
        (((size_t)b * a.Hq + (size_t)g * G + h) * a.nchunks + chunk) * k;
    const int cnt = sh->cnt[h];
    for (int e = tid; e < k; e += kThreads)
      out[e] = e < cnt ? buf[(size_t)h * cap + e] : 0ull;
  }
}

// Bitonic sort (ascending) of n_pow2 uint32 values in shared memory.
__device__ void cta_sort_u32(uint32_t* v, int n_pow2) {
  for (int size = 2; size <= n_pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < n_pow2 / 2; t += blockDim.x) {
        int lo = 2 * t - (t & (stride - 1));
        int hi2 = lo + stride;
        bool up = ((lo & size) == 0);
        uint32_t x = v[lo], y = v[hi2];
        if ((x > y) == up) {
          v[lo] = y;
          v[hi2] = x;
        }
      }
    }
  }
  __syncthreads();
}

template <typename T, int D, typename TO>
__global__ void __launch_bounds__(kMergeThreads)
decode_merge_attend(DecodeArgs a) {
  constexpr int DL = D / 32;  // head dims per lane in the gather
  constexpr int NW = kMergeThreads / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  const int k = a.k;
  const int ncand = a.nchunks * k;
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem);   // [ncand]
  uint32_t* topj = reinterpret_cast<uint32_t*>(cand + ncand);  // [kpow2]
  SelectState<1>* st = reinterpret_cast<SelectState<1>*>(topj + a.kpow2);
  __shared__ int s_n, s_kk, s_m;
  __shared__ uint64_t s_T;
  __shared__ float s_m_w[NW], s_l_w[NW];
  __shared__ float s_o_w[NW][D];

  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = h / (a.Hq / a.Hkv);
  const int64_t L = a.L, i = L - 1;
  const int Wb = row_window(a.W_i, b, a.W, (int)L, a.status, false);
  const int64_t lo = (i - Wb + 1) > 0 ? (i - Wb + 1) : 0;
  const int64_t ncand_pos = (i - Wb) > 0 ? (i - Wb) : 0;  // |[1, i-W]|
  const int m = (int)(k < ncand_pos ? k : ncand_pos);

  // 1. gather the chunk lists (dropping empty slots)
  if (tid == 0) s_n = 0;
  __syncthreads();
  const uint64_t* src = a.cand + ((size_t)b * a.Hq + h) * ncand;
  for (int e = tid; e < ncand; e += kMergeThreads) {
    uint64_t key = src[e];
    if (key != 0ull) cand[atomicAdd(&s_n, 1)] = key;
  }
  __syncthreads();
  // 2. exact Top-m of the union
  if (tid == 0) s_kk = m > 0 ? m : 1;
  __syncthreads();
  cta_select_thresholds<kMergeThreads, 1>(cand, 0, &s_n, &s_kk, &s_T, st);
  if (tid == 0) s_m = 0;
  for (int e = tid; e < a.kpow2; e += kMergeThreads) topj[e] = 0xFFFFFFFFu;
  __syncthreads();
  if (m > 0) {
    for (int e = tid; e < s_n; e += kMergeThreads) {
      uint64_t key = cand[e];
      if (key >= s_T) {
        const uint32_t j = key_index(key);
        const int p = atomicAdd(&s_m, 1);
        if (p < a.kpow2 && j >= 1 && (int64_t)j <= i - Wb) topj[p] = j;
        else raise_flag(a.status, kErrInternal);
      }
    }
  }
  __syncthreads();
  if (m > 0 && s_m != m && tid == 0) raise_flag(a.status, kErrInternal);
  // an inconsistent candidate list must never steer the gather out of range
  for (int e = tid; e < a.kpow2; e += kMergeThreads)
    if (e >= m || topj[e] == 0xFFFFFFFFu) topj[e] = e < m ? 0u : 0xFFFFFFFFu;
  cta_sort_u32(topj, a.kpow2);

  // 3. C_i = {0} U sorted Top-k U [lo, i], ascending
  const int anc = lo > 0 ? 1 : 0;
  const int64_t count = anc + m + (i - lo + 1);
  int32_t* idx_row = a.idx + ((size_t)b * a.Hq + h) * a.C_max;
  if (count > a.C_max && tid == 0) raise_flag(a.status, kErrCmax);
  const int64_t wcount = count < a.C_max ? count : a.C_max;
  for (int64_t r = tid; r < a.C_max; r += kMergeThreads) {
    int32_t v;
    if (r >= wcount) v = -1;
    else if (r < anc) v = 0;
    else if (r < anc + m) v = (int32_t)topj[r - anc];
    else v = (int32_t)(lo + (r - anc - m));
    idx_row[r] = v;
  }
  if (tid == 0) a.idx_count[(size_t)b * a.Hq + h] = (int32_t)count;

  // 4. fp32 online softmax over C_i; warps take entries r = warp + NW*t,
  //    lanes split the head dimension.
  const T* qh = reinterpret_cast<const T*>(a.q) + ((size_t)b * a.Hq + h) * D;
  float qv[DL];
  load_f32<T, DL>(qh + lane * DL, qv);
  const T* Kg = reinterpret_cast<const T*>(a.K) + ((size_t)b * a.Hkv + g) * L * D;
  const T* Vg = reinterpret_cast<const T*>(a.V) + ((size_t)b * a.Hkv + g) * L * D;
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);  // log2(e)/sqrt(d)
  float mx = -INFINITY, den = 0.f, o[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) o[e] = 0.f;
  constexpr int UG = 4;  // entries in flight per warp
#pragma unroll 1
  for (int64_t r0 = warp; r0 < count; r0 += NW * UG) {
    float kf[UG][DL], vf[UG][DL];
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      const int64_t r = r0 + (int64_t)NW * u;
      int64_t j = 0;
      if (r < anc) j = 0;
      else if (r < anc + m) j = topj[r - anc];
      else if (r < count) j = lo + (r - anc - m);
      load_f32<T, DL>(Kg + (size_t)j * D + lane * DL, kf[u]);
      load_f32<T, DL>(Vg + (size_t)j * D + lane * DL, vf[u]);
    }
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      if (r0 + (int64_t)NW * u >= count) break;  // warp-uniform
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) dot = fmaf(qv[e], kf[u][e], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
      const float s = dot * sl2;
      const float mn = fmaxf(mx, s);
      const float corr = exp2f(mx - mn);
      const float p = exp2f(s - mn);
      den = den * corr + p;
#pragma unroll
      for (int e = 0; e < DL; ++e) o[e] = fmaf(p, vf[u][e], o[e] * corr);
      mx = mn;
    }
  }
  if (lane == 0) {
    s_m_w[warp] = mx;
    s_l_w[warp] = den;
  }
#pragma unroll
  for (int e = 0; e < DL; ++e) s_o_w[warp][lane * DL + e] = o[e];
  __syncthreads();
  if (tid < D) {
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, s_m_w[w]);
    float l = 0.f, acc = 0.f;
    for (int w = 0; w < NW; ++w) {
      if (s_l_w[w] == 0.f) continue;
      const float c = exp2f(s_m_w[w] - M);
      l += s_l_w[w] * c;
      acc += s_o_w[w][tid] * c;
    }
    TO* out = reinterpret_cast<TO*>(a.O) + ((size_t)b * a.Hq + h) * D;
    store_out<TO>(out + tid, acc / l);
  }
}

template <typename T, int D, int G>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t stream) {
  const int cap = a.k + kSub + kSlack;
  size_t smem1 = (size_t)G * cap * 8 + (size_t)a.k * 8 + sizeof(TopkShared<G>);
  auto k1 = decode_score_topk<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(
      k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  dim3 grid1(a.nchunks, a.Hkv, a.B);
  prof_before(stream, "decode_score_topk");
  k1<<<grid1, kThreads, smem1, stream>>>(a);
  prof_after(stream);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  size_t smem2 = (size_t)a.nchunks * a.k * 8 + (size_t)a.kpow2 * 4 +
                 sizeof(SelectState<1>);
  dim3 grid2(a.Hq, a.B);
  if (a.o_bf16) {
    auto k2 = decode_merge_attend<T, D, __nv_bfloat16>;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem2);
    if (e != cudaSuccess) return e;
    prof_before(stream, "decode_merge_attend");
    k2<<<grid2, kMergeThreads, smem2, stream>>>(a);
    prof_after(stream);
  } else {
    auto k2 = decode_merge_attend<T, D, float>;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem2);
    if (e != cudaSuccess) return e;
    prof_before(stream, "decode_merge_attend");
    k2<<<grid2, kMergeThreads, smem2, stream>>>(a);
    prof_after(stream);
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_typed<T, D, 1>(a, s);
    case 2: return launch_typed<T, D, 2>(a, s);
    case 4: return launch_typed<T, D, 4>(a, s);
    case 8: return launch_typed<T, D, 8>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int decode_chunks(int B, int L, int Hkv, int k) {
  // About two CTAs per SM of a 148-SM part, each chunk a multiple of 64 keys,
  // and at most 8192 merged candidates per q-head.
  const int units = B * Hkv;
  int per = (kDecodeTargetCtas + units - 1) / units;
  int cap_merge = kDecodeMaxMerge / (k > 0 ? k : 1);
  if (per > cap_merge) per = cap_merge;
  int max_by_len = (L + 255) / 256;
  if (per > max_by_len) per = max_by_len;
  if (per < 1) per = 1;
  return per;
}

int decode_chunk_len(int L, int nchunks) {
  int len = (L + nchunks - 1) / nchunks;
  return (len + 63) / 64 * 64;
}

cudaError_t decode_launch(const DecodeArgs& a, bool bf16, int d,
                          cudaStream_t s) {
  if (bf16) {
    if (d == 64) return launch_d<__nv_bfloat16, 64>(a, s);
    if (d == 128) return launch_d<__nv_bfloat16, 128>(a, s);
  } else {
    if (d == 64) return launch_d<float, 64>(a, s);
    if (d == 128) return launch_d<float, 128>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ca

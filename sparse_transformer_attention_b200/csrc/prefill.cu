// Prefill path: causal Condensate attention over n positions.
// "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质", §2.1 Definition 1,
// §2.2.1-§2.2.3, §2.4 Corollaries 2-3, §5.2.2 (identify the set, then attend
// on the subset).
//
// Launch 1 (score + select), one CTA per 128-query tile of one (batch, head):
//   bf16: the tcgen05 pipeline of prefill_tc.cu; rows whose candidates
//         overflowed its buffers go to the exact CUDA-core fallback here.
//   fp32: a per-row heap selector fed by an FFMA dot-product loop over
//         32-key tiles staged in shared memory (no TF32, so selection stays
//         exact).
// Launch 2 (gather + softmax): per row, sort the selected positions, write
//   C_i (ascending) and |C_i|, and run an fp32 online softmax over
//   {0} U Top-k U window, re-using the selector's fp32 scores for Top-k.
//   bf16 runs the window on warp-level MMA, 16 query rows per warp.
#include "common.cuh"
#include "launch.cuh"
#include "prefill.cuh"
#include "prefill_rows.cuh"
#include "profile.cuh"
#include "row_topk.cuh"
#include "select.cuh"
#include "sm100.cuh"
#include "warp_sort.cuh"

namespace ca {

namespace {

// Raw (undecoded) copy of DL consecutive elements of a row.
template <typename T, int DL>
struct RawRow {
  static constexpr int kWords = DL * (int)sizeof(T) / 16;  // 16-byte pieces
  uint4 w[kWords];
  __device__ __forceinline__ void load(const T* p) {
    const uint4* s = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int c = 0; c < kWords; ++c) w[c] = __ldg(s + c);
  }
  // 16-byte piece c as fp32 (8 bf16 or 4 fp32 elements)
  __device__ __forceinline__ void piece_f32(int c, float* f) const {
    if constexpr (sizeof(T) == 2) {
      f[0] = bf16lo(w[c].x);
      f[1] = bf16hi(w[c].x);
      f[2] = bf16lo(w[c].y);
      f[3] = bf16hi(w[c].y);
      f[4] = bf16lo(w[c].z);
      f[5] = bf16hi(w[c].z);
      f[6] = bf16lo(w[c].w);
      f[7] = bf16hi(w[c].w);
    } else {
      f[0] = __uint_as_float(w[c].x);
      f[1] = __uint_as_float(w[c].y);
      f[2] = __uint_as_float(w[c].z);
      f[3] = __uint_as_float(w[c].w);
    }
  }
  __device__ __forceinline__ void to_f32(float (&f)[DL]) const {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int c = 0; c < kWords; ++c) {
        f[8 * c + 0] = bf16lo(w[c].x);
        f[8 * c + 1] = bf16hi(w[c].x);
        f[8 * c + 2] = bf16lo(w[c].y);
        f[8 * c + 3] = bf16hi(w[c].y);
        f[8 * c + 4] = bf16lo(w[c].z);
        f[8 * c + 5] = bf16hi(w[c].z);
        f[8 * c + 6] = bf16lo(w[c].w);
        f[8 * c + 7] = bf16hi(w[c].w);
      }
    } else {
#pragma unroll
      for (int c = 0; c < kWords; ++c) {
        f[4 * c + 0] = __uint_as_float(w[c].x);
        f[4 * c + 1] = __uint_as_float(w[c].y);
        f[4 * c + 2] = __uint_as_float(w[c].z);
        f[4 * c + 3] = __uint_as_float(w[c].w);
      }
    }
  }
};

// Exact fallback for rows whose candidate buffer overflowed: one CTA per
// listed row scores every candidate on CUDA cores (fp32 FMA of the bf16 or
// fp32 inputs).  Scores are taken 2048 keys at a time; a key goes into the
// buffer only if it reaches the current threshold T (the Top-k so far are
// exactly the k keys >= T, so a key below T can never be selected), and the
// CTA radix select runs only when the buffer could not take another chunk,
// and once at the end.
constexpr int kFbThreads = 512;
constexpr int kFbBlocksPerSm = 3;  // resident CTAs per SM (registers)
constexpr int kFbChunk = 2048;
constexpr int kFbBuf = 2 * kFbChunk;  // buffered keys beyond k

template <typename T, int D>
__global__ void __launch_bounds__(kFbThreads, kFbBlocksPerSm)
prefill_overflow_rows(PrefillArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int k = a.k;
  const int lane = threadIdx.x & 31;
  float* q = reinterpret_cast<float*>(smem);               // [D], 16-byte aligned
  uint64_t* keys = reinterpret_cast<uint64_t*>(q + D);     // [k + kFbBuf]
  __shared__ int s_n, s_kk, s_w;
  __shared__ uint64_t s_T;
  __shared__ SelectState<1> st;
  const uint32_t rows = (uint32_t)(a.B * a.Hq * a.nq);
  uint32_t nrows = *a.ovf_count;
  // debug builds: the list holds at most one entry per row, each a row
  if (!in_bounds(nrows <= rows, a.status)) nrows = rows;
  for (uint32_t it = blockIdx.x; it < nrows; it += gridDim.x) {
    const uint32_t grow = a.ovf_rows[it];
    if (!in_bounds(grow < rows, a.status)) continue;
    const int r = (int)(grow % (uint32_t)a.nq);
    const uint32_t bh = grow / (uint32_t)a.nq;
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
    const int g = h / (a.Hq / a.Hkv);
    const int w = row_window(a.W_i, (int64_t)b * a.nq + r, a.W_h, h, a.W,
                             a.L, a.status, false);
    const int kh = head_k(a.k_h, h, k, a.status, false);
    const int hi = a.p0 + r - w;
    const T* Qr = reinterpret_cast<const T*>(a.Q) + (size_t)grow * D;
    const T* Kg = reinterpret_cast<const T*>(a.K) +
                  ((size_t)b * a.Hkv + g) * (size_t)a.L * D;
    for (int e = threadIdx.x; e < D; e += kFbThreads) q[e] = Elem<T>::load1(Qr + e);
    if (threadIdx.x == 0) {
      s_n = 0;
      s_T = 0ull;  // every real key is above 0
    }
    __syncthreads();
    for (int c0 = 1; c0 <= hi; c0 += kFbChunk) {
      const uint64_t thr = s_T;
      for (int jj0 = 0; jj0 < kFbChunk; jj0 += kFbThreads) {
        const int j = c0 + jj0 + (int)threadIdx.x;
        uint64_t key = 0ull;
        if (j <= hi) {
          // the key row in 16-byte pieces, every load issued before the
          // first FMA (the compiler otherwise keeps a few in flight: the
          // loop then waits on memory once per piece); q as 16-byte reads
          RawRow<T, D> kr;
          kr.load(Kg + (size_t)j * D);
          asm volatile("" ::: "memory");
          const float4* q4 = reinterpret_cast<const float4*>(q);
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int c = 0; c < RawRow<T, D>::kWords; ++c) {
            constexpr int EPW = 16 / (int)sizeof(T);  // elements per piece
            float f[EPW];
            kr.piece_f32(c, f);
#pragma unroll
            for (int e = 0; e < EPW; e += 4) {
              const float4 qv = q4[(c * EPW + e) / 4];
              a0 = fmaf(qv.x, f[e], a0);
              a1 = fmaf(qv.y, f[e + 1], a1);
              a0 = fmaf(qv.z, f[e + 2], a0);
              a1 = fmaf(qv.w, f[e + 3], a1);
            }
          }
          key = make_key(a0 + a1, (uint32_t)j);
        }
        const bool keep = j <= hi && key >= thr;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&s_n, __popc(bal));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        if (keep) keys[base + __popc(bal & ((1u << lane) - 1u))] = key;
      }
      __syncthreads();
      const bool last = c0 + kFbChunk > hi;
      if (last ? s_n > kh : s_n > k + kFbBuf - kFbChunk) {  // uniform
        if (threadIdx.x == 0) s_kk = kh;
        __syncthreads();
        cta_select_thresholds<kFbThreads, 1>(keys, 0, &s_n, &s_kk, &s_T, &st,
                                             threadIdx.x);
        // keep the keys >= T, packed to the front
        if (threadIdx.x == 0) s_w = 0;
        __syncthreads();
        uint64_t mine[(kPrefillMaxK + kFbBuf) / kFbThreads + 1];
        int cntm = 0;
        for (int e = threadIdx.x; e < s_n; e += kFbThreads) mine[cntm++] = keys[e];
        __syncthreads();
        for (int c = 0; c < cntm; ++c)
          if (mine[c] >= s_T) keys[atomicAdd(&s_w, 1)] = mine[c];
        __syncthreads();
        if (threadIdx.x == 0) s_n = kh;
        __syncthreads();
      }
    }
    uint64_t* out = a.topk + (size_t)grow * k;
    for (int e = threadIdx.x; e < k; e += kFbThreads) out[e] = e < s_n ? keys[e] : 0ull;
    __syncthreads();
  }
}

// ============================================================ fp32 FFMA kernel
template <int D, bool MASS>
__global__ void __launch_bounds__(kTileRows)
prefill_score_topk_f32(PrefillArgs a) {
  constexpr int TJ = 32;     // keys per tile
  constexpr int S = 32;      // staging slots per row
  extern __shared__ __align__(16) unsigned char smem[];
  float* sK = reinterpret_cast<float*>(smem);                       // [TJ][D]
  uint64_t* heap = reinterpret_cast<uint64_t*>(sK + TJ * D);         // [k][128]
  uint2* stage = reinterpret_cast<uint2*>(heap + (size_t)a.k * kTileRows);
  __shared__ int s_hi[kTileRows];
  __shared__ int s_maxhi;

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = qt * kTileRows;  // first query row of the tile
  const int r = threadIdx.x, row = i0 + r;
  const int kh = head_k(a.k_h, h, a.k, a.status, qt == 0 && r == 0);
  tile_rows(a, b, h, i0, s_hi, &s_maxhi);
  const int hi = s_hi[r];
  const int maxhi = s_maxhi;

  float q[D];
  const float* Qr = reinterpret_cast<const float*>(a.Q) +
                    ((size_t)(b * a.Hq + h) * a.nq + (row < a.nq ? row : 0)) * D;
#pragma unroll
  for (int e = 0; e < D; e += 4) {
    float4 v = *reinterpret_cast<const float4*>(Qr + e);
    q[e] = v.x; q[e + 1] = v.y; q[e + 2] = v.z; q[e + 3] = v.w;
  }
  const float* Kg = reinterpret_cast<const float*>(a.K) +
                    (size_t)(b * a.Hkv + g) * a.L * D;
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);
  float mrow = -INFINITY, lrow = 0.f;  // candidates' (max, sum) for masses
  RowTopk sel;
  sel.init(heap, stage, r, kh, S);
  const int T = maxhi >= 1 ? maxhi / TJ + 1 : 0;
  for (int t = 0; t < T; ++t) {
    __syncthreads();
    for (int e = threadIdx.x * 4; e < TJ * D; e += kTileRows * 4) {
      const int jj = t * TJ + e / D;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jj < a.L) v = *reinterpret_cast<const float4*>(Kg + (size_t)jj * D + e % D);
      *reinterpret_cast<float4*>(sK + e) = v;
    }
    __syncthreads();
    uint32_t raw[32];
#pragma unroll
    for (int c = 0; c < TJ; ++c) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < D; e += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(sK + c * D + e);
        acc = fmaf(q[e], kv.x, acc);
        acc = fmaf(q[e + 1], kv.y, acc);
        acc = fmaf(q[e + 2], kv.z, acc);
        acc = fmaf(q[e + 3], kv.w, acc);
      }
      raw[c] = __float_as_uint(acc);
    }
    const int j0 = t * TJ;
    if constexpr (MASS) {
      float tm = -INFINITY;
#pragma unroll
      for (int c = 0; c < TJ; ++c)
        if (j0 + c >= 1 && j0 + c <= hi)
          tm = fmaxf(tm, __uint_as_float(raw[c]));
      if (tm > -INFINITY) {
        const float mn = fmaxf(mrow, tm);
        lrow *= exp2f((mrow - mn) * sl2);
#pragma unroll
        for (int c = 0; c < TJ; ++c)
          if (j0 + c >= 1 && j0 + c <= hi)
            lrow += exp2f((__uint_as_float(raw[c]) - mn) * sl2);
        mrow = mn;
      }
    }
    if (kh > 0) {  // uniform over the CTA (one head)
      const bool interior = (j0 >= 1) && (j0 + 31 <= hi);
      if (__all_sync(0xFFFFFFFFu, interior))
        sel.offer<false>(raw, j0, 1, hi);
      else
        sel.offer<true>(raw, j0, 1, hi);
    }
  }
  const size_t grow = (size_t)(b * a.Hq + h) * a.nq + row;
  if (kh > 0) sel.drain();
  if (row < a.nq && a.k > 0) {
    uint64_t* out = a.topk + grow * a.k;
    sel.store(out);
    for (int e = kh; e < a.k; ++e) out[e] = 0ull;
  }
  if constexpr (MASS) {
    if (row < a.nq) a.cand_ml[grow] = make_float2(mrow * sl2, lrow);
  }
}

// ============================================================ gather kernel
// Warp-wide ascending bitonic sort of 32*NPL values (element e = t*32+lane
// lives in v[t] of that lane).
template <int NPL>
__device__ __forceinline__ void warp_sort(uint32_t (&v)[NPL], int lane) {
  constexpr int N = 32 * NPL;
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      uint32_t nv[NPL];
#pragma unroll
      for (int t = 0; t < NPL; ++t) {
        const int e = t * 32 + lane;
        const bool up = (e & size) == 0;
        uint32_t other = (stride >= 32)
                             ? v[t ^ (stride >> 5)]
                             : __shfl_xor_sync(0xFFFFFFFFu, v[t], stride);
        const bool lower = (e & stride) == 0;
        const uint32_t mn = min(v[t], other), mx = max(v[t], other);
        nv[t] = (lower == up) ? mn : mx;
      }
#pragma unroll
      for (int t = 0; t < NPL; ++t) v[t] = nv[t];
    }
  }
}

// Four query rows per warp, eight lanes per row (each lane holds D/8 head
// dimensions of q, of the output and of every K and V row it reads).
//   1. For each row, with the whole warp: sort the Top-k positions and write
//      C_i (ascending, -1 padded) and |C_i|.
//   2. fp32 softmax over C_i, KPC keys at a time: the K and V loads of a
//      chunk are issued together, then the chunk's scores (Top-k scores come
//      with the keys, anchor and window scores are dot products reduced over
//      the row's eight lanes) move the running maximum once.  Window rows are
//      shared by the warp's neighbouring queries, so they mostly hit L1.
constexpr int kGatherWarps = 8;
constexpr int kGatherRPW = 4;              // rows per warp
constexpr int kGatherLPR = 32 / kGatherRPW;  // lanes per row

// Write C_i (ascending, -1 padded) and |C_i| of one row, with the whole
// warp: v[] holds the row's Top-k positions (0xFFFFFFFF for empty slots,
// element t*32 + lane in v[t]), m of them real.
template <int NPL>
__device__ __forceinline__ void write_set(const PrefillArgs& a, int64_t row,
                                          uint32_t (&v)[NPL], int m, int i,
                                          int lo, int lane) {
  warp_sort<NPL>(v, lane);
  const int anc = lo > 0 ? 1 : 0;
  const int count = anc + m + (i - lo + 1);
  if (count > a.C_max && lane == 0) raise_flag(a.status, kErrCmax);
  const int wcount = count < a.C_max ? count : a.C_max;
  int32_t* out = a.idx + row * a.C_max;
  for (int rb = 0; rb < a.C_max; rb += 32) {
    const int rpos = rb + lane;
    // the sorted Top-k value for slot rpos-anc sits in lane (rpos-anc)%32
    const int tk = rpos - anc;
    uint32_t sv = 0;
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      const uint32_t x = __shfl_sync(0xFFFFFFFFu, v[t], tk & 31);
      if ((tk >> 5) == t) sv = x;
    }
    if (rpos < a.C_max) {
      int32_t val;
      if (rpos >= wcount) val = -1;
      else if (rpos < anc) val = 0;
      else if (tk < m) val = (int32_t)sv;
      else val = lo + (tk - m);
      out[rpos] = val;
    }
  }
  if (lane == 0) a.idx_count[row] = count;
}

template <typename T, int D, typename TO, int NPL, bool MASS>
__global__ void __launch_bounds__(kGatherWarps * 32)
prefill_gather(PrefillArgs a) {
  constexpr int DL = D / kGatherLPR;
  constexpr int KPC = 4;  // keys per chunk
  __shared__ uint64_t s_key[kGatherWarps][kGatherRPW][kPrefillMaxK];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nq = a.nq;
  const int64_t R = (int64_t)a.B * a.Hq * nq;
  const int64_t row0 = ((int64_t)blockIdx.x * kGatherWarps + wid) * kGatherRPW;
  if (row0 >= R) return;  // the whole warp
  const int k = a.k;

  // ---- 1: C_i, one row at a time across the warp
#pragma unroll 1
  for (int rr = 0; rr < kGatherRPW; ++rr) {
    const int64_t row = row0 + rr;
    if (row >= R) break;
    const int64_t bh = row / nq;
    const int r = (int)(row - bh * nq);
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
    const int i = a.p0 + r;
    const int w = row_window(a.W_i, (int64_t)b * nq + r, a.W_h, h, a.W, a.L,
                             a.status, false);
    const int lo = i - w + 1 > 0 ? i - w + 1 : 0;
    uint32_t v[NPL];
    int m = 0;
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      const int e = t * 32 + lane;
      uint64_t key = 0ull;
      if (e < k) key = a.topk[row * k + e];
      if (e < k) s_key[wid][rr][e] = key;
      v[t] = key ? key_index(key) : 0xFFFFFFFFu;
      m += __popc(__ballot_sync(0xFFFFFFFFu, key != 0ull));
    }
    write_set<NPL>(a, row, v, m, i, lo, lane);
  }
  __syncwarp();

  // ---- 2: softmax over C_i, eight lanes per row
  const int rloc = lane / kGatherLPR, sub = lane % kGatherLPR;
  const int64_t row = row0 + rloc;
  const bool live = row < R;
  const int64_t rowc = live ? row : R - 1;
  const int64_t bh = rowc / nq;
  const int r = (int)(rowc - bh * nq);
  const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const int i = a.p0 + r;
  const int w = row_window(a.W_i, (int64_t)b * nq + r, a.W_h, h, a.W, a.L,
                           a.status, false);
  const int lo = i - w + 1 > 0 ? i - w + 1 : 0;
  const int anc = lo > 0 ? 1 : 0;
  const T* Kg = reinterpret_cast<const T*>(a.K) +
                ((size_t)b * a.Hkv + g) * (size_t)a.L * D + sub * DL;
  const T* Vg = reinterpret_cast<const T*>(a.V) +
                ((size_t)b * a.Hkv + g) * (size_t)a.L * D + sub * DL;
  float qv[DL];
  {
    RawRow<T, DL> qr;
    qr.load(reinterpret_cast<const T*>(a.Q) + rowc * D + sub * DL);
    qr.to_f32(qv);
  }
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);
  float mrun = -INFINITY, den = 0.f, o[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) o[e] = 0.f;

  // fold a chunk of scores s[u] (log2 units; -inf = no key) and V rows
  auto fold = [&](const float (&s)[KPC], const RawRow<T, DL> (&vr)[KPC]) {
    float cm = s[0];
#pragma unroll
    for (int u = 1; u < KPC; ++u) cm = fmaxf(cm, s[u]);
    if (cm == -INFINITY) return;  // uniform over the row's lanes
    const float mn = fmaxf(mrun, cm);
    const float sc = exp2f(mrun - mn);
    den *= sc;
#pragma unroll
    for (int e = 0; e < DL; ++e) o[e] *= sc;
#pragma unroll
    for (int u = 0; u < KPC; ++u) {
      const float p = exp2f(s[u] - mn);  // 0 for s = -inf
      float vf[DL];
      vr[u].to_f32(vf);
      den += p;
#pragma unroll
      for (int e = 0; e < DL; ++e) o[e] = fmaf(p, vf[e], o[e]);
    }
    mrun = mn;
  };

  // anchor and window first: dot products over the row's eight lanes
  const int nw = live ? anc + (i - lo + 1) : 0;
  int nmax = nw;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    nmax = max(nmax, __shfl_xor_sync(0xFFFFFFFFu, nmax, off));
  for (int c0 = 0; c0 < nmax; c0 += KPC) {
    RawRow<T, DL> kr[KPC], vr[KPC];
    int jj[KPC];
#pragma unroll
    for (int u = 0; u < KPC; ++u) {
      const int li = c0 + u;
      jj[u] = li < nw ? ((anc && li == 0) ? 0 : lo + li - anc) : 0;
      kr[u].load(Kg + (size_t)jj[u] * D);
      vr[u].load(Vg + (size_t)jj[u] * D);
    }
    float s[KPC];
#pragma unroll
    for (int u = 0; u < KPC; ++u) {
      float kf[DL];
      kr[u].to_f32(kf);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < DL; e += 2) {
        d0 = fmaf(qv[e], kf[e], d0);
        d1 = fmaf(qv[e + 1], kf[e + 1], d1);
      }
      s[u] = d0 + d1;
    }
#pragma unroll
    for (int off = kGatherLPR / 2; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < KPC; ++u)
        s[u] += __shfl_xor_sync(0xFFFFFFFFu, s[u], off);
#pragma unroll
    for (int u = 0; u < KPC; ++u)
      s[u] = (c0 + u < nw) ? s[u] * sl2 : -INFINITY;
    fold(s, vr);
  }
  const float m_wa = mrun, l_wa = den;  // window + anchor alone
  // Top-k entries: the selector's fp32 scores
  for (int c0 = 0; c0 < k; c0 += KPC) {
    float s[KPC];
    RawRow<T, DL> vr[KPC];
#pragma unroll
    for (int u = 0; u < KPC; ++u) {
      const int e = c0 + u;
      const uint64_t key = (live && e < k) ? s_key[wid][rloc][e] : 0ull;
      uint32_t j = key ? key_index(key) : 0u;
      bool act = key != 0ull;
      if (act && (j == 0 || (int64_t)j > (int64_t)(i - w))) {  // not a candidate
        raise_flag(a.status, kErrInternal);
        act = false;
        j = 0;
      }
      s[u] = act ? key_score(key) * sl2 : -INFINITY;
      vr[u].load(Vg + (size_t)j * D);
    }
    fold(s, vr);
  }
  if (live) {
    TO* op = reinterpret_cast<TO*>(a.O) + rowc * D + sub * DL;
    const float inv = 1.f / den;
#pragma unroll
    for (int e = 0; e < DL; ++e) store_out<TO>(op + e, o[e] * inv);
  }
  if constexpr (MASS) {
    // the anchor's own score (inside the window when it reaches 0)
    RawRow<T, DL> k0;
    k0.load(Kg);
    float kf[DL];
    k0.to_f32(kf);
    float d0 = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) d0 = fmaf(qv[e], kf[e], d0);
#pragma unroll
    for (int off = kGatherLPR / 2; off > 0; off >>= 1)
      d0 += __shfl_xor_sync(0xFFFFFFFFu, d0, off);
    if (live && sub == 0) {
      const float2 cm = a.cand_ml[row];
      mass_report(a.mass, a.lse, (size_t)row, mrun, den, m_wa, l_wa, cm.x,
                  cm.y, d0 * sl2, anc != 0);
    }
  }
}

// ------------------------------------------------- tensor-core window part
// Warp-level MMA (mma.sync) on the banded window scores: 16 query rows per
// warp against 16-key blocks of the rows' window span.  Scores: m16n8k16 with
// bf16 Q and K, fp32 accumulation (exact products, like the CUDA-core dot).
// p * V: m16n8k8 with tf32 p (rounded from fp32, 11 significant bits) and V
// (bf16 widened exactly), so the weights keep more precision than bf16.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4],
                                               const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_tf32_1688(float (&d)[4], uint32_t a0,
                                              uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ uint32_t ld_b32(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const unsigned int*>(p));
}

constexpr int kMmaWarps = 4;  // 16 query rows each

// Shared memory of the bf16 gather: the Top-k keys of every warp's 16 rows
// (kept to the end), then the window's K and V rows staged in chunks of 64
// keys (two buffers, rows padded by 16 bytes so that the fragment loads of
// eight rows fall on different banks).  After the window phase the staging
// bytes hold each warp's window state (o, max, sums) instead.
template <int D>
struct MmaGatherSmem {
  static constexpr int CK = 64;                 // keys per staged chunk
  static constexpr int RS = D * 2 + 16;         // padded row stride (bytes)
  static constexpr size_t chunk = (size_t)CK * RS;
  static constexpr size_t stage = 4 * chunk;    // two buffers of K and V
  static constexpr size_t state = (size_t)16 * D * 4 + 3 * 16 * 4;
  static_assert(stage >= kMmaWarps * state, "window state fits the staging");
  __host__ __device__ static size_t keys(int k) {
    return (size_t)kMmaWarps * 16 * k * 8;
  }
  __host__ __device__ static size_t bytes(int k) { return keys(k) + stage; }
};

__device__ __forceinline__ uint32_t lds32(const unsigned char* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}
__device__ __forceinline__ uint32_t lds_bf16_as_f32(const unsigned char* p) {
  return (uint32_t)(*reinterpret_cast<const unsigned short*>(p)) << 16;
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// bf16 gather with the window on tensor cores.  A CTA owns 64 consecutive
// query rows of one (batch, head), a warp 16 of them.
//   1. The Top-k keys of the warp's rows into shared memory in one batch of
//      loads, then C_i and |C_i| for each row (whole warp per row).
//   2. The window [lo_i, i] of all rows: the CTA stages the K and V rows of
//      the window span in 64-key chunks (16-byte asynchronous copies, the
//      next chunk in flight while the current one is used); each warp runs
//      its rows over the 16-key blocks it needs: MMA scores, masked per row,
//      an online softmax per row, and the MMA p * V, with every fragment
//      read from shared memory.  The state (max, sum, unnormalised o) then
//      goes to shared memory.
//   3. Eight lanes per row, four rows at a time: start from the window state
//      and fold in the Top-k keys (scores from the selector) and the anchor
//      (score computed here), then write the output row.
template <int D, typename TO, int NPL, bool MASS>
__global__ void __launch_bounds__(kMmaWarps * 32)
prefill_gather_mma(PrefillArgs a) {
  using T = __nv_bfloat16;
  using SM = MmaGatherSmem<D>;
  constexpr int KS = D / 16;  // k-steps of the score MMA
  constexpr int NT = D / 8;   // head-dim tiles of the p * V MMA
  constexpr int RS = SM::RS;
  extern __shared__ __align__(16) unsigned char g_smem[];
  __shared__ int s_kmin;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  // query rows r at positions p0 + r, keys 0..L-1
  const int nq = a.nq, L = a.L, p0 = a.p0, k = a.k;
  uint64_t* s_key = reinterpret_cast<uint64_t*>(g_smem) + (size_t)wid * 16 * k;
  unsigned char* stage = g_smem + SM::keys(k);
  float* s_o = reinterpret_cast<float*>(stage + wid * SM::state);
  float* s_m = s_o + 16 * D;
  float* s_l = s_m + 16;
  float* s_lx = s_l + 16;  // window sums of the unrounded weights (reports)
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int r0 = blockIdx.x * kMmaWarps * 16;  // first query row of the CTA
  const int i0 = r0 + wid * 16;                // first query row of the warp
  const bool wlive = i0 < nq;  // every warp takes part in the staging
  const int64_t rowbase = (int64_t)bh * nq;
  const T* Qg = reinterpret_cast<const T*>(a.Q) + rowbase * D;
  const T* Kg = reinterpret_cast<const T*>(a.K) + ((size_t)b * a.Hkv + g) * (size_t)L * D;
  const T* Vg = reinterpret_cast<const T*>(a.V) + ((size_t)b * a.Hkv + g) * (size_t)L * D;
  if (threadIdx.x == 0) s_kmin = 0x7FFFFFFF;
  __syncthreads();

  if (wlive) {
  // ---- 1: the Top-k keys of the warp's rows (16 consecutive rows of one
  // head: one contiguous run) into shared memory, 16 loads in flight per
  // lane, then C_i one row at a time across the warp
  {
    const int nk = min(16, nq - i0) * k;
    const uint64_t* kg = a.topk + (rowbase + i0) * k;
#pragma unroll 1
    for (int e0 = 0; e0 < nk; e0 += 16 * 32) {
      uint64_t t16[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int e = e0 + u * 32 + lane;
        t16[u] = e < nk ? __ldg(kg + e) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int e = e0 + u * 32 + lane;
        if (e < nk) s_key[e] = t16[u];
      }
    }
    __syncwarp();
  }
#pragma unroll 1
  for (int rr = 0; rr < 16; ++rr) {
    const int r = i0 + rr;
    if (r >= nq) break;
    const int i = p0 + r;  // position
    const int w = row_window(a.W_i, (int64_t)b * nq + r, a.W_h, h, a.W, L,
                             a.status, false);
    const int lo = i - w + 1 > 0 ? i - w + 1 : 0;
    uint32_t v[NPL];
    int m = 0;
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      const int e = t * 32 + lane;
      const uint64_t key = e < k ? s_key[rr * k + e] : 0ull;
      v[t] = key ? key_index(key) : 0xFFFFFFFFu;
      m += __popc(__ballot_sync(0xFFFFFFFFu, key != 0ull));
    }
    write_set<NPL>(a, rowbase + r, v, m, i, lo, lane);
  }

  }  // wlive

  // ---- 2: window on tensor cores
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);
  const int gr = lane >> 2, tq = lane & 3;  // fragment row group, thread in group
  const int ra = i0 + gr, rb = i0 + gr + 8;  // this lane's two rows
  const bool va = ra < nq, vb = rb < nq;
  const int ca = va ? ra : nq - 1, cb = vb ? rb : nq - 1;
  const int ia = p0 + ca, ib = p0 + cb;      // their positions
  const int wa = row_window(a.W_i, (int64_t)b * nq + ca, a.W_h, h, a.W, L,
                            a.status, false);
  const int wb = row_window(a.W_i, (int64_t)b * nq + cb, a.W_h, h, a.W, L,
                            a.status, false);
  const int loa = ia - wa + 1 > 0 ? ia - wa + 1 : 0;
  const int lob = ib - wb + 1 > 0 ? ib - wb + 1 : 0;
  int kmin = min(loa, lob);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    kmin = min(kmin, __shfl_xor_sync(0xFFFFFFFFu, kmin, off));
  const int kmax = p0 + min(i0 + 15, nq - 1);
  if (wlive && lane == 0) atomicMin(&s_kmin, kmin);
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int c = 16 * ks + 2 * tq;
    qa[ks][0] = ld_b32(Qg + (size_t)ca * D + c);
    qa[ks][1] = ld_b32(Qg + (size_t)cb * D + c);
    qa[ks][2] = ld_b32(Qg + (size_t)ca * D + c + 8);
    qa[ks][3] = ld_b32(Qg + (size_t)cb * D + c + 8);
  }
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
  float lax = 0.f, lbx = 0.f;  // the same sums over the unrounded weights
  float o[NT][4];
#pragma unroll
  for (int nd = 0; nd < NT; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;

  // the CTA's window span, staged in chunks of SM::CK keys starting at a
  // multiple of 16 (a 16-key block never straddles two chunks)
  __syncthreads();
  const int cs0 = s_kmin & ~15;
  const int kmax_c = p0 + min(r0 + kMmaWarps * 16 - 1, nq - 1);
  const int nch = (kmax_c - cs0) / SM::CK + 1;
  auto stage_chunk = [&](int m) {
    unsigned char* dK = stage + (m & 1) * 2 * SM::chunk;
    unsigned char* dV = dK + SM::chunk;
    const int cs = cs0 + m * SM::CK;
    constexpr int kPieces = D * 2 / 16;  // 16-byte pieces per row
    for (int e = threadIdx.x; e < SM::CK * kPieces; e += kMmaWarps * 32) {
      const int rr = e / kPieces, pc = e % kPieces;
      const int j = min(cs + rr, L - 1);  // rows past the cache: any valid
      cp_async16(dK + rr * RS + pc * 16, Kg + (size_t)j * D + pc * 8);
      cp_async16(dV + rr * RS + pc * 16, Vg + (size_t)j * D + pc * 8);
    }
    cp_async_commit();
  };
  stage_chunk(0);
#pragma unroll 1
  for (int m = 0; m < nch; ++m) {
    if (m + 1 < nch) {
      stage_chunk(m + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int cs = cs0 + m * SM::CK;
    const unsigned char* sK = stage + (m & 1) * 2 * SM::chunk;
    const unsigned char* sV = sK + SM::chunk;
    const int jlo = max(cs, kmin & ~15), jhi = min(cs + SM::CK - 1, kmax);
#pragma unroll 1
    for (int j0 = jlo; wlive && j0 <= jhi; j0 += 16) {
        float s[2][4];
    #pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          const unsigned char* kr = sK + (j0 - cs + 8 * h8 + gr) * RS;
    #pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int c = 16 * ks + 2 * tq;
            mma_bf16_16816(acc, qa[ks], lds32(kr + c * 2), lds32(kr + c * 2 + 16));
          }
          const int kc = j0 + 8 * h8 + 2 * tq;  // key of acc[0] / acc[2]
          s[h8][0] = (va && kc >= loa && kc <= ia) ? acc[0] * sl2 : -INFINITY;
          s[h8][1] = (va && kc + 1 >= loa && kc + 1 <= ia) ? acc[1] * sl2 : -INFINITY;
          s[h8][2] = (vb && kc >= lob && kc <= ib) ? acc[2] * sl2 : -INFINITY;
          s[h8][3] = (vb && kc + 1 >= lob && kc + 1 <= ib) ? acc[3] * sl2 : -INFINITY;
        }
        float xa = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        float xb = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
        xa = fmaxf(xa, __shfl_xor_sync(0xFFFFFFFFu, xa, 1));
        xa = fmaxf(xa, __shfl_xor_sync(0xFFFFFFFFu, xa, 2));
        xb = fmaxf(xb, __shfl_xor_sync(0xFFFFFFFFu, xb, 1));
        xb = fmaxf(xb, __shfl_xor_sync(0xFFFFFFFFu, xb, 2));
        const float na = fmaxf(ma, xa), nb = fmaxf(mb, xb);
        const float sa = na == -INFINITY ? 1.f : exp2f(ma - na);
        const float sb = nb == -INFINITY ? 1.f : exp2f(mb - nb);
        la *= sa;
        lb *= sb;
        if constexpr (MASS) {
          lax *= sa;
          lbx *= sb;
        }
    #pragma unroll
        for (int nd = 0; nd < NT; ++nd) {
          o[nd][0] *= sa;
          o[nd][1] *= sa;
          o[nd][2] *= sb;
          o[nd][3] *= sb;
        }
        uint32_t p[2][4];
    #pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const float p0 = s[h8][0] == -INFINITY ? 0.f : exp2f(s[h8][0] - na);
          const float p1 = s[h8][1] == -INFINITY ? 0.f : exp2f(s[h8][1] - na);
          const float p2 = s[h8][2] == -INFINITY ? 0.f : exp2f(s[h8][2] - nb);
          const float p3 = s[h8][3] == -INFINITY ? 0.f : exp2f(s[h8][3] - nb);
          p[h8][0] = to_tf32(p0);
          p[h8][1] = to_tf32(p1);
          p[h8][2] = to_tf32(p2);
          p[h8][3] = to_tf32(p3);
          // the sums use the rounded weights, as the MMA does
          la += __uint_as_float(p[h8][0]) + __uint_as_float(p[h8][1]);
          lb += __uint_as_float(p[h8][2]) + __uint_as_float(p[h8][3]);
          if constexpr (MASS) {
            lax += p0 + p1;
            lbx += p2 + p3;
          }
        }
        // p * V, keys of the k8 step ordered (2t, 2t+1) -> (t, t+4) so that the
        // score fragment is the A fragment as it stands
    #pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const unsigned char* v0r = sV + (j0 - cs + 8 * h8 + 2 * tq) * RS;
          const unsigned char* v1r = v0r + RS;
    #pragma unroll
          for (int nd = 0; nd < NT; ++nd) {
            const uint32_t b0 = lds_bf16_as_f32(v0r + (8 * nd + gr) * 2);
            const uint32_t b1 = lds_bf16_as_f32(v1r + (8 * nd + gr) * 2);
            mma_tf32_1688(o[nd], p[h8][0], p[h8][2], p[h8][1], p[h8][3], b0, b1);
          }
        }
        ma = na;
        mb = nb;
    }
    __syncthreads();  // the next chunk overwrites this buffer
  }
  if (!wlive) return;
  la += __shfl_xor_sync(0xFFFFFFFFu, la, 1);
  la += __shfl_xor_sync(0xFFFFFFFFu, la, 2);
  lb += __shfl_xor_sync(0xFFFFFFFFu, lb, 1);
  lb += __shfl_xor_sync(0xFFFFFFFFu, lb, 2);
  if constexpr (MASS) {
    lax += __shfl_xor_sync(0xFFFFFFFFu, lax, 1);
    lax += __shfl_xor_sync(0xFFFFFFFFu, lax, 2);
    lbx += __shfl_xor_sync(0xFFFFFFFFu, lbx, 1);
    lbx += __shfl_xor_sync(0xFFFFFFFFu, lbx, 2);
  }
  if (tq == 0) {
    s_m[gr] = ma;
    s_m[gr + 8] = mb;
    s_l[gr] = la;
    s_l[gr + 8] = lb;
    s_lx[gr] = lax;
    s_lx[gr + 8] = lbx;
  }
#pragma unroll
  for (int nd = 0; nd < NT; ++nd) {
    *reinterpret_cast<float2*>(s_o + gr * D + 8 * nd + 2 * tq) =
        make_float2(o[nd][0], o[nd][1]);
    *reinterpret_cast<float2*>(s_o + (gr + 8) * D + 8 * nd + 2 * tq) =
        make_float2(o[nd][2], o[nd][3]);
  }
  __syncwarp();

  // ---- 3: Top-k keys and the anchor, eight lanes per row
  constexpr int DL = D / 8;
  constexpr int KPC = D == 64 ? 8 : 4;
  const int sub = lane & 7, rq = lane >> 3;
  // the anchor's K and V rows are the same for all of the warp's rows
  RawRow<T, DL> k0r, v0r;
  k0r.load(Kg + sub * DL);
  v0r.load(Vg + sub * DL);
#pragma unroll 1
  for (int rg = 0; rg < 4; ++rg) {
    const int r = rg * 4 + rq;
    const bool live = i0 + r < nq;
    const int rc = live ? i0 + r : nq - 1;  // query row (clamped)
    const int ic = p0 + rc;                 // its position
    const int64_t row = rowbase + rc;
    const int w = row_window(a.W_i, (int64_t)b * nq + rc, a.W_h, h, a.W, L,
                             a.status, false);
    const int lo = ic - w + 1 > 0 ? ic - w + 1 : 0;
    const float m_win = s_m[r], l_win = s_lx[r];  // the window alone
    // den: sum over C_i with the window's rounded weights (normalises the
    // output); denx: the same with unrounded weights (mass reports)
    float mrun = s_m[r], den = s_l[r], denx = s_lx[r], ov[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) ov[e] = s_o[r * D + sub * DL + e];
    float qv[DL];
    {
      RawRow<T, DL> qr;
      qr.load(Qg + (size_t)rc * D + sub * DL);
      qr.to_f32(qv);
    }
    auto fold = [&](const float (&sc)[KPC], const RawRow<T, DL> (&vr)[KPC]) {
      float cm = sc[0];
#pragma unroll
      for (int u = 1; u < KPC; ++u) cm = fmaxf(cm, sc[u]);
      if (cm == -INFINITY) return;  // uniform over the row's lanes
      const float mn = fmaxf(mrun, cm);
      const float f = exp2f(mrun - mn);
      den *= f;
      if constexpr (MASS) denx *= f;
#pragma unroll
      for (int e = 0; e < DL; ++e) ov[e] *= f;
#pragma unroll
      for (int u = 0; u < KPC; ++u) {
        const float pw = exp2f(sc[u] - mn);
        float vf[DL];
        vr[u].to_f32(vf);
        den += pw;
        if constexpr (MASS) denx += pw;
#pragma unroll
        for (int e = 0; e < DL; ++e) ov[e] = fmaf(pw, vf[e], ov[e]);
      }
      mrun = mn;
    };
    const T* Vs = Vg + sub * DL;
    for (int c0 = 0; c0 < k; c0 += KPC) {
      float sc[KPC];
      RawRow<T, DL> vr[KPC];
#pragma unroll
      for (int u = 0; u < KPC; ++u) {
        const int e = c0 + u;
        const uint64_t key = (live && e < k) ? s_key[r * k + e] : 0ull;
        uint32_t j = key ? key_index(key) : 0u;
        bool act = key != 0ull;
        if (act && (j == 0 || (int64_t)j > (int64_t)(ic - w))) {  // not a candidate
          raise_flag(a.status, kErrInternal);
          act = false;
          j = 0;
        }
        sc[u] = act ? key_score(key) * sl2 : -INFINITY;
        vr[u].load(Vs + (size_t)j * D);
      }
      fold(sc, vr);
    }
    // the anchor (position 0) when it lies outside the window
    {
      float kf[DL];
      k0r.to_f32(kf);
      float d0 = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) d0 = fmaf(qv[e], kf[e], d0);
#pragma unroll
      for (int off = 4; off > 0; off >>= 1)
        d0 += __shfl_xor_sync(0xFFFFFFFFu, d0, off);
      if (live && lo > 0) {  // uniform over the row's lanes
        const float s0 = d0 * sl2;
        const float mn = fmaxf(mrun, s0);
        const float f = exp2f(mrun - mn);
        const float pw = exp2f(s0 - mn);
        float vf[DL];
        v0r.to_f32(vf);
        den = den * f + pw;
        if constexpr (MASS) denx = denx * f + pw;
#pragma unroll
        for (int e = 0; e < DL; ++e) ov[e] = fmaf(pw, vf[e], ov[e] * f);
        mrun = mn;
      }
      if constexpr (MASS) {
        if (live && sub == 0) {
          Lse2 wa;  // window + anchor
          wa.merge(m_win, l_win);
          if (lo > 0) wa.add(d0 * sl2);
          const float2 cm = a.cand_ml[row];
          mass_report(a.mass, a.lse, (size_t)row, mrun, denx, wa.m, wa.l,
                      cm.x, cm.y, d0 * sl2, lo > 0);
        }
      }
    }
    if (live) {
      TO* op = reinterpret_cast<TO*>(a.O) + row * D + sub * DL;
      const float inv = 1.f / den;
#pragma unroll
      for (int e = 0; e < DL; ++e) store_out<TO>(op + e, ov[e] * inv);
    }
  }
}

// ============================================================ host side
bool want_mass(const PrefillArgs& a) {
  return a.mass != nullptr || a.lse != nullptr;
}

template <int D>
cudaError_t launch_overflow_d(const PrefillArgs& a, cudaStream_t s) {
  const size_t fb_smem = (size_t)(a.k + kFbBuf) * 8 + D * 4;
  // A listed row is one CTA's job, latency-bound on its key-row loads: 512
  // threads per row and every resident CTA slot of the GPU (three per SM)
  // keep the most loads in flight (the row count is only known on the
  // device; CTAs without a row leave at once).
  prof_before(s, "prefill_overflow_rows");
  prefill_overflow_rows<__nv_bfloat16, D>
      <<<kFbBlocksPerSm * sm_count(), kFbThreads, fb_smem, s>>>(a);
  prof_after(s);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_select_f32(const PrefillArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)32 * D * 4 + (size_t)a.k * kTileRows * 8 +
                      (size_t)32 * kTileRows * 8;
  auto kern = want_mass(a) ? prefill_score_topk_f32<D, true>
                           : prefill_score_topk_f32<D, false>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.nq + 127) / 128, a.Hq, a.B);
  prof_before(s, "prefill_score_topk_f32");
  kern<<<grid, kTileRows, smem, s>>>(a);
  prof_after(s);
  return cudaGetLastError();
}

template <typename T, int D, typename TO, int NPL>
void gather_f32_as(const PrefillArgs& a, dim3 grid, int nt, cudaStream_t s) {
  if (want_mass(a)) prefill_gather<T, D, TO, NPL, true><<<grid, nt, 0, s>>>(a);
  else prefill_gather<T, D, TO, NPL, false><<<grid, nt, 0, s>>>(a);
}

template <typename T, int D>
cudaError_t launch_gather(const PrefillArgs& a, cudaStream_t s) {
  const int64_t R = (int64_t)a.B * a.Hq * a.nq;
  const int64_t rows_per_cta = (int64_t)kGatherWarps * kGatherRPW;
  dim3 grid((unsigned)((R + rows_per_cta - 1) / rows_per_cta));
  const int nt = kGatherWarps * 32;
  prof_before(s, "prefill_gather");
  if (a.k <= 32) {
    if (a.o_bf16) gather_f32_as<T, D, __nv_bfloat16, 1>(a, grid, nt, s);
    else gather_f32_as<T, D, float, 1>(a, grid, nt, s);
  } else if (a.k <= 64) {
    if (a.o_bf16) gather_f32_as<T, D, __nv_bfloat16, 2>(a, grid, nt, s);
    else gather_f32_as<T, D, float, 2>(a, grid, nt, s);
  } else {
    if (a.o_bf16) gather_f32_as<T, D, __nv_bfloat16, 4>(a, grid, nt, s);
    else gather_f32_as<T, D, float, 4>(a, grid, nt, s);
  }
  prof_after(s);
  return cudaGetLastError();
}

template <int D, int NPL, bool MASS>
cudaError_t gather_mma_as(const PrefillArgs& a, dim3 grid, size_t smem,
                          cudaStream_t s) {
  auto kern = a.o_bf16 ? prefill_gather_mma<D, __nv_bfloat16, NPL, MASS>
                       : prefill_gather_mma<D, float, NPL, MASS>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  prof_before(s, "prefill_gather");
  kern<<<grid, kMmaWarps * 32, smem, s>>>(a);
  prof_after(s);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_gather_mma(const PrefillArgs& a, cudaStream_t s) {
  dim3 grid((unsigned)((a.nq + 16 * kMmaWarps - 1) / (16 * kMmaWarps)),
            (unsigned)(a.B * a.Hq));
  const size_t smem = MmaGatherSmem<D>::bytes(a.k);
  const bool m = want_mass(a);
  if (a.k <= 32)
    return m ? gather_mma_as<D, 1, true>(a, grid, smem, s)
             : gather_mma_as<D, 1, false>(a, grid, smem, s);
  if (a.k <= 64)
    return m ? gather_mma_as<D, 2, true>(a, grid, smem, s)
             : gather_mma_as<D, 2, false>(a, grid, smem, s);
  return m ? gather_mma_as<D, 4, true>(a, grid, smem, s)
           : gather_mma_as<D, 4, false>(a, grid, smem, s);
}

}  // namespace

size_t prefill_topk_bytes(int64_t rows, int k) {
  size_t bytes = (size_t)rows * (size_t)(k > 0 ? k : 1) * 8;
  return (bytes + 255) / 256 * 256;
}

size_t prefill_workspace(int64_t rows, int k) {
  // per-row Top-k keys, the list of rows for the exact fallback, and the
  // candidates' (max, sum) per row for the mass reports
  return prefill_topk_bytes(rows, k) + ((size_t)rows * 4 + 255) / 256 * 256 +
         ((size_t)rows * 8 + 255) / 256 * 256;
}

cudaError_t prefill_launch(const PrefillArgs& a, bool bf16, int d,
                           cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (a.k > 0 || want_mass(a)) {
    if (bf16) {
      e = launch_select_tc(a, d, s);
      // rows whose candidates overflowed their buffers (rare on typical
      // inputs): the exact fallback
      if (e == cudaSuccess && a.k > 0)
        e = d == 64 ? launch_overflow_d<64>(a, s) : launch_overflow_d<128>(a, s);
    } else {
      e = d == 64 ? launch_select_f32<64>(a, s) : launch_select_f32<128>(a, s);
    }
    if (e != cudaSuccess) return e;
  }
  if (bf16) e = d == 64 ? launch_gather_mma<64>(a, s) : launch_gather_mma<128>(a, s);
  else e = d == 64 ? launch_gather<float, 64>(a, s) : launch_gather<float, 128>(a, s);
  return e;
}

}  // namespace ca

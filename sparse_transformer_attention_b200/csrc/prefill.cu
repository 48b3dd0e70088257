// Prefill path: causal Condensate attention over n positions.
// "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质", §2.1 Definition 1,
// §2.2.1-§2.2.3, §2.4 Corollaries 2-3, §5.2.2 (identify the set, then attend
// on the subset).
//
// Launch 1 (score + select), one CTA per 128-query tile of one (batch, head):
//   bf16: warp-specialised tcgen05 pipeline.  Warp 0 issues TMA loads of the
//         Q tile (once) and of 128-key K tiles into a ring of shared-memory
//         stages; warp 1 issues tcgen05.mma (M=128, N=128, K=16 steps, bf16
//         in, fp32 out) into one of two TMEM accumulators; warps 2-5 read the
//         scores back with tcgen05.ld (one thread per query row) and feed the
//         row's streaming Top-k.  Only key tiles that hold candidates of some
//         row of the tile are computed (causal tile skipping), and the score
//         matrix never leaves the SM.
//   fp32: the same selector fed by an FFMA dot-product loop over 32-key
//         tiles staged in shared memory (no TF32, so selection stays exact).
// Launch 2 (gather + softmax): per row, sort the selected positions, write
//   C_i (ascending) and |C_i|, and run an fp32 online softmax over
//   {0} U Top-k U window, re-using the selector's fp32 scores for Top-k.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "prefill.cuh"
#include "profile.cuh"
#include "row_topk.cuh"
#include "select.cuh"
#include "sm100.cuh"
#include "warp_sort.cuh"

namespace ca {

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per bounded wait
constexpr int kGatherThreads = 256;

// ------------------------------------------------------------ shared prologue
// Window and last candidate position of each row of the tile; returns the
// largest last-candidate position over the tile's rows (-1 if none).
__device__ void tile_rows(const PrefillArgs& a, int b, int i0, int* s_hi,
                          int* s_maxhi) {
  const int tid = threadIdx.x;
  if (tid == 0) *s_maxhi = -1;
  __syncthreads();
  if (tid < kTileRows) {
    const int i = i0 + tid;
    int hi = -1;
    if (i < a.n) {
      const int w = row_window(a.W_i, (int64_t)b * a.n + i, a.W, a.n,
                               a.status, true);
      hi = i - w;
    }
    s_hi[tid] = hi;
    atomicMax(s_maxhi, hi);
  }
  __syncthreads();
}

// ============================================================ tcgen05 kernel
// Two passes over the row tile's key tiles (the tensor pipe has room for
// them; the selector is what costs):
//   pass 1: every selector thread keeps, for its query row, the maximum over
//           each of 32 column positions of its 32-column chunk of every key
//           tile (128 slots per row over the four chunk groups).  The k-th
//           largest slot maximum L is a lower bound of the row's k-th best
//           score: the top k slots are k distinct candidates, all >= L.
//   pass 2: recompute the scores and append every candidate with score >= L
//           to the row's buffer (about 1.1-1.4 k entries on random data).
// The exact Top-k is then taken from the buffer with a small heap.  A row
// whose buffer would overflow is listed for an exact CUDA-core fallback.
constexpr int kSelWarps = 16;                       // 4 chunk groups x 4 quarters
constexpr int kTcThreads = 64 + 32 * kSelWarps;     // + TMA warp + MMA warp
constexpr int kMinCap = 64;                         // the slot table needs 64 KiB
using SelBar = GroupBarrier<1, 32 * kSelWarps>;

template <int D>
struct TcLayout {
  static constexpr int BM = 128, BN = 128;
  static constexpr int KB = D / 64;                   // 128-byte column blocks
  static constexpr int NS = (D == 64) ? 4 : 2;        // K stages
  static constexpr uint32_t kQBytes = BM * D * 2;
  static constexpr uint32_t kKBytes = BN * D * 2;
  static constexpr uint32_t kBlockBytes = 128 * 128;  // 128 rows x 128 bytes
  static constexpr size_t q_off = 0;
  static constexpr size_t k_off = q_off + kQBytes;
  static constexpr size_t buf_off = k_off + (size_t)NS * kKBytes;
  // row buffers [cap][128] keys; + 1 KiB for the manual 1024-byte alignment
  __host__ __device__ static size_t bytes(int cap) {
    return buf_off + (size_t)cap * kTileRows * 8 + 1024;
  }
};

struct TcShared {
  uint64_t kfull[4], kempty[4], qfull, tfull[2], tempty[2];
  uint32_t tmem;
  int abort;
  int maxhi;
  int hi[kTileRows];
  float L[kTileRows];
  int cnt[kTileRows];
  int ovf[kTileRows];
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag,
                                              uint32_t* status) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  while (true) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (sm100::globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      raise_flag(status, kErrTimeout);
      return false;
    }
  }
}

// Min-heap of k keys for row r, stored at h[e * 128 + r]; replace the root
// by `key` (> root) and sift down.
__device__ __forceinline__ uint64_t heap_replace(uint64_t* h, int k, int r,
                                                 uint64_t key) {
  int p = 0;
#pragma unroll 1
  while (true) {
    int c = 2 * p + 1;
    if (c >= k) break;
    uint64_t cv = h[c * kTileRows + r];
    if (c + 1 < k) {
      const uint64_t c2 = h[(c + 1) * kTileRows + r];
      if (c2 < cv) {
        cv = c2;
        c = c + 1;
      }
    }
    if (cv >= key) break;
    h[p * kTileRows + r] = cv;
    p = c;
  }
  h[p * kTileRows + r] = key;
  return h[r];
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
prefill_score_topk_tc(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK, PrefillArgs a,
                      int cap) {
  using Lay = TcLayout<D>;
  constexpr int BN = Lay::BN, NS = Lay::NS, KB = Lay::KB;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + Lay::q_off;
  unsigned char* sK = smem + Lay::k_off;
  uint64_t* rbuf = reinterpret_cast<uint64_t*>(smem + Lay::buf_off);
  float* table = reinterpret_cast<float*>(smem + Lay::buf_off);  // pass-1 slots
  uint64_t* heap = reinterpret_cast<uint64_t*>(sK);  // K ring, free at the end
  __shared__ TcShared sh;

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = qt * Lay::BM;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = a.k;

  tile_rows(a, b, i0, sh.hi, &sh.maxhi);
  if (tid < kTileRows) {
    sh.cnt[tid] = 0;
    sh.ovf[tid] = 0;
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      sm100::mbar_init(&sh.kfull[s], 1);
      sm100::mbar_init(&sh.kempty[s], 1);
    }
    sm100::mbar_init(&sh.qfull, 1);
    for (int t = 0; t < 2; ++t) {
      sm100::mbar_init(&sh.tfull[t], 1);
      sm100::mbar_init(&sh.tempty[t], kSelWarps);
    }
    sh.abort = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(&sh.tmem, 256);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const int maxhi = sh.maxhi;
  const int T = maxhi >= 1 ? maxhi / BN + 1 : 0;  // key tiles with candidates
  const int TT = 2 * T;                           // two passes
  volatile int* abort_flag = &sh.abort;

  if (warp == 0) {
    // ---------------- TMA producer: key tiles 0..T-1, twice
    if (lane == 0 && T > 0) {
      sm100::prefetch_tmap(&tmQ);
      sm100::prefetch_tmap(&tmK);
      const int qrow = ((b * a.Hq + h) * a.n) + i0;
      const int krow = (b * a.Hkv + g) * a.n;
      sm100::mbar_arrive_expect_tx(&sh.qfull, Lay::kQBytes);
      for (int kb = 0; kb < KB; ++kb)
        sm100::tma_load_2d(sQ + kb * Lay::kBlockBytes, &tmQ, &sh.qfull, kb * 64,
                           qrow);
      int issued = 0;
      for (int t = 0; t < TT; ++t) {
        const int s = t % NS;
        const int tile = t < T ? t : t - T;
        if (t >= NS &&
            !wait_or_abort(&sh.kempty[s], ((t / NS) & 1) ^ 1, abort_flag,
                           a.status))
          break;
        sm100::mbar_arrive_expect_tx(&sh.kfull[s], Lay::kKBytes);
        unsigned char* dst = sK + (size_t)s * Lay::kKBytes;
        for (int kb = 0; kb < KB; ++kb)
          sm100::tma_load_2d(dst + kb * Lay::kBlockBytes, &tmK, &sh.kfull[s],
                             kb * 64, krow + tile * BN);
        issued = t + 1;
      }
      // Let every copy this thread started land before the CTA can exit.
      sm100::mbar_wait(&sh.qfull, 0, kWaitLimitNs);
      for (int t = issued - NS < 0 ? 0 : issued - NS; t < issued; ++t)
        sm100::mbar_wait(&sh.kfull[t % NS], (t / NS) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(Lay::BM, BN);
      const uint32_t aq = sm100::smem_u32(sQ);
      const uint32_t ak = sm100::smem_u32(sK);
      int done = 0;
      if (wait_or_abort(&sh.qfull, 0, abort_flag, a.status)) {
        for (int t = 0; t < TT; ++t) {
          const int s = t % NS, buf = t & 1;
          if (!wait_or_abort(&sh.kfull[s], (t / NS) & 1, abort_flag, a.status))
            break;
          if (t >= 2 && !wait_or_abort(&sh.tempty[buf], ((t >> 1) & 1) ^ 1,
                                       abort_flag, a.status))
            break;
          sm100::tc_fence_after();
          const uint32_t d_tmem = tmem + buf * BN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * Lay::kBlockBytes + (kk & 3) * 32;
            sm100::mma_bf16(d_tmem, sm100::desc_k_sw128(aq + off),
                            sm100::desc_k_sw128(ak + s * Lay::kKBytes + off),
                            idesc, kk > 0 ? 1u : 0u);
          }
          sm100::mma_commit(&sh.kempty[s]);
          sm100::mma_commit(&sh.tfull[buf]);
          done = t + 1;
        }
      }
      // The last commit covers every MMA issued: wait for it before exit.
      if (done > 0)
        sm100::mbar_wait(&sh.tfull[(done - 1) & 1], ((done - 1) >> 1) & 1,
                         kWaitLimitNs);
    }
  } else {
    // ---------------- selector warps: thread = query row, group = chunk
    const int sw = warp - 2;               // 0..15
    const int grp = sw >> 2;               // 32-column chunk of every tile
    const int quarter = warp & 3;          // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const int hi = sh.hi[r];
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + grp * 32;

    // ---- pass 1: slot maxima
    float colmax[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) colmax[x] = -INFINITY;
    int t = 0;
    for (; t < T; ++t) {
      const int buf = t & 1;
      if (!__all_sync(0xFFFFFFFFu, wait_or_abort(&sh.tfull[buf], (t >> 1) & 1,
                                                 abort_flag, a.status)))
        break;
      sm100::tc_fence_after();
      uint32_t raw[32];
      sm100::tmem_ld_32x32b_x32(tl + buf * BN, raw);
      sm100::tmem_wait_ld();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sh.tempty[buf]);
      const int j0 = t * BN + grp * 32;
      if (__all_sync(0xFFFFFFFFu, j0 >= 1 && j0 + 31 <= hi)) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          colmax[x] = fmaxf(colmax[x], __uint_as_float(raw[x]));
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (j0 + x >= 1 && j0 + x <= hi)
            colmax[x] = fmaxf(colmax[x], __uint_as_float(raw[x]));
      }
    }
    // ---- bound: k-th largest of the row's 128 slot maxima.  The table
    // row is stored with its 16-byte pieces XOR-swizzled by the row index so
    // that 32 rows written (or one row read) at once spread over the banks.
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int piece = (grp * 8 + c) ^ (r & 31);
      *reinterpret_cast<float4*>(table + r * 128 + piece * 4) =
          make_float4(colmax[4 * c], colmax[4 * c + 1], colmax[4 * c + 2],
                      colmax[4 * c + 3]);
    }
    SelBar::sync();
    for (int rr = 0; rr < 8; ++rr) {
      const int row = sw * 8 + rr;
      const int piece = lane ^ (row & 31);
      const float4 v = *reinterpret_cast<const float4*>(table + row * 128 +
                                                         piece * 4);
      uint32_t key[4] = {ord_f32(v.x), ord_f32(v.y), ord_f32(v.z),
                         ord_f32(v.w)};
      warp_bitonic<4>(key, lane);  // ascending over 128 slots
      const int e = 128 - k;       // the k-th largest
      const uint32_t kk = __shfl_sync(0xFFFFFFFFu, key[e >> 5], e & 31);
      if (lane == 0)
        sh.L[row] = (kk <= ord_f32(-INFINITY)) ? -INFINITY : unord_f32(kk);
    }
    SelBar::sync();
    const float Lr = sh.L[r];
    bool ovf_local = false;
    // ---- pass 2: append every candidate >= L
    for (; t < TT; ++t) {
      const int buf = t & 1;
      if (!__all_sync(0xFFFFFFFFu, wait_or_abort(&sh.tfull[buf], (t >> 1) & 1,
                                                 abort_flag, a.status)))
        break;
      sm100::tc_fence_after();
      uint32_t raw[32];
      sm100::tmem_ld_32x32b_x32(tl + buf * BN, raw);
      sm100::tmem_wait_ld();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sh.tempty[buf]);
      const int j0 = (t - T) * BN + grp * 32;
      // A score can only qualify if it reaches L; one warp vote per column
      // keeps the (rare) append off the common path.
      auto append = [&](uint32_t bits, int j) {
        const int pos = atomicAdd(&sh.cnt[r], 1);
        if (pos < cap)
          rbuf[(size_t)pos * kTileRows + r] = make_key(__uint_as_float(bits),
                                                       (uint32_t)j);
        else
          ovf_local = true;
      };
      if (__all_sync(0xFFFFFFFFu, j0 >= 1 && j0 + 31 <= hi)) {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const bool p = __uint_as_float(raw[x]) >= Lr;
          if (__any_sync(0xFFFFFFFFu, p)) {
            if (p) append(raw[x], j0 + x);
          }
        }
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const bool p = j0 + x >= 1 && j0 + x <= hi &&
                         __uint_as_float(raw[x]) >= Lr;
          if (__any_sync(0xFFFFFFFFu, p)) {
            if (p) append(raw[x], j0 + x);
          }
        }
      }
    }
    if (ovf_local) sh.ovf[r] = 1;
    SelBar::sync();
    // ---- exact Top-k of the row's buffer (one thread per row)
    if (grp == 0) {
      const int i = i0 + r;
      if (i < a.n && k > 0) {
        const size_t grow = (size_t)(b * a.Hq + h) * a.n + i;
        uint64_t* out = a.topk + grow * k;
        if (sh.ovf[r]) {
          // listed for the exact fallback pass; it writes this row
          const uint32_t pos = atomicAdd(a.ovf_count, 1u);
          a.ovf_rows[pos] = (uint32_t)grow;
        } else {
          for (int e = 0; e < k; ++e) heap[e * kTileRows + r] = 0ull;
          uint64_t root = 0ull;
          const int n = sh.cnt[r];
          for (int e = 0; e < n; ++e) {
            const uint64_t key = rbuf[(size_t)e * kTileRows + r];
            if (key > root) root = heap_replace(heap, k, r, key);
          }
          for (int e = 0; e < k; ++e) out[e] = heap[e * kTileRows + r];
        }
      }
    }
  }
  __syncwarp();  // reconverge single-lane roles before the CTA barrier
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 256);
  }
}

// Exact fallback for rows whose candidate buffer overflowed: one CTA per
// listed row scores every candidate on CUDA cores (fp32 FMA of the bf16 or
// fp32 inputs) and keeps the best k keys with the CTA radix select.
constexpr int kFbThreads = 256;
constexpr int kFbChunk = 2048;

template <typename T, int D>
__global__ void __launch_bounds__(kFbThreads)
prefill_overflow_rows(PrefillArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int k = a.k;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);      // [k + chunk]
  float* q = reinterpret_cast<float*>(keys + k + kFbChunk);  // [D]
  __shared__ int s_n, s_kk, s_w;
  __shared__ uint64_t s_T;
  __shared__ SelectState<1> st;
  const uint32_t nrows = *a.ovf_count;
  for (uint32_t it = blockIdx.x; it < nrows; it += gridDim.x) {
    const uint32_t grow = a.ovf_rows[it];
    const int i = (int)(grow % (uint32_t)a.n);
    const uint32_t bh = grow / (uint32_t)a.n;
    const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
    const int g = h / (a.Hq / a.Hkv);
    const int w = row_window(a.W_i, (int64_t)b * a.n + i, a.W, a.n, a.status,
                             false);
    const int hi = i - w;
    const T* Qr = reinterpret_cast<const T*>(a.Q) + (size_t)grow * D;
    const T* Kg = reinterpret_cast<const T*>(a.K) + ((size_t)b * a.Hkv + g) * a.n * D;
    for (int e = threadIdx.x; e < D; e += kFbThreads) q[e] = Elem<T>::load1(Qr + e);
    if (threadIdx.x == 0) s_n = 0;
    __syncthreads();
    for (int c0 = 1; c0 <= hi; c0 += kFbChunk) {
      for (int jj = threadIdx.x; jj < kFbChunk && c0 + jj <= hi; jj += kFbThreads) {
        const int j = c0 + jj;
        const T* kr = Kg + (size_t)j * D;
        float acc = 0.f;
        for (int e = 0; e < D; ++e) acc = fmaf(q[e], Elem<T>::load1(kr + e), acc);
        keys[s_n + jj] = make_key(acc, (uint32_t)j);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        s_n += (hi - c0 + 1 < kFbChunk) ? (hi - c0 + 1) : kFbChunk;
        s_kk = k;
      }
      __syncthreads();
      cta_select_thresholds<kFbThreads, 1>(keys, 0, &s_n, &s_kk, &s_T, &st,
                                           threadIdx.x);
      if (s_n > k) {
        // keep the keys >= T, packed to the front
        if (threadIdx.x == 0) s_w = 0;
        __syncthreads();
        uint64_t mine[(kPrefillMaxK + kFbChunk) / kFbThreads + 1];
        int cntm = 0;
        for (int e = threadIdx.x; e < s_n; e += kFbThreads) mine[cntm++] = keys[e];
        __syncthreads();
        for (int c = 0; c < cntm; ++c)
          if (mine[c] >= s_T) keys[atomicAdd(&s_w, 1)] = mine[c];
        __syncthreads();
        if (threadIdx.x == 0) s_n = k;
        __syncthreads();
      }
    }
    uint64_t* out = a.topk + (size_t)grow * k;
    for (int e = threadIdx.x; e < k; e += kFbThreads) out[e] = e < s_n ? keys[e] : 0ull;
    __syncthreads();
  }
}

// ============================================================ fp32 FFMA kernel
template <int D>
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
  const int i0 = qt * kTileRows;
  const int r = threadIdx.x, i = i0 + r;
  tile_rows(a, b, i0, s_hi, &s_maxhi);
  const int hi = s_hi[r];
  const int maxhi = s_maxhi;

  float q[D];
  const float* Qr = reinterpret_cast<const float*>(a.Q) +
                    ((size_t)(b * a.Hq + h) * a.n + (i < a.n ? i : 0)) * D;
#pragma unroll
  for (int e = 0; e < D; e += 4) {
    float4 v = *reinterpret_cast<const float4*>(Qr + e);
    q[e] = v.x; q[e + 1] = v.y; q[e + 2] = v.z; q[e + 3] = v.w;
  }
  const float* Kg = reinterpret_cast<const float*>(a.K) +
                    (size_t)(b * a.Hkv + g) * a.n * D;
  RowTopk sel;
  sel.init(heap, stage, r, a.k, S);
  const int T = maxhi >= 1 ? maxhi / TJ + 1 : 0;
  for (int t = 0; t < T; ++t) {
    __syncthreads();
    for (int e = threadIdx.x * 4; e < TJ * D; e += kTileRows * 4) {
      const int jj = t * TJ + e / D;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jj < a.n) v = *reinterpret_cast<const float4*>(Kg + (size_t)jj * D + e % D);
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
    const bool interior = (j0 >= 1) && (j0 + 31 <= hi);
    if (__all_sync(0xFFFFFFFFu, interior))
      sel.offer<false>(raw, j0, 1, hi);
    else
      sel.offer<true>(raw, j0, 1, hi);
  }
  sel.drain();
  if (i < a.n && a.k > 0)
    sel.store(a.topk + ((size_t)(b * a.Hq + h) * a.n + i) * a.k);
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

template <typename T, int D, typename TO, int NPL>
__global__ void __launch_bounds__(kGatherThreads)
prefill_gather(PrefillArgs a) {
  constexpr int LPR = 4;          // lanes per row in the softmax
  constexpr int RPW = 32 / LPR;   // rows per warp
  constexpr int DL = D / LPR;     // head dims per lane
  const int lane = threadIdx.x & 31;
  const int64_t wglob = ((int64_t)blockIdx.x * kGatherThreads + threadIdx.x) >> 5;
  const int64_t R = (int64_t)a.B * a.Hq * a.n;
  const int64_t row0 = wglob * RPW;
  if (row0 >= R) return;
  const int k = a.k;

  // ---- phase 1: one row at a time across the warp: sort, write C_i
#pragma unroll 1
  for (int rr = 0; rr < RPW; ++rr) {
    const int64_t row = row0 + rr;
    if (row >= R) break;
    const int64_t bh = row / a.n;
    const int i = (int)(row - bh * a.n);
    const int b = (int)(bh / a.Hq);
    const int w = row_window(a.W_i, (int64_t)b * a.n + i, a.W, a.n, a.status,
                             false);
    const int lo = i - w + 1 > 0 ? i - w + 1 : 0;
    const int anc = lo > 0 ? 1 : 0;
    uint32_t v[NPL];
    int m = 0;
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      const int e = t * 32 + lane;
      uint64_t key = 0ull;
      if (e < k) key = a.topk[row * k + e];
      v[t] = key ? key_index(key) : 0xFFFFFFFFu;
      m += __popc(__ballot_sync(0xFFFFFFFFu, key != 0ull));
    }
    warp_sort<NPL>(v, lane);
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

  // ---- phase 2: LPR lanes per row, fp32 online softmax over C_i
  const int sub = lane % LPR;
  const int64_t row = row0 + lane / LPR;
  const bool live = row < R;
  const int64_t rowc = live ? row : R - 1;
  const int64_t bh = rowc / a.n;
  const int i = (int)(rowc - bh * a.n);
  const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const int w = row_window(a.W_i, (int64_t)b * a.n + i, a.W, a.n, a.status,
                           false);
  const int lo = i - w + 1 > 0 ? i - w + 1 : 0;
  const T* qp = reinterpret_cast<const T*>(a.Q) + rowc * D + sub * DL;
  const T* Kg = reinterpret_cast<const T*>(a.K) +
                ((size_t)b * a.Hkv + g) * a.n * D + sub * DL;
  const T* Vg = reinterpret_cast<const T*>(a.V) +
                ((size_t)b * a.Hkv + g) * a.n * D + sub * DL;
  float qv[DL];
#pragma unroll
  for (int e = 0; e < DL; e += 4) load_f32<T, 4>(qp + e, qv + e);
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);
  float mx = -INFINITY, den = 0.f, o[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) o[e] = 0.f;

  auto accumulate = [&](float s_scaled, const T* vrow) {
    float vf[DL];
#pragma unroll
    for (int e = 0; e < DL; e += 4) load_f32<T, 4>(vrow + e, vf + e);
    const float mn = fmaxf(mx, s_scaled);
    const float corr = exp2f(mx - mn);
    const float p = exp2f(s_scaled - mn);
    den = den * corr + p;
#pragma unroll
    for (int e = 0; e < DL; ++e) o[e] = fmaf(p, vf[e], o[e] * corr);
    mx = mn;
  };

  // Top-k entries: scores come with the keys (the selector's fp32 values)
  const uint64_t* tk = a.topk + rowc * k;
#pragma unroll 1
  for (int e = 0; e < k; ++e) {
    const uint64_t key = live ? tk[e] : 0ull;
    if (key == 0ull) continue;
    const uint32_t j = key_index(key);
    if (j == 0 || (int)j > i - w) {  // never written by the selector
      raise_flag(a.status, kErrInternal);
      continue;
    }
    accumulate(key_score(key) * sl2, Vg + (size_t)j * D);
  }
  // anchor and window: scores computed here, 4 lanes per dot product
  const int nw = live ? (i - lo + 1) + (lo > 0 ? 1 : 0) : 0;
  int nmax = nw;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    nmax = max(nmax, __shfl_xor_sync(0xFFFFFFFFu, nmax, off));
#pragma unroll 1
  for (int t = 0; t < nmax; ++t) {
    const bool act = t < nw;
    int j = 0;
    if (lo > 0) j = (t == 0) ? 0 : lo + t - 1;
    else j = lo + t;
    if (!act) j = 0;
    float kf[DL];
#pragma unroll
    for (int e = 0; e < DL; e += 4) load_f32<T, 4>(Kg + (size_t)j * D + e, kf + e);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) dot = fmaf(qv[e], kf[e], dot);
    dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 1);
    dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 2);
    if (act) accumulate(dot * sl2, Vg + (size_t)j * D);
  }
  if (live) {
    TO* op = reinterpret_cast<TO*>(a.O) + rowc * D + sub * DL;
    const float inv = 1.f / den;
#pragma unroll
    for (int e = 0; e < DL; ++e) store_out<TO>(op + e, o[e] * inv);
  }
}

// ============================================================ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major [rows, d] bf16 tensor, boxes of 128 rows x 64 columns, 128-byte
// swizzle (matches the UMMA K-major SW128 descriptor).
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, int d) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_select_tc(const PrefillArgs& a, cudaStream_t s) {
  using Lay = TcLayout<D>;
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, a.Q, (uint64_t)a.B * a.Hq * a.n, D)) return cudaErrorInvalidValue;
  if (!make_tmap(&tk, a.K, (uint64_t)a.B * a.Hkv * a.n, D)) return cudaErrorInvalidValue;
  // row buffer: 3k candidates (the pass-1 bound leaves about 1.1-1.4 k),
  // at least kMinCap slots, at most what fits next to Q and the K ring
  const size_t budget = 227 * 1024 - sizeof(TcShared);
  const int cap_max = (int)((budget - Lay::bytes(0)) / (kTileRows * 8));
  int cap = 3 * a.k;
  if (cap < kMinCap) cap = kMinCap;
  if (cap > cap_max) cap = cap_max;
  if (cap < a.k || cap < kMinCap) return cudaErrorNotSupported;
  const size_t smem = Lay::bytes(cap);
  auto kern = prefill_score_topk_tc<D>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.n + 127) / 128, a.Hq, a.B);
  prof_before(s, "prefill_score_topk_tc");
  kern<<<grid, kTcThreads, smem, s>>>(tq, tk, a, cap);
  prof_after(s);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // rows whose buffer overflowed (none on typical inputs): exact fallback
  const size_t fb_smem = (size_t)(a.k + kFbChunk) * 8 + D * 4;
  prof_before(s, "prefill_overflow_rows");
  prefill_overflow_rows<__nv_bfloat16, D><<<148, kFbThreads, fb_smem, s>>>(a);
  prof_after(s);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_select_f32(const PrefillArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)32 * D * 4 + (size_t)a.k * kTileRows * 8 +
                      (size_t)32 * kTileRows * 8;
  auto kern = prefill_score_topk_f32<D>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.n + 127) / 128, a.Hq, a.B);
  prof_before(s, "prefill_score_topk_f32");
  kern<<<grid, kTileRows, smem, s>>>(a);
  prof_after(s);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_gather(const PrefillArgs& a, cudaStream_t s) {
  const int64_t R = (int64_t)a.B * a.Hq * a.n;
  const int64_t warps = (R + 7) / 8;
  const int64_t blocks = (warps * 32 + kGatherThreads - 1) / kGatherThreads;
  dim3 grid((unsigned)blocks);
  prof_before(s, "prefill_gather");
  if (a.k <= 32) {
    if (a.o_bf16) prefill_gather<T, D, __nv_bfloat16, 1><<<grid, kGatherThreads, 0, s>>>(a);
    else prefill_gather<T, D, float, 1><<<grid, kGatherThreads, 0, s>>>(a);
  } else {
    if (a.o_bf16) prefill_gather<T, D, __nv_bfloat16, 2><<<grid, kGatherThreads, 0, s>>>(a);
    else prefill_gather<T, D, float, 2><<<grid, kGatherThreads, 0, s>>>(a);
  }
  prof_after(s);
  return cudaGetLastError();
}

}  // namespace

size_t prefill_topk_bytes(int B, int n, int Hq, int k) {
  size_t bytes = (size_t)B * Hq * n * (size_t)(k > 0 ? k : 1) * 8;
  return (bytes + 255) / 256 * 256;
}

size_t prefill_workspace(bool, int B, int n, int Hq, int, int, int k) {
  // per-row Top-k keys, then the list of rows for the exact fallback
  return prefill_topk_bytes(B, n, Hq, k) +
         ((size_t)B * Hq * n * 4 + 255) / 256 * 256;
}

cudaError_t prefill_launch(const PrefillArgs& a, bool bf16, int d,
                           cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (a.k > 0) {
    if (bf16) e = d == 64 ? launch_select_tc<64>(a, s) : launch_select_tc<128>(a, s);
    else e = d == 64 ? launch_select_f32<64>(a, s) : launch_select_f32<128>(a, s);
    if (e != cudaSuccess) return e;
  }
  if (bf16) e = d == 64 ? launch_gather<__nv_bfloat16, 64>(a, s)
                        : launch_gather<__nv_bfloat16, 128>(a, s);
  else e = d == 64 ? launch_gather<float, 64>(a, s) : launch_gather<float, 128>(a, s);
  return e;
}

}  // namespace ca

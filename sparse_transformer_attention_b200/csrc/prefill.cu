// Prefill path: causal Condensate attention over n positions.
// "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质", §2.1 Definition 1,
// §2.2.1-§2.2.3, §2.4 Corollaries 2-3, §5.2.2 (identify the set, then attend
// on the subset).
//
// Launch 1 (score + select), one CTA per 128-query tile of one (batch, head):
//   bf16: warp-specialised tcgen05 pipeline.  Warp 0 issues TMA loads of the
//         Q tile (once) and of 128-key K tiles into a ring of shared-memory
//         stages, twice over (two passes); warp 1 issues tcgen05.mma (M=128,
//         N=128, K=16 steps, bf16 in, fp32 out) into four TMEM accumulators;
//         sixteen selector warps read the scores back with tcgen05.ld (thread
//         = query row x 32-column chunk group).  Pass 1 keeps 128 column-slot
//         maxima per row, whose k-th largest bounds the row's k-th best score
//         from below; pass 2 appends every candidate at or above the bound to
//         the thread's shared-memory segment; the exact Top-k is then cut per
//         row.  Only key tiles that hold candidates of some row of the tile
//         are computed, and the score matrix never leaves the SM.  Rows whose
//         segments overflow go to an exact CUDA-core fallback.
//   fp32: a per-row heap selector fed by an FFMA dot-product loop over
//         32-key tiles staged in shared memory (no TF32, so selection stays
//         exact).
// Launch 2 (gather + softmax): per row, sort the selected positions, write
//   C_i (ascending) and |C_i|, and run an fp32 online softmax over
//   {0} U Top-k U window, re-using the selector's fp32 scores for Top-k.
//   bf16 runs the window on warp-level MMA, 16 query rows per warp.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.cuh"
#include "prefill.cuh"
#include "profile.cuh"
#include "row_topk.cuh"
#include "select.cuh"
#include "sm100.cuh"
#include "warp_sort.cuh"

namespace ca {

namespace {

// ------------------------------------------------------------ shared prologue
// Window and last candidate position of each row of the tile (query rows
// r0 .. r0+127 of head h, at positions p0 + r); returns the largest
// last-candidate position over the tile's rows (-1 if none).
__device__ void tile_rows(const PrefillArgs& a, int b, int h, int r0,
                          int* s_hi, int* s_maxhi) {
  const int tid = threadIdx.x;
  if (tid == 0) *s_maxhi = -1;
  __syncthreads();
  if (tid < kTileRows) {
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

// ============================================================ tcgen05 kernel
// Two passes over the row tile's key tiles (the tensor pipe has room for
// them; the selector is what costs):
//   pass 1: every selector thread keeps, for its query row, the maximum over
//           each of 32 column positions of its 32-column chunk of every key
//           tile (128 slots per row over the four chunk groups).  The k-th
//           largest slot maximum L is a lower bound of the row's k-th best
//           score: the top k slots are k distinct candidates, all >= L.
//   pass 2: recompute the scores and append every candidate with score >= L
//           to the thread's own segment (about 1.1-1.4 k entries per row on
//           random data), with predicated stores and no atomics.
// The exact Top-k is then found per row by one warp (bisection on the key
// bits over the row's four segments).  A row whose segment would overflow is
// listed for an exact CUDA-core fallback.
constexpr int kSelWarps = 16;                       // 4 chunk groups x 4 quarters
constexpr int kSelThreads = 32 * kSelWarps;         // (row, chunk group) pairs
constexpr int kTcThreads = 64 + kSelThreads;        // + TMA warp + MMA warp
constexpr int kTmemBufs = 4;                        // 128-column accumulators
constexpr int kMinSeg = 16;                         // smallest segment (entries)
constexpr int kPoolCols = 16;                       // spare segments per CTA
constexpr int kSegCols = kSelThreads + kPoolCols;   // segment columns
constexpr int kScoreStride = (kSegCols + 1) * 4;    // bytes between positions
constexpr int kCodeStride = (kSegCols + 2) * 2;     // (odd word strides: the
                                                    //  entries of one column
                                                    //  spread over the banks)
constexpr uint32_t kMaskedScore = 0x7FC00000u;      // NaN: never >= L, ignored
                                                    // by fmaxf
using SelBar = GroupBarrier<1, kSelThreads>;

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
  static constexpr size_t seg_off = k_off + (size_t)NS * kKBytes;
  // Segments: P positions of scores (u32) then of codes (u16); the pass-1
  // slot table (128 rows x 128 fp32) uses the same bytes first.
  __host__ __device__ static size_t code_off(int P) {
    return seg_off + ((size_t)P * kScoreStride + 15) / 16 * 16;
  }
  __host__ __device__ static size_t bytes(int P) {
    size_t seg = code_off(P) - seg_off + (size_t)P * kCodeStride;
    if (seg < (size_t)kTileRows * 128 * 4) seg = (size_t)kTileRows * 128 * 4;
    return seg_off + seg + 1024;  // + the manual 1024-byte alignment
  }
};

struct TcShared {
  uint64_t kfull[4], kempty[4], qfull, tfull[kTmemBufs], tempty[kTmemBufs];
  uint64_t never;  // failure-path test hook: a barrier nothing signals
  uint32_t tmem;
  int abort;
  int maxhi;
  int hi[kTileRows];
  float L[kTileRows];
  float M[kTileRows];       // row maximum over the candidates (mass reports)
  short cnt[kSelThreads];   // entries in the thread's own segment, -1: overflow
  short xcnt[kSelThreads];  // entries in its spare segment
  signed char xcol[kSelThreads];  // spare segment index, -1: none
  int pool;                 // spare segments handed out
};

// Append (score, code) at the segment cursor when score >= L; predicated
// stores, so a warp never branches on the comparison.
__device__ __forceinline__ void seg_append(uint32_t& as, uint32_t& ac,
                                           uint32_t bits, float L,
                                           uint32_t code) {
  asm volatile(
      "{ .reg .pred p; .reg .b16 c;\n\t"
      "setp.ge.f32 p, %2, %3;\n\t"
      "cvt.u16.u32 c, %5;\n\t"
      "@p st.shared.b32 [%0], %4;\n\t"
      "@p st.shared.b16 [%1], c;\n\t"
      "@p add.u32 %0, %0, %6;\n\t"
      "@p add.u32 %1, %1, %7; }"
      : "+r"(as), "+r"(ac)
      : "f"(__uint_as_float(bits)), "f"(L), "r"(bits), "r"(code),
        "n"(kScoreStride), "n"(kCodeStride)
      : "memory");
}

// Append the 32 scores of one key tile chunk.  Cursors are checked every 8
// columns: a cursor past `*_max` (8 positions before the end) is clamped
// and `full` is set, and the caller redoes the tile elsewhere.
__device__ __forceinline__ void append_tile(const uint32_t (&raw)[32],
                                            uint32_t& as, uint32_t& ac,
                                            float L, uint32_t cbase,
                                            uint32_t as_max, uint32_t ac_max,
                                            bool& full) {
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    seg_append(as, ac, raw[x], L, cbase + x);
    if ((x & 7) == 7) {
      full |= as > as_max;
      as = min(as, as_max);
      ac = min(ac, ac_max);
    }
  }
}

// Segments of one row: slot g < 4 is chunk group g's own segment (column
// g * 128 + row), slot 4 + g its spare one (column 512 + spare index, empty
// when there is none).  Entry f lives in the last slot s with start[s] <= f
// (empty slots share the start of the next one).
struct RowSegs {
  int n;           // entries of the row
  int row;         // row within the tile
  int start[8];    // prefix of the slot counts
  int xcolm[4];    // spare segment column of each group
  bool bad;        // a segment overflowed
};

__device__ __forceinline__ void row_segs(const TcShared& sh, int row,
                                         RowSegs& q) {
  q.row = row;
  q.n = 0;
  q.bad = false;
#pragma unroll
  for (int gq = 0; gq < 4; ++gq) {
    const int c = sh.cnt[gq * kTileRows + row];
    q.bad |= c < 0;
    q.start[gq] = q.n;
    q.n += c < 0 ? 0 : c;
  }
#pragma unroll
  for (int gq = 0; gq < 4; ++gq) {
    const int x = sh.xcol[gq * kTileRows + row];
    q.start[4 + gq] = q.n;
    q.xcolm[gq] = kSelThreads + (x < 0 ? 0 : x);
    if (x >= 0) q.n += sh.xcnt[gq * kTileRows + row];
  }
}

__device__ __forceinline__ void seg_locate(const RowSegs& rs, int f, int& col,
                                           int& grp, int& e) {
  int s = 0;
#pragma unroll
  for (int q = 1; q < 8; ++q) s += f >= rs.start[q];
  int st = rs.start[0];
#pragma unroll
  for (int q = 1; q < 8; ++q)
    if (q == s) st = rs.start[q];
  int xcol = rs.xcolm[0];
#pragma unroll
  for (int q = 1; q < 4; ++q)
    if (q == (s & 3)) xcol = rs.xcolm[q];
  grp = s & 3;
  col = s < 4 ? grp * kTileRows + rs.row : xcol;
  e = f - st;
}

__device__ __forceinline__ uint32_t seg_hi(const unsigned char* seg, int col,
                                           int e) {
  const uint32_t bits = *reinterpret_cast<const uint32_t*>(
      seg + (size_t)e * kScoreStride + col * 4);
  return ord_f32(__uint_as_float(bits));
}

__device__ __forceinline__ uint32_t seg_lo(const unsigned char* codes,
                                           int col, int grp, int e) {
  const uint32_t code = *reinterpret_cast<const uint16_t*>(
      codes + (size_t)e * kCodeStride + col * 2);
  const uint32_t j = (code >> 5) * 128 + grp * 32 + (code & 31);
  return 0xFFFFFFFFu - j;
}

// Sum over the four lanes of a row group.
__device__ __forceinline__ int quad_sum(int v) {
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
  return v + __shfl_xor_sync(0xFFFFFFFFu, v, 2);
}

// Exact Top-k of the rows of one warp, four lanes per row (lane & 3 = part;
// entry f of the row is held by part f & 3).  `sel` rows take the k largest
// keys (ord(score), ~j) of their n entries, found by bisection on the score
// bits (and on the index bits only when equal scores straddle the cut);
// `all` rows (n <= k) take every entry.  The selected keys go to out[0..) in
// any order, padded with empty keys.  Missing entries hold 0, below every
// probe.
template <int NE>
__device__ __forceinline__ void quad_select(const unsigned char* seg,
                                            const unsigned char* codes,
                                            const RowSegs& rs, bool live,
                                            uint32_t lob, int k, int kpad,
                                            uint64_t* out, int part) {
  uint32_t hv[NE];
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    const int f = part + 4 * t;
    hv[t] = 0u;
    if (live && f < rs.n) {
      int col, grp, e;
      seg_locate(rs, f, col, grp, e);
      hv[t] = seg_hi(seg, col, e);
    }
  }
  const bool sel = live && rs.n > k;
  // bisection start: the common high bits of the bound and the row maximum
  uint32_t mx = 0u;
#pragma unroll
  for (int t = 0; t < NE; ++t) mx = max(mx, hv[t]);
  mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  const uint32_t diff = lob ^ mx;
  const int nb = sel ? (diff ? 32 - __clz(diff) : 0) : 0;
  uint32_t tau = nb == 32 ? 0u : (lob >> nb) << nb;
  bool done = nb == 0, exact = false;
  const int bmax = __reduce_max_sync(0xFFFFFFFFu, nb);
#pragma unroll 1
  for (int b = bmax - 1; b >= 0; --b) {
    if (__all_sync(0xFFFFFFFFu, done)) break;
    const uint32_t c = tau | (1u << b);
    int m = 0;
#pragma unroll
    for (int t = 0; t < NE; ++t) m += hv[t] >= c;
    m = quad_sum(m);
    const bool up = !done && b < nb && m >= k;
    tau = up ? c : tau;
    const bool fin = up && m == k;
    done |= fin;
    exact |= fin;
  }
  uint32_t th_hi = sel ? tau : 0u, th_lo = 0u;
  // equal scores straddling the cut: the lower positions win
  int gt = 0, ge = 0;
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    gt += hv[t] > th_hi;
    ge += hv[t] >= th_hi;
  }
  gt = quad_sum(gt);
  ge = quad_sum(ge);
  const int need = (sel && !exact && ge > k) ? k - gt : 0;
  if (__any_sync(0xFFFFFFFFu, need > 0)) {
    uint32_t lo[NE];
#pragma unroll
    for (int t = 0; t < NE; ++t) {
      const int f = part + 4 * t;
      lo[t] = 0u;
      if (need > 0 && f < rs.n && hv[t] == th_hi) {
        int col, grp, e;
        seg_locate(rs, f, col, grp, e);
        lo[t] = seg_lo(codes, col, grp, e);
      }
    }
#pragma unroll 1
    for (int b = 31; b >= 0; --b) {
      const uint32_t c = th_lo | (1u << b);
      int m = 0;
#pragma unroll
      for (int t = 0; t < NE; ++t) m += hv[t] == th_hi && lo[t] >= c;
      m = quad_sum(m);
      th_lo = (need > 0 && m >= need) ? c : th_lo;
    }
  }
  // write the selected keys: exclusive prefix over the four parts
  int cnt = 0;
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    const int f = part + 4 * t;
    if (live && f < rs.n && hv[t] >= th_hi) {
      bool s = hv[t] > th_hi || th_lo == 0u;
      if (!s) {
        int col, grp, e;
        seg_locate(rs, f, col, grp, e);
        s = seg_lo(codes, col, grp, e) >= th_lo;
      }
      cnt += s;
    }
  }
  const int up1 = __shfl_up_sync(0xFFFFFFFFu, cnt, 1);
  const int up2 = __shfl_up_sync(0xFFFFFFFFu, cnt, 2);
  const int up3 = __shfl_up_sync(0xFFFFFFFFu, cnt, 3);
  const int pre =
      (part >= 1 ? up1 : 0) + (part >= 2 ? up2 : 0) + (part >= 3 ? up3 : 0);
  const int total = quad_sum(cnt);
  if (live) {
    int pos = pre;
#pragma unroll
    for (int t = 0; t < NE; ++t) {
      const int f = part + 4 * t;
      if (f < rs.n && hv[t] >= th_hi) {
        int col, grp, e;
        seg_locate(rs, f, col, grp, e);
        const uint32_t lo = seg_lo(codes, col, grp, e);
        if (hv[t] > th_hi || lo >= th_lo) {
          out[pos++] = ((uint64_t)hv[t] << 32) | lo;
        }
      }
    }
    for (int e = total + part; e < kpad; e += 4) out[e] = 0ull;
  }
}

template <int D, bool MASS>
__global__ void __launch_bounds__(kTcThreads, 1)
prefill_score_topk_tc(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK, PrefillArgs a,
                      int P) {
  using Lay = TcLayout<D>;
  constexpr int BN = Lay::BN, NS = Lay::NS, KB = Lay::KB;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + Lay::q_off;
  unsigned char* sK = smem + Lay::k_off;
  unsigned char* seg = smem + Lay::seg_off;     // scores [P][512] (stride 513)
  unsigned char* codes = smem + Lay::code_off(P);  // codes [P][512] (514)
  float* table = reinterpret_cast<float*>(seg);  // pass-1 slots, then free
  __shared__ TcShared sh;

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = qt * Lay::BM;  // first query row of the tile
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = head_k(a.k_h, h, a.k, a.status, qt == 0 && tid == 0);

  tile_rows(a, b, h, i0, sh.hi, &sh.maxhi);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      sm100::mbar_init(&sh.kfull[s], 1);
      sm100::mbar_init(&sh.kempty[s], 1);
    }
    sm100::mbar_init(&sh.qfull, 1);
    sm100::mbar_init(&sh.never, 1);
    for (int t = 0; t < kTmemBufs; ++t) {
      sm100::mbar_init(&sh.tfull[t], 1);
      sm100::mbar_init(&sh.tempty[t], kSelWarps);
    }
    sh.abort = 0;
    sh.pool = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(&sh.tmem, kTmemBufs * BN);
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
      const int qrow = ((b * a.Hq + h) * a.nq) + i0;
      const int krow = (b * a.Hkv + g) * a.L;
      sm100::mbar_arrive_expect_tx(&sh.qfull, Lay::kQBytes);
      for (int kb = 0; kb < KB; ++kb)
        sm100::tma_load_2d(sQ + kb * Lay::kBlockBytes, &tmQ, &sh.qfull, kb * 64,
                           qrow);
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;
      for (int t = 0; t < TT; ++t) {
        const int tile = t < T ? t : t - T;
        if (t >= NS &&
            !sm100::wait_or_abort(&sh.kempty[s], ph ^ 1, abort_flag, a.status,
                                   a.wait_ns))
          break;
        sm100::mbar_arrive_expect_tx(&sh.kfull[s], Lay::kKBytes);
        unsigned char* dst = sK + (size_t)s * Lay::kKBytes;
        for (int kb = 0; kb < KB; ++kb)
          sm100::tma_load_2d(dst + kb * Lay::kBlockBytes, &tmK, &sh.kfull[s],
                             kb * 64, krow + tile * BN);
        issued = t + 1;
        if (++s == NS) {
          s = 0;
          ph ^= 1;
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      bool drained = sm100::mbar_wait(&sh.qfull, 0, kDrainWaitNs);
      for (int t = issued - NS < 0 ? 0 : issued - NS; t < issued; ++t)
        drained &= sm100::mbar_wait(&sh.kfull[t % NS], (t / NS) & 1,
                                    kDrainWaitNs);
      if (!drained) raise_flag(a.status, kErrTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(Lay::BM, BN);
      const uint32_t aq = sm100::smem_u32(sQ);
      const uint32_t ak = sm100::smem_u32(sK);
      int done = 0;
      if (a.stall_ns) {
        // Failure-path test hook: wait on a barrier that nothing signals, so
        // the wait runs out, raises the time-out flag and aborts every wait
        // of the CTA; the kernel then leaves through its normal path.
        sm100::wait_or_abort(&sh.never, 0, abort_flag, a.status, a.stall_ns);
      }
      if (sm100::wait_or_abort(&sh.qfull, 0, abort_flag, a.status, a.wait_ns)) {
        int s = 0;
        uint32_t ph = 0;
        for (int t = 0; t < TT; ++t) {
          const int buf = t & (kTmemBufs - 1);
          if (!sm100::wait_or_abort(&sh.kfull[s], ph, abort_flag, a.status,
                                    a.wait_ns))
            break;
          if (t >= kTmemBufs &&
              !sm100::wait_or_abort(&sh.tempty[buf], ((t / kTmemBufs) & 1) ^ 1,
                                    abort_flag, a.status, a.wait_ns))
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
          if (++s == NS) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // The last commit covers every MMA issued: wait for it before exit.
      if (done > 0 &&
          !sm100::mbar_wait(&sh.tfull[(done - 1) & (kTmemBufs - 1)],
                            ((done - 1) / kTmemBufs) & 1, kDrainWaitNs))
        raise_flag(a.status, kErrTimeout);
    }
  } else {
    // ---------------- selector warps: thread = (query row, chunk group)
    const int sw = warp - 2;               // 0..15
    const int grp = sw >> 2;               // 32-column chunk of every tile
    const int quarter = warp & 3;          // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const int col = grp * kTileRows + r;   // this thread's segment column
    const int hi = sh.hi[r];
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + grp * 32;

    // Scores of key tile t for this thread's row and chunk, with
    // non-candidates (j = 0, the window, the future) replaced by NaN.
    auto fetch = [&](int t, uint32_t (&raw)[32]) -> bool {
      const int buf = t & (kTmemBufs - 1);
      if (!__all_sync(0xFFFFFFFFu,
                      sm100::wait_or_abort(&sh.tfull[buf], (t / kTmemBufs) & 1,
                                           abort_flag, a.status, a.wait_ns)))
        return false;
      sm100::tc_fence_after();
      sm100::tmem_ld_32x32b_x32(tl + buf * BN, raw);
      sm100::tmem_wait_ld();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sh.tempty[buf]);
      return true;
    };

    // ---- pass 1: slot maxima
    float colmax[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) colmax[x] = -INFINITY;
    int t = 0;
    for (; t < T; ++t) {
      uint32_t raw[32];
      if (!fetch(t, raw)) break;
      const int j0 = t * BN + grp * 32;
      if (!(j0 >= 1 && j0 + 31 <= hi)) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (!(j0 + x >= 1 && j0 + x <= hi)) raw[x] = kMaskedScore;
      }
#pragma unroll
      for (int x = 0; x < 32; ++x)
        colmax[x] = fmaxf(colmax[x], __uint_as_float(raw[x]));
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
    {
      // Four lanes per row (part = slots part*32 .. part*32+31), eight rows
      // per warp.  tau is the largest value with its low 14 bits zero and at
      // least k slots >= tau (or the first probe that leaves exactly k); any
      // such tau is a valid bound.
      const int row = sw * 8 + (lane >> 2), part = lane & 3;
      uint32_t key[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int piece = (part * 8 + c) ^ (row & 31);
        const float4 v = *reinterpret_cast<const float4*>(table + row * 128 +
                                                           piece * 4);
        key[4 * c] = ord_f32(v.x);
        key[4 * c + 1] = ord_f32(v.y);
        key[4 * c + 2] = ord_f32(v.z);
        key[4 * c + 3] = ord_f32(v.w);
      }
      uint32_t tau = 0u;
      bool done = false;
#pragma unroll 1
      for (int bit = 31; bit >= 14; --bit) {
        const uint32_t c = tau | (1u << bit);
        int m = 0;
#pragma unroll
        for (int x = 0; x < 32; ++x) m += key[x] >= c;
        m = quad_sum(m);
        const bool up = !done && m >= k;
        tau = up ? c : tau;
        done |= up && m == k;
        if (__all_sync(0xFFFFFFFFu, done)) break;
      }
      if (part == 0)
        sh.L[row] = k == 0 ? INFINITY  // nothing to select: no appends
                    : (tau <= ord_f32(-INFINITY)) ? -INFINITY
                                                  : unord_f32(tau);
      if constexpr (MASS) {
        uint32_t mx = 0u;
#pragma unroll
        for (int x = 0; x < 32; ++x) mx = max(mx, key[x]);
        mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
        mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
        if (part == 0) sh.M[row] = unord_f32(mx);
      }
    }
    SelBar::sync();
    const float Lr = sh.L[r];
    const float sl2 = 1.4426950408889634f / sqrtf((float)D);
    const float Mr = MASS ? sh.M[r] : 0.f;
    float xs = 0.f;  // this thread's share of the candidates' sum
    // ---- pass 2: append every candidate >= L to this thread's segment; a
    // full segment continues in a spare one (rare), else the row is listed
    // for the exact fallback.
    const uint32_t seg_s = sm100::smem_u32(seg), seg_c = sm100::smem_u32(codes);
    uint32_t as0 = seg_s + col * 4, ac0 = seg_c + col * 2;
    // cursors are checked every 8 columns so that 8 more entries still fit
    uint32_t as_max = as0 + (uint32_t)(P - 8) * kScoreStride;
    uint32_t ac_max = ac0 + (uint32_t)(P - 8) * kCodeStride;
    uint32_t as = as0, ac = ac0;
    int xc = -1, own = 0;
    bool ovf = false;
    for (; t < TT; ++t) {
      uint32_t raw[32];
      if (!fetch(t, raw)) break;
      const int tile = t - T;
      const int j0 = tile * BN + grp * 32;
      if (!(j0 >= 1 && j0 + 31 <= hi)) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (!(j0 + x >= 1 && j0 + x <= hi)) raw[x] = kMaskedScore;
      }
      if constexpr (MASS) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          xs += exp2f(fmaxf((__uint_as_float(raw[x]) - Mr) * sl2, -INFINITY));
      }
      const uint32_t cbase = (uint32_t)tile * 32;
      const uint32_t as_t = as;  // cursor at the tile start
      bool full = false;
      append_tile(raw, as, ac, Lr, cbase, as_max, ac_max, full);
      if (__any_sync(0xFFFFFFFFu, full)) {
        // An own segment is full: drop this tile's entries from it and redo
        // the tile in a spare segment (once per thread, while any is left);
        // otherwise the row goes to the exact fallback.  The whole warp runs
        // the redo; threads with nothing to redo append nothing (L = +inf).
        float Lredo = INFINITY;
        if (full) {
          const int px = (xc < 0 && !ovf) ? atomicAdd(&sh.pool, 1) : kPoolCols;
          if (px < kPoolCols) {
            own = (as_t - as0) / kScoreStride;
            xc = px;
            as0 = seg_s + (kSelThreads + px) * 4;
            ac0 = seg_c + (kSelThreads + px) * 2;
            as_max = as0 + (uint32_t)(P - 8) * kScoreStride;
            ac_max = ac0 + (uint32_t)(P - 8) * kCodeStride;
            as = as0;
            ac = ac0;
            Lredo = Lr;
          } else {
            ovf = true;
          }
        }
        bool full2 = false;
        append_tile(raw, as, ac, Lredo, cbase, as_max, ac_max, full2);
        ovf |= full2;
      }
    }
    const int last = (as - as0) / kScoreStride;
    sh.cnt[col] = ovf ? (short)-1 : (short)(xc < 0 ? last : own);
    sh.xcnt[col] = (short)(xc < 0 ? 0 : last);
    sh.xcol[col] = (signed char)xc;
    // per thread: sum of 2^((s - M) log2e/sqrt(d)) over its candidates, in
    // the Q tile's bytes (every MMA reading them has completed: this
    // thread consumed the last accumulator)
    float* xsum = reinterpret_cast<float*>(sQ);
    if constexpr (MASS) xsum[col] = xs;
    SelBar::sync();
    // ---- exact Top-k per row: four lanes per row, eight rows per warp
    {
      const int row = sw * 8 + (lane >> 2), part = lane & 3;
      const int r = i0 + row;
      RowSegs rs;
      row_segs(sh, row, rs);
      const size_t grow = (size_t)(b * a.Hq + h) * a.nq + r;
      bool live = r < a.nq;
      if (live && (rs.bad || rs.n > 128)) {
        // listed for the exact fallback pass; it writes this row
        if (part == 0) {
          const uint32_t pos = atomicAdd(a.ovf_count, 1u);
          a.ovf_rows[pos] = (uint32_t)grow;
        }
        live = false;
      }
      if constexpr (MASS) {
        float t = reinterpret_cast<const float*>(sQ)[part * kTileRows + row];
        t += __shfl_xor_sync(0xFFFFFFFFu, t, 1);
        t += __shfl_xor_sync(0xFFFFFFFFu, t, 2);
        if (r < a.nq && part == 0)
          a.cand_ml[grow] = make_float2(sh.M[row] * sl2, t);
      }
      const uint32_t lob = ord_f32(sh.L[row]);
      uint64_t* out = a.topk + grow * a.k;
      if (__all_sync(0xFFFFFFFFu, !live || rs.n <= 64))
        quad_select<16>(seg, codes, rs, live, lob, k, a.k, out, part);
      else
        quad_select<32>(seg, codes, rs, live, lob, k, a.k, out, part);
    }
  }
  __syncwarp();  // reconverge single-lane roles before the CTA barrier
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemBufs * BN);
  }
}

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
constexpr int kFbThreads = 256;
constexpr int kFbChunk = 2048;
constexpr int kFbBuf = 2 * kFbChunk;  // buffered keys beyond k

template <typename T, int D>
__global__ void __launch_bounds__(kFbThreads)
prefill_overflow_rows(PrefillArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int k = a.k;
  const int lane = threadIdx.x & 31;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem);      // [k + kFbBuf]
  float* q = reinterpret_cast<float*>(keys + k + kFbBuf);  // [D]
  __shared__ int s_n, s_kk, s_w;
  __shared__ uint64_t s_T;
  __shared__ SelectState<1> st;
  const uint32_t nrows = *a.ovf_count;
  for (uint32_t it = blockIdx.x; it < nrows; it += gridDim.x) {
    const uint32_t grow = a.ovf_rows[it];
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
          // the key row in 16-byte pieces, all loads issued before the FMAs
          RawRow<T, D> kr;
          kr.load(Kg + (size_t)j * D);
          float kf[D];
          kr.to_f32(kf);
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int e = 0; e < D; e += 2) {
            a0 = fmaf(q[e], kf[e], a0);
            a1 = fmaf(q[e + 1], kf[e + 1], a1);
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
__device__ __forceinline__ uint32_t bf16_bits_as_f32(const __nv_bfloat16* p) {
  return (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p)) << 16;
}

constexpr int kMmaWarps = 4;  // 16 query rows each

// Per warp: the window state (o, max, sum) of its 16 rows, then their Top-k
// keys as loaded in step 1.
template <int D>
struct MmaGatherSmem {
  static constexpr size_t state = (size_t)16 * D * 4 + 3 * 16 * 4;
  __host__ __device__ static size_t per_warp(int k) {
    return state + (size_t)16 * k * 8;
  }
  __host__ __device__ static size_t bytes(int k) { return kMmaWarps * per_warp(k); }
};

// bf16 gather with the window on tensor cores.  A warp owns 16 consecutive
// query rows of one (batch, head).
//   1. The Top-k keys of its rows into shared memory in one batch of loads,
//      then C_i and |C_i| for each row (whole warp per row).
//   2. The window [lo_i, i] of all 16 rows: MMA scores, masked per row, an
//      online softmax per row over 16-key blocks, and the MMA p * V.  The
//      state (max, sum, unnormalised o) goes to shared memory.
//   3. Eight lanes per row, four rows at a time: start from the window state
//      and fold in the Top-k keys (scores from the selector) and the anchor
//      (score computed here), then write the output row.
template <int D, typename TO, int NPL, bool MASS>
__global__ void __launch_bounds__(kMmaWarps * 32)
prefill_gather_mma(PrefillArgs a) {
  using T = __nv_bfloat16;
  constexpr int KS = D / 16;  // k-steps of the score MMA
  constexpr int NT = D / 8;   // head-dim tiles of the p * V MMA
  extern __shared__ __align__(16) unsigned char g_smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  // query rows r at positions p0 + r, keys 0..L-1
  const int nq = a.nq, L = a.L, p0 = a.p0, k = a.k;
  float* s_o = reinterpret_cast<float*>(g_smem + wid * MmaGatherSmem<D>::per_warp(k));
  float* s_m = s_o + 16 * D;
  float* s_l = s_m + 16;
  float* s_lx = s_l + 16;  // window sums of the unrounded weights (reports)
  uint64_t* s_key = reinterpret_cast<uint64_t*>(s_lx + 16);  // [16][k]
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = (blockIdx.x * kMmaWarps + wid) * 16;  // first query row
  if (i0 >= nq) return;  // the whole warp
  const int64_t rowbase = (int64_t)bh * nq;
  const T* Qg = reinterpret_cast<const T*>(a.Q) + rowbase * D;
  const T* Kg = reinterpret_cast<const T*>(a.K) + ((size_t)b * a.Hkv + g) * (size_t)L * D;
  const T* Vg = reinterpret_cast<const T*>(a.V) + ((size_t)b * a.Hkv + g) * (size_t)L * D;

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

#pragma unroll 1
  for (int j0 = kmin & ~15; j0 <= kmax; j0 += 16) {
    float s[2][4];
#pragma unroll
    for (int h8 = 0; h8 < 2; ++h8) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const int krow = min(j0 + 8 * h8 + gr, L - 1);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c = 16 * ks + 2 * tq;
        mma_bf16_16816(acc, qa[ks], ld_b32(Kg + (size_t)krow * D + c),
                       ld_b32(Kg + (size_t)krow * D + c + 8));
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
      const int kv0 = min(j0 + 8 * h8 + 2 * tq, L - 1);
      const int kv1 = min(j0 + 8 * h8 + 2 * tq + 1, L - 1);
#pragma unroll
      for (int nd = 0; nd < NT; ++nd) {
        const uint32_t b0 = bf16_bits_as_f32(Vg + (size_t)kv0 * D + 8 * nd + gr);
        const uint32_t b1 = bf16_bits_as_f32(Vg + (size_t)kv1 * D + 8 * nd + gr);
        mma_tf32_1688(o[nd], p[h8][0], p[h8][2], p[h8][1], p[h8][3], b0, b1);
      }
    }
    ma = na;
    mb = nb;
  }
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

bool want_mass(const PrefillArgs& a) {
  return a.mass != nullptr || a.lse != nullptr;
}

template <int D>
cudaError_t launch_select_tc(const PrefillArgs& a, cudaStream_t s) {
  using Lay = TcLayout<D>;
  // segment codes hold tile * 32 + column in 16 bits
  if ((a.L + Lay::BN - 1) / Lay::BN > 2048) return cudaErrorNotSupported;
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, a.Q, (uint64_t)a.B * a.Hq * a.nq, D)) return cudaErrorInvalidValue;
  if (!make_tmap(&tk, a.K, (uint64_t)a.B * a.Hkv * a.L, D)) return cudaErrorInvalidValue;
  // Segment positions per (row, chunk group) thread: about k/4 entries are
  // expected (1.1-1.4 k per row), but one key tile can put 31 entries into
  // one segment (rows with fewer than k candidates); the cursor check every
  // 8 columns keeps 8 positions in reserve.
  const size_t budget = 227 * 1024 - sizeof(TcShared);
  int P = a.k > 32 ? 46 : 40;
  while (P > kMinSeg && Lay::bytes(P) > budget) --P;
  if (Lay::bytes(P) > budget || P < 40) return cudaErrorNotSupported;
  const size_t smem = Lay::bytes(P);
  auto kern = want_mass(a) ? prefill_score_topk_tc<D, true>
                           : prefill_score_topk_tc<D, false>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.nq + 127) / 128, a.Hq, a.B);
  prof_before(s, "prefill_score_topk_tc");
  kern<<<grid, kTcThreads, smem, s>>>(tq, tk, a, P);
  prof_after(s);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.k == 0) return cudaSuccess;  // run for the mass reports only
  // rows whose segments overflowed (rare on typical inputs): exact fallback
  const size_t fb_smem = (size_t)(a.k + kFbBuf) * 8 + D * 4;
  prof_before(s, "prefill_overflow_rows");
  prefill_overflow_rows<__nv_bfloat16, D><<<sm_count(), kFbThreads, fb_smem, s>>>(a);
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
  } else {
    if (a.o_bf16) gather_f32_as<T, D, __nv_bfloat16, 2>(a, grid, nt, s);
    else gather_f32_as<T, D, float, 2>(a, grid, nt, s);
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
  return m ? gather_mma_as<D, 2, true>(a, grid, smem, s)
           : gather_mma_as<D, 2, false>(a, grid, smem, s);
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
    if (bf16) e = d == 64 ? launch_select_tc<64>(a, s) : launch_select_tc<128>(a, s);
    else e = d == 64 ? launch_select_f32<64>(a, s) : launch_select_f32<128>(a, s);
    if (e != cudaSuccess) return e;
  }
  if (bf16) e = d == 64 ? launch_gather_mma<64>(a, s) : launch_gather_mma<128>(a, s);
  else e = d == 64 ? launch_gather<float, 64>(a, s) : launch_gather<float, 128>(a, s);
  return e;
}

}  // namespace ca

// Prefill score + Top-k selection on tcgen05 tensor cores (bf16 Q and K).
// "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质", §2.1 Definition 1
// (S = Q K^T over every causal position), §2.2.3 (Dynamic Top-k), §5.2.2
// (identify the set, then attend on it).
//
// One CTA per 128-query tile of one (batch, head):
//   TMA warps  the key tiles 0..T-1 twice (two passes)
//              through a ring of two 32 KB stages, one stage per producer
//              warp (warps 0 and 2).  Every copy moves 32 KB (two 128-key
//              tiles at d = 64, one tile with both 64-column halves at
//              d = 128).  On this part the copy rate per SM grows with the
//              size of each copy and with the number of threads issuing them
//              (one thread's copies do not overlap: 16 KB copies from one
//              thread stream at about a quarter of what 32 KB copies from two
//              threads do).
//   warp 1     MMA: tcgen05.mma kind::f16, M = N = 128, bf16 in, fp32 out, into
//              128-column TMEM accumulators.  At d = 64 the Q tile (A) sits in
//              shared memory, written once by the first selector warps in the
//              128-byte swizzle, and TMEM holds four accumulators; at d = 128
//              Q is read from TMEM (64 columns after three accumulators), which
//              leaves its 32 KB of shared memory to the candidate segments.
//              Pass 1 is bound by the round trip of an accumulator (MMA,
//              commit, every selector warp's read and release), so the count
//              of accumulators sets its pace.
//   16 warps   selectors (after the TMA and MMA warps), thread = (query row,
//              32-column chunk group of every
//              key tile), reading the accumulators with tcgen05.ld 32x32b:
//     pass 1   64 slot maxima per thread (its 32 columns of the even and of the
//              odd key tiles), rounded toward zero to bf16 and kept in pairs:
//              256 slots per row; with k <= 32, 32 slots per thread (column
//              pairs, a three-input fp32 max per two scores): 128 per row.
//              The k-th largest slot L bounds the row's k-th best score from
//              below (the top k slots are k distinct candidates >= L; a
//              negative slot is first moved one bf16 step down, since
//              rounding toward zero raised it).
//     pass 2   every candidate >= L is appended to the thread's segment as an
//              8-byte entry {fp32 score bits, key position} by one predicated
//              vector store (about 1.1 k entries per row on random data),
//              with a room check every 8 columns.  A segment without room
//              moves to one of 16 spare segments; with none left the row goes
//              to the exact CUDA-core fallback.
//     cut      four lanes per row (one per chunk group) find the exact k-th
//              best key by bisection on the score bits (and on the positions
//              only when equal scores straddle it) and write the row's Top-k.
// Only key tiles holding a candidate of some row of the tile are computed,
// and the scores never leave the SM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.cuh"
#include "prefill.cuh"
#include "prefill_rows.cuh"
#include "profile.cuh"
#include "select.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace ca {

namespace {

constexpr int kBM = kPrefillTileRows;  // query rows per CTA
constexpr int kBN = 128;               // keys per accumulator tile
constexpr int kSelWarps = 16;          // 4 chunk groups x 4 TMEM lane quarters
constexpr int kSelThreads = 32 * kSelWarps;
constexpr int kTmemBufs = 4;  // most accumulators (d = 64; three at 128)
constexpr uint32_t kStageBytes = 32768;
constexpr uint32_t kBlockBytes = 128 * 128;  // 128 rows x 128 bytes
constexpr int kPool = 16;                    // spare segments per CTA
constexpr int kSegCols = kSelThreads + kPool;
// Entry f of segment column c sits at f * kEntStride + c * 8: the columns of
// one position are contiguous (a warp's 32 threads at equal cursors store
// 256 contiguous bytes), and positions are 2 banks apart.
constexpr int kEntStride = (kSegCols + 1) * 8;
constexpr int kCheck = 8;                    // columns between room checks
constexpr int kCutNE = 40;                   // entries per lane in the cut
constexpr uint32_t kMaskedScore = 0x7FC00000u;  // NaN: never >= L
using SelBar = GroupBarrier<1, kSelThreads>;

template <int D>
struct Layout {
  static constexpr int KT = D == 64 ? 2 : 1;  // key tiles per stage
  static constexpr int kStages = 2;  // = producer warps
  // At d = 64 the Q tile (16 KB) sits in shared memory and TMEM holds four
  // 128-column accumulators; at d = 128 Q (64 TMEM columns) sits in TMEM
  // after three accumulators, and its 32 KB stay with the segments.
  static constexpr bool kQSmem = D == 64;
  static constexpr int kBufs = kQSmem ? 4 : 3;
  static constexpr int kQCol = 3 * 128;  // TMEM columns of Q at d = 128
  // warp 0 and warp 2 produce, warp 1 issues MMAs, then the selectors
  static constexpr int kFirstSel = kStages + 1;
  static constexpr int kThreads = 32 * kFirstSel + kSelThreads;
  static constexpr size_t k_off = 0;
  static constexpr size_t q_off = k_off + (size_t)kStages * kStageBytes;
  static constexpr size_t seg_off = q_off + (kQSmem ? (size_t)kBM * 128 : 0);
  // segments, or the pass-1 slot table (128 rows x 256 bf16) before them
  __host__ __device__ static size_t bytes(int P) {
    size_t seg = (size_t)P * kEntStride;
    const size_t table = (size_t)kBM * 256 * 2;
    if (seg < table) seg = table;
    return seg_off + seg + 1024;  // + the manual 1024-byte alignment
  }
  static_assert(KT * kBN * D * 2 == (int)kStageBytes, "32 KB stages");
};

constexpr int kMaxStages = 3;

struct Shared {
  uint64_t kfull[kMaxStages], kempty[kMaxStages], qfull;
  uint64_t tfull[kTmemBufs], tempty[kTmemBufs];
  uint64_t never;  // failure-path test hook: a barrier nothing signals
  uint32_t tmem;
  int abort;
  int maxhi;
  int pool;                       // spare segments handed out
  int hi[kBM];
  float L[kBM];
  float M[kBM];                   // row maximum (mass reports)
  unsigned char cnt[kSelThreads];   // entries in the own segment
  unsigned char xcnt[kSelThreads];  // entries in the spare segment
  signed char xcol[kSelThreads];    // spare segment index, -1: none
  unsigned char ovf[kSelThreads];   // 1: candidates did not fit
  float xsum[kSelThreads];          // per thread: candidates' sum (masses)
};

__device__ __forceinline__ int quad_sum(int v) {
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
  return v + __shfl_xor_sync(0xFFFFFFFFu, v, 2);
}
__device__ __forceinline__ uint32_t quad_max(uint32_t v) {
  v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, 1));
  return max(v, __shfl_xor_sync(0xFFFFFFFFu, v, 2));
}
__device__ __forceinline__ uint32_t quad_min(uint32_t v) {
  v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, 1));
  return min(v, __shfl_xor_sync(0xFFFFFFFFu, v, 2));
}

// Order-preserving 16-bit codes of a packed pair of bf16 values: each half
// becomes v ^ 0x8000 when non-negative and ~v when negative.
__device__ __forceinline__ uint32_t ord_bf16x2(uint32_t w) {
  const uint32_t s = (w >> 15) & 0x00010001u;
  return w ^ (s * 0x7FFFu | 0x80008000u);
}
__device__ __forceinline__ float unord_bf16(uint32_t o) {
  const uint32_t v = (o & 0x8000u) ? (o ^ 0x8000u) : (~o & 0xFFFFu);
  return __uint_as_float(v << 16);
}

// Append the scores of columns x0..x0+kCheck-1 of a tile that reach L to the
// segment at `cur`: one predicated 8-byte store {score bits, position} and
// a predicated cursor step per column.
template <int X0>
__device__ __forceinline__ void append_run(const uint32_t (&raw)[32],
                                           uint32_t& cur, float L, int j0) {
#pragma unroll
  for (int x = X0; x < X0 + kCheck; ++x) {
    asm volatile(
        "{ .reg .pred p;\n\t"
        "setp.ge.f32 p, %1, %2;\n\t"
        "@p st.shared.v2.b32 [%0], {%3, %4};\n\t"
        "@p add.u32 %0, %0, %5; }"
        : "+r"(cur)
        : "f"(__uint_as_float(raw[x])), "f"(L), "r"(raw[x]), "r"(j0 + x),
          "n"(kEntStride)
        : "memory");
  }
}

// Exact Top-k of one row by its four lanes (lane part holds its chunk
// group's entries: the own segment, then the spare one).  Writes the k
// largest keys (ord(score) << 32 | ~position), or every entry when the row
// has at most k, to out[0..), padded with 0 up to kpad.
template <int NE>
__device__ __forceinline__ void quad_cut(const unsigned char* seg, int col_own,
                                         int n_own, int col_x, int n_part,
                                         bool live, uint32_t lob, int k,
                                         int kpad, uint64_t* out, int part) {
  auto addr = [&](int f) -> const uint32_t* {
    const int c = f < n_own ? col_own : col_x;
    const int e = f < n_own ? f : f - n_own;
    return reinterpret_cast<const uint32_t*>(seg + (size_t)e * kEntStride +
                                             (size_t)c * 8);
  };
  uint32_t hv[NE];
#pragma unroll
  for (int t = 0; t < NE; ++t)
    hv[t] = (live && t < n_part) ? ord_f32(__uint_as_float(*addr(t))) : 0u;
  const int total = quad_sum(live ? n_part : 0);
  const bool sel = live && total > k;
  uint32_t mx = 0u;
#pragma unroll
  for (int t = 0; t < NE; ++t) mx = max(mx, hv[t]);
  mx = quad_max(mx);
  // bisection from the common high bits of the bound and the row maximum
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
  const uint32_t th_hi = sel ? tau : 0u;
  uint32_t th_lo = 0u;
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
    for (int t = 0; t < NE; ++t)
      lo[t] = (need > 0 && t < n_part && hv[t] == th_hi)
                  ? 0xFFFFFFFFu - addr(t)[1]
                  : 0u;
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
  // write the selected keys: exclusive prefix over the four lanes
  int cnt = 0;
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    if (live && t < n_part && hv[t] >= th_hi) {
      bool s = hv[t] > th_hi || th_lo == 0u;
      if (!s) s = 0xFFFFFFFFu - addr(t)[1] >= th_lo;
      cnt += s;
    }
  }
  const int up1 = __shfl_up_sync(0xFFFFFFFFu, cnt, 1);
  const int up2 = __shfl_up_sync(0xFFFFFFFFu, cnt, 2);
  const int up3 = __shfl_up_sync(0xFFFFFFFFu, cnt, 3);
  const int pre =
      (part >= 1 ? up1 : 0) + (part >= 2 ? up2 : 0) + (part >= 3 ? up3 : 0);
  const int got = quad_sum(cnt);
  if (live) {
    int pos = pre;
#pragma unroll
    for (int t = 0; t < NE; ++t) {
      if (t < n_part && hv[t] >= th_hi) {
        const uint32_t lo = 0xFFFFFFFFu - addr(t)[1];
        if (hv[t] > th_hi || lo >= th_lo)
          out[pos++] = ((uint64_t)hv[t] << 32) | lo;
      }
    }
    for (int e = got + part; e < kpad; e += 4) out[e] = 0ull;
  }
}

// PAIR: one slot per two columns (128 per row; a three-input max per two
// scores in pass 1 and half the bound's counting) when k <= 32, where the
// extra collisions of the best keys in a slot cost a few candidates per row;
// else one slot per column and tile parity (256 per row).
template <int D, bool MASS, bool PAIR>
__global__ void __launch_bounds__(Layout<D>::kThreads, 1)
prefill_score_topk_tc(const __grid_constant__ CUtensorMap tmK, PrefillArgs a,
                      int P, int maps3d) {
  using Lay = Layout<D>;
  constexpr int KT = Lay::KT;
  constexpr int kStages = Lay::kStages;
  constexpr int kFirstSel = Lay::kFirstSel;
  constexpr int kBufs = Lay::kBufs;
  constexpr int kQCol = Lay::kQCol;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sK = smem + Lay::k_off;
  unsigned char* sQ = smem + Lay::q_off;  // d = 64: the Q tile, 128-byte rows
  unsigned char* seg = smem + Lay::seg_off;
  __shared__ Shared sh;

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = qt * kBM;  // first query row of the tile
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = head_k(a.k_h, h, a.k, a.status, qt == 0 && tid == 0);
  static_assert(kStages <= kMaxStages, "stages");

  tile_rows(a, b, h, i0, sh.hi, &sh.maxhi);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      sm100::mbar_init(&sh.kfull[s], 1);
      sm100::mbar_init(&sh.kempty[s], 1);
    }
    sm100::mbar_init(&sh.qfull, 4);  // the four Q-writing selector warps
    sm100::mbar_init(&sh.never, 1);
    for (int t = 0; t < kBufs; ++t) {
      sm100::mbar_init(&sh.tfull[t], 1);
      sm100::mbar_init(&sh.tempty[t], kSelWarps);
    }
    sh.abort = 0;
    sh.pool = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(&sh.tmem, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const int maxhi = sh.maxhi;
  const int T = maxhi >= 1 ? maxhi / kBN + 1 : 0;  // key tiles with candidates
  const int TS = (T + KT - 1) / KT;                // stages per pass
  volatile int* abort_flag = &sh.abort;

  if (warp == 0 || (warp >= 2 && warp < kFirstSel)) {
    // ---------------- TMA producers: stage p of the ring is producer p's
    // (warp 0: p = 0, warp 2: p = 1, warp 3: p = 2); the key tiles of both
    // passes
    const int p = warp == 0 ? 0 : warp - 1;
    if (lane == 0 && T > 0) {
      sm100::prefetch_tmap(&tmK);
      const int krow = (b * a.Hkv + g) * a.L;
      int last = -1;  // the last stage sequence index this producer issued
      for (int u = p; u < 2 * TS; u += kStages) {
        const int s = p;
        const uint32_t ph = (u / kStages) & 1;
        if (u >= kStages &&
            !sm100::wait_or_abort(&sh.kempty[s], ph ^ 1, abort_flag, a.status,
                                  a.wait_ns))
          break;
        const int t0 = (u < TS ? u : u - TS) * KT;  // first tile of the stage
        unsigned char* dst = sK + (size_t)s * kStageBytes;
        sm100::mbar_arrive_expect_tx(&sh.kfull[s], kStageBytes);
        if (D == 64) {
          sm100::tma_load_2d(dst, &tmK, &sh.kfull[s], 0, krow + t0 * kBN);
        } else if (maps3d) {
          sm100::tma_load_3d(dst, &tmK, &sh.kfull[s], 0, krow + t0 * kBN, 0);
        } else {
          for (int kb = 0; kb < 2; ++kb)
            sm100::tma_load_2d(dst + kb * kBlockBytes, &tmK, &sh.kfull[s],
                               kb * 64, krow + t0 * kBN);
        }
        last = u;
      }
      // every copy this thread started must land before the CTA can exit
      bool drained = true;
      if (last >= 0)
        drained &= sm100::mbar_wait(&sh.kfull[p], (last / kStages) & 1,
                                    kDrainWaitNs);
      if (!drained) raise_flag(a.status, kErrTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop (waits,
    // addresses and descriptors warp-uniform); one elected lane issues each
    // MMA and commit
    if (T > 0) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(kBM, kBN);
      const uint32_t ak = sm100::smem_u32(sK);
      const bool leader = sm100::elect_one();
      int tt = 0;  // accumulator tiles issued, both passes
      if (a.stall_ns) {
        // Failure-path test hook: wait on a barrier that nothing signals, so
        // the wait runs out, raises the time-out flag and aborts every wait
        // of the CTA; the kernel then leaves through its normal path.
        if (leader)
          sm100::wait_or_abort(&sh.never, 0, abort_flag, a.status, a.stall_ns);
        __syncwarp();
      }
      if (__all_sync(0xFFFFFFFFu,
                     sm100::wait_or_abort(&sh.qfull, 0, abort_flag, a.status,
                                          a.wait_ns))) {
        bool ok = true;
        for (int u = 0; u < 2 * TS && ok; ++u) {
          const int s = u % kStages;
          const uint32_t ph = (u / kStages) & 1;
          if (!__all_sync(0xFFFFFFFFu,
                          sm100::wait_or_abort(&sh.kfull[s], ph, abort_flag,
                                               a.status, a.wait_ns)))
            break;
          const int t0 = (u < TS ? u : u - TS) * KT;
#pragma unroll
          for (int q = 0; q < KT; ++q) {
            if (t0 + q >= T) break;
            const int buf = tt % kBufs;
            if (tt >= kBufs &&
                !__all_sync(0xFFFFFFFFu,
                            sm100::wait_or_abort(&sh.tempty[buf],
                                                 ((tt / kBufs) & 1) ^ 1,
                                                 abort_flag, a.status,
                                                 a.wait_ns))) {
              ok = false;
              break;
            }
            sm100::tc_fence_after();
            const uint32_t d_tmem = tmem + buf * kBN;
            const uint32_t kt = ak + s * kStageBytes + q * kBlockBytes;
            if (leader) {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * kBlockBytes + (kk & 3) * 32;
                if constexpr (Lay::kQSmem)
                  sm100::mma_bf16(d_tmem,
                                  sm100::desc_k_sw128(sm100::smem_u32(sQ) +
                                                      (kk & 3) * 32),
                                  sm100::desc_k_sw128(kt + off), idesc,
                                  kk > 0 ? 1u : 0u);
                else
                  sm100::mma_bf16_ts(d_tmem, tmem + kQCol + kk * 8,
                                     sm100::desc_k_sw128(kt + off), idesc,
                                     kk > 0 ? 1u : 0u);
              }
              sm100::mma_commit(&sh.tfull[buf]);
            }
            __syncwarp();
            ++tt;
          }
          if (leader) sm100::mma_commit(&sh.kempty[s]);
          __syncwarp();
        }
      }
      // The last commit covers every MMA issued: wait for it before exit.
      if (leader && tt > 0 &&
          !sm100::mbar_wait(&sh.tfull[(tt - 1) % kBufs],
                            ((tt - 1) / kBufs) & 1, kDrainWaitNs))
        raise_flag(a.status, kErrTimeout);
    }
  } else {
    // ---------------- selector warps: thread = (query row, chunk group)
    const int sw = warp - kFirstSel;       // 0..15
    const int grp = sw >> 2;               // 32-column chunk of every tile
    const int quarter = warp & 3;          // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;     // query row in the tile
    const int col = grp * kBM + r;         // own segment column
    const int hi = sh.hi[r];
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + grp * 32;

    if (grp == 0 && Lay::kQSmem) {
      // the Q tile into shared memory: this warp's 32 rows, each thread its
      // own 128-byte row, 16-byte pieces placed as the 128-byte swizzle
      // places them (piece c of row r at c ^ (r % 8)), zeros past the last
      // query row; then made visible to the tensor core's reads
      const bool qv = i0 + r < a.nq;
      const uint4* qp = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(a.Q) +
          ((size_t)(b * a.Hq + h) * a.nq + (qv ? i0 + r : 0)) * D);
      uint4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = qv ? qp[c] : make_uint4(0u, 0u, 0u, 0u);
      uint4* qrow = reinterpret_cast<uint4*>(sQ + (size_t)r * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c) qrow[c ^ (r & 7)] = v[c];
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sh.qfull);
    } else if (grp == 0) {
      // the Q tile into TMEM columns kQCol..: this warp's 32 rows, each
      // thread its own row as bf16 pairs (zeros past the last query row)
      const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16) + kQCol;
      const bool qv = i0 + r < a.nq;
      const uint4* qp = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(a.Q) +
          ((size_t)(b * a.Hq + h) * a.nq + (qv ? i0 + r : 0)) * D);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 v = qv ? qp[c * 8 + e] : make_uint4(0u, 0u, 0u, 0u);
          w[4 * e] = v.x;
          w[4 * e + 1] = v.y;
          w[4 * e + 2] = v.z;
          w[4 * e + 3] = v.w;
        }
        sm100::tmem_st_32x32b_x32(tq + c * 32, w);
      }
      sm100::tmem_wait_st();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sh.qfull);
    }

    // Scores of accumulator tile tt (key tile t of its pass) for this
    // thread's row and chunk, non-candidates (j = 0, the window, the future)
    // replaced by NaN.
    auto fetch = [&](int tt, int t, uint32_t (&raw)[32]) -> bool {
      const int buf = tt % kBufs;
      if (!__all_sync(0xFFFFFFFFu,
                      sm100::wait_or_abort(&sh.tfull[buf], (tt / kBufs) & 1,
                                           abort_flag, a.status, a.wait_ns)))
        return false;
      sm100::tc_fence_after();
      sm100::tmem_ld_32x32b_x32(tl + buf * kBN, raw);
      sm100::tmem_wait_ld();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&sh.tempty[buf]);
      const int j0 = t * kBN + grp * 32;
      if (!(j0 >= 1 && j0 + 31 <= hi)) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (!(j0 + x >= 1 && j0 + x <= hi)) raw[x] = kMaskedScore;
      }
      return true;
    };

    // ---- pass 1: bf16 slot maxima, even tiles in sl[0], odd tiles in sl[1]
    // (PAIR: fp32 maxima of column pairs over all tiles, in fl)
    uint32_t sl[2][16];
    float fl[2][16];
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        sl[p][x] = 0xFF80FF80u;  // (-inf, -inf)
        fl[p][x] = -INFINITY;
      }
    auto slot_max = [&](const uint32_t (&raw)[32], int p) {
      if constexpr (PAIR) {
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float m3;
          asm("max.f32 %0, %1, %2, %3;"
              : "=f"(m3)
              : "f"(fl[p][x]), "f"(__uint_as_float(raw[2 * x])),
                "f"(__uint_as_float(raw[2 * x + 1])));
          fl[p][x] = m3;
        }
      } else {
#pragma unroll
        for (int x = 0; x < 16; ++x)
          sl[p][x] = sm100::max_bf16x2(
              sl[p][x], sm100::cvt_rz_bf16x2(__uint_as_float(raw[2 * x + 1]),
                                             __uint_as_float(raw[2 * x])));
      }
    };
    bool live_pass = true;
#pragma unroll 1
    for (int t = 0; t < T; t += 2) {
      uint32_t raw[32];
      if (!fetch(t, t, raw)) {
        live_pass = false;
        break;
      }
      slot_max(raw, 0);
      if (t + 1 < T) {
        if (!fetch(t + 1, t + 1, raw)) {
          live_pass = false;
          break;
        }
        slot_max(raw, 1);
      }
    }
    // ---- the slot table: row r's 512 bytes, 16-byte pieces XOR-swizzled
    // by the row so that 32 rows written (or one row read) at once spread
    // over the banks
    {
      uint4* table = reinterpret_cast<uint4*>(seg);
      if constexpr (PAIR) {
        // 32 slots, rounded toward zero to bf16, two per word: row r's 256
        // bytes, 16-byte pieces swizzled by the row
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int x = 0; x < 8; ++x)
            sl[p][x] = sm100::cvt_rz_bf16x2(fl[p][2 * x + 1], fl[p][2 * x]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int piece = (grp * 4 + c) ^ (r & 15);
          const uint32_t* src = &sl[c >> 1][(c & 1) * 4];
          table[r * 16 + piece] = make_uint4(src[0], src[1], src[2], src[3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int piece = (grp * 8 + c) ^ (r & 31);
          const uint32_t* src = &sl[c >> 2][(c & 3) * 4];
          table[r * 32 + piece] = make_uint4(src[0], src[1], src[2], src[3]);
        }
      }
    }
    SelBar::sync();
    {
      // ---- bound: four lanes per row (part = chunk group), eight rows per
      // warp.  tau is the largest 16-bit code with at least k slots >= it
      // (or the first probe that leaves exactly k): the k-th largest slot.
      const int row = sw * 8 + (lane >> 2), part = lane & 3;
      const uint4* table = reinterpret_cast<const uint4*>(seg);
      // ord codes: hw compares the high halves as is, lw the low halves
      // moved up (a 16-bit code c is compared as c << 16)
      constexpr int NWD = PAIR ? 16 : 32;  // slot words per lane
      uint32_t hw[NWD], lw[NWD];
      uint32_t mx = 0u, mn = 0xFFFFu;
#pragma unroll
      for (int c = 0; c < NWD / 4; ++c) {
        const uint4 v = PAIR
            ? table[row * 16 + ((part * 4 + c) ^ (row & 15))]
            : table[row * 32 + ((part * 8 + c) ^ (row & 31))];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t o = ord_bf16x2(w[e]);
          hw[c * 4 + e] = o;
          lw[c * 4 + e] = o << 16;
          mx = max(mx, max(o >> 16, o & 0xFFFFu));
          mn = min(mn, min(o >> 16, o & 0xFFFFu));
        }
      }
      mx = quad_max(mx);
      mn = quad_min(mn);
      const uint32_t diff = mn ^ mx;
      const int nb = diff ? 32 - __clz(diff) : 0;  // at most 16
      uint32_t tau = (mn >> nb) << nb;  // every slot is >= this prefix
      bool done = nb == 0 || k == 0;
      const int bmax = __reduce_max_sync(0xFFFFFFFFu, nb);
#pragma unroll 1
      for (int bit = bmax - 1; bit >= 0; --bit) {
        if (__all_sync(0xFFFFFFFFu, done)) break;
        const uint32_t c = tau | (1u << bit);
        const uint32_t C = c << 16;
        int m = 0;
#pragma unroll
        for (int x = 0; x < NWD; ++x) m += (hw[x] >= C) + (lw[x] >= C);
        m = quad_sum(m);
        const bool up = !done && bit < nb && m >= k;
        tau = up ? c : tau;
        done |= up && m == k;
      }
      if (part == 0) {
        float L;
        if (k == 0) L = INFINITY;               // nothing to select
        else if (tau <= 0x7Fu) L = -INFINITY;   // fewer than k candidates
        else if (tau & 0x8000u) L = unord_bf16(tau);
        else L = unord_bf16(tau - 1);  // negative: undo the rounding up
        sh.L[row] = L;
        if constexpr (MASS) sh.M[row] = mx > 0x7Fu ? unord_bf16(mx) : -INFINITY;
      }
    }
    SelBar::sync();

    // ---- pass 2: every candidate >= L into this thread's segment; a
    // segment without room for kCheck more entries continues in a spare one
    // (once per thread, while any is left), else the row goes to the exact
    // fallback
    const float Lr = sh.L[r];
    const float sl2 = 1.4426950408889634f / sqrtf((float)D);
    const float Mr = MASS ? sh.M[r] : 0.f;
    float xs = 0.f;  // this thread's share of the candidates' sum
    const uint32_t seg_s = sm100::smem_u32(seg);
    uint32_t base = seg_s + col * 8;
    uint32_t cur = base;
    uint32_t lim = base + (uint32_t)(P - kCheck) * kEntStride;
    int xc = -1, own = 0;
    bool ovf = false;
    // make room for kCheck more entries (per thread; rare after the first
    // tiles of a row)
    auto room = [&]() {
      if (cur > lim && !ovf) {
        const int px = xc < 0 ? atomicAdd(&sh.pool, 1) : kPool;
        if (px < kPool) {
          own = (cur - base) / kEntStride;
          xc = px;
          base = seg_s + (kSelThreads + px) * 8;
          cur = base;
          lim = base + (uint32_t)(P - kCheck) * kEntStride;
        } else {
          ovf = true;
        }
      }
      // debug builds: the next run's kCheck entries must fit the segment
      if (!ovf && !in_bounds(cur <= lim, a.status)) ovf = true;
    };
#pragma unroll 1
    for (int t = 0; t < T && live_pass; ++t) {
      uint32_t raw[32];
      if (!fetch(T + t, t, raw)) break;
      if constexpr (MASS) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          xs += exp2f(fmaxf((__uint_as_float(raw[x]) - Mr) * sl2, -INFINITY));
      }
      const int j0 = t * kBN + grp * 32;
      static_assert(32 % kCheck == 0 && 32 / kCheck == 4, "four runs");
      room();
      append_run<0>(raw, cur, ovf ? INFINITY : Lr, j0);
      room();
      append_run<kCheck>(raw, cur, ovf ? INFINITY : Lr, j0);
      room();
      append_run<2 * kCheck>(raw, cur, ovf ? INFINITY : Lr, j0);
      room();
      append_run<3 * kCheck>(raw, cur, ovf ? INFINITY : Lr, j0);
    }
    const int last = (cur - base) / kEntStride;
    sh.cnt[col] = (unsigned char)(xc < 0 ? last : own);
    sh.xcnt[col] = (unsigned char)(xc < 0 ? 0 : last);
    sh.xcol[col] = (signed char)xc;
    sh.ovf[col] = ovf ? 1 : 0;
    // per thread: sum of 2^((s - M) log2e/sqrt(d)) over its candidates
    if constexpr (MASS) sh.xsum[col] = xs;
    SelBar::sync();
    {
      // ---- exact Top-k per row: four lanes per row, eight rows per warp
      const int row = sw * 8 + (lane >> 2), part = lane & 3;
      const int rq = i0 + row;  // query row
      const int cown = part * kBM + row;
      const int n_own = sh.cnt[cown];
      const int x = sh.xcol[cown];
      const int n_part = n_own + (x >= 0 ? sh.xcnt[cown] : 0);
      const int col_x = kSelThreads + (x >= 0 ? x : 0);
      // debug builds: the entry counts must lie within the segments
      const bool seg_ok = in_bounds(
          n_own <= P && (x < 0 || (x < kPool && sh.xcnt[cown] <= P)),
          a.status);
      const bool bad =
          quad_sum(sh.ovf[cown] || n_part > kCutNE || !seg_ok) > 0;
      const size_t grow = (size_t)(b * a.Hq + h) * a.nq + rq;
      bool live = rq < a.nq;
      if constexpr (MASS) {
        float t = sh.xsum[cown];
        t += __shfl_xor_sync(0xFFFFFFFFu, t, 1);
        t += __shfl_xor_sync(0xFFFFFFFFu, t, 2);
        if (live && part == 0)
          a.cand_ml[grow] = make_float2(sh.M[row] * sl2, t);
      }
      if (live && bad) {
        // listed for the exact fallback pass, which writes this row
        if (part == 0) {
          const uint32_t pos = atomicAdd(a.ovf_count, 1u);
          if (in_bounds(pos < (uint32_t)(a.B * a.Hq * a.nq), a.status))
            a.ovf_rows[pos] = (uint32_t)grow;
        }
        live = false;
      }
      const uint32_t lob = ord_f32(sh.L[row]);
      uint64_t* out = a.topk + grow * a.k;
      // entries per lane sized by the warp's fullest lane: the bisection
      // counts every slot of the array at each step
      if (__all_sync(0xFFFFFFFFu, !live || n_part <= 16))
        quad_cut<16>(seg, cown, n_own, col_x, n_part, live, lob, k, a.k, out,
                     part);
      else if (__all_sync(0xFFFFFFFFu, !live || n_part <= 24))
        quad_cut<24>(seg, cown, n_own, col_x, n_part, live, lob, k, a.k, out,
                     part);
      else if (__all_sync(0xFFFFFFFFu, !live || n_part <= 32))
        quad_cut<32>(seg, cown, n_own, col_x, n_part, live, lob, k, a.k, out,
                     part);
      else
        quad_cut<kCutNE>(seg, cown, n_own, col_x, n_part, live, lob, k, a.k,
                         out, part);
    }
  }
  __syncwarp();  // reconverge single-lane roles before the CTA barrier
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
template <int D>
cudaError_t launch_d(const PrefillArgs& a, cudaStream_t s) {
  using Lay = Layout<D>;
  CUtensorMap tk;
  int maps3d = 0;
  const uint64_t krows = (uint64_t)a.B * a.Hkv * a.L;
  if (D == 64) {
    if (!make_tmap_2d(&tk, a.K, krows, D, kBN * Lay::KT))
      return cudaErrorInvalidValue;
  } else if (make_tmap_3d(&tk, a.K, krows, kBN)) {
    maps3d = 1;
  } else if (!make_tmap_2d(&tk, a.K, krows, D, kBN)) {
    // two 16 KB copies per stage when the 3-D view is refused
    return cudaErrorInvalidValue;
  }
  // Segment positions per (row, chunk group) thread: about k/4 entries are
  // expected (about 1.1 k per row), with the spare segments for the rest.
  const size_t budget = 227 * 1024 - sizeof(Shared);
  int P = 64;
  while (P > kCheck && Lay::bytes(P) > budget) --P;
  // a fresh (spare) segment must hold one run of kCheck entries
  if (Lay::bytes(P) > budget || P < kCheck + 8) return cudaErrorNotSupported;
  const size_t smem = Lay::bytes(P);
  const bool mass = a.mass != nullptr || a.lse != nullptr;
  const bool pair = a.k <= 32;
  auto kern = mass ? (pair ? prefill_score_topk_tc<D, true, true>
                           : prefill_score_topk_tc<D, true, false>)
                   : (pair ? prefill_score_topk_tc<D, false, true>
                           : prefill_score_topk_tc<D, false, false>);
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.nq + kBM - 1) / kBM, a.Hq, a.B);
  prof_before(s, "prefill_score_topk_tc");
  kern<<<grid, Lay::kThreads, smem, s>>>(tk, a, P, maps3d);
  prof_after(s);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_tc(const PrefillArgs& a, int d, cudaStream_t s) {
  // positions are 32-bit; the MMA tiles need a whole number of 16-byte
  // pieces per row
  if (d == 64) return launch_d<64>(a, s);
  if (d == 128) return launch_d<128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace ca

// Decode score pass with a per-chunk Top-k on tcgen05 tensor cores (bf16 K
// and q).  "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质", §2.1
// Definition 1 (C_i for the last row), §2.2.3 (Dynamic Top-k), §2.4
// Corollary 3 (per-query window).
//
// Grid (workers, Hkv, B), about two CTAs per SM; the workers of one (batch,
// kv-head) share its cache for the G = Hq/Hkv q-heads reading it.  The cache
// is cut into units of 32 KB (one 128-key tile with both 64-column halves at
// d = 128, two tiles at d = 64); each worker takes units as it goes (the
// first ones fixed by its index, the rest claimed from a per-group counter),
// so that workers which stream faster take more of them, and keeps one
// candidate list per q-head over the keys it saw.
//   warp 0     TMA: the group's q rows once (16 rows: the G heads, the rest
//              of the box ignored), then one claimed unit per stage of a ring;
//              a stage marked empty (position -1) ends the stream.
//   warp 1     MMA: tcgen05.mma kind::f16 with M = 128 keys and N = 16 heads,
//              A = the key tile, B = the q rows, fp32 accumulators of 16
//              columns in TMEM (eight buffers).  The score of key j for head h
//              lands in TMEM lane j, column h.
//   warps 2-9  selectors, two per TMEM lane quarter taking alternate tiles;
//              thread = key.  tcgen05.ld 32x32b.xG gives the thread its key's
//              G scores; each goes through the per-head candidate list of the
//              CUDA-core kernel (the first 512 keys into their own slots, then
//              admission behind a threshold that only rises, lists cut back to
//              the head's k by one warp each after every 512 keys).
// Every list is a union of whole units of the group's keys, so the union of
// the workers' best-k lists holds the group's global Top-k for each head.
// The score pass no longer spends CUDA-core instructions on the dot products:
// the tensor pipe computes them, and the stream is bound by HBM.
#include "common.cuh"
#include "decode.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "select.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace ca {

namespace {

constexpr int kKeys = 128;        // keys per accumulator tile (MMA M)
constexpr int kN = 16;            // MMA N: the group's q-heads, padded
constexpr int kTBufs = 8;         // accumulators of kN columns
constexpr int kTmemCols = 128;    // kTBufs * kN
constexpr int kSelW = 8;          // selector warps
constexpr int kSelT = 32 * kSelW;
constexpr int kThreads = 64 + kSelT;
constexpr uint32_t kStage = 32768;
constexpr int kMaxSt = 4;
constexpr int kStretchTiles = 4;  // tiles between list checks (512 keys)
constexpr int kSubKeys = kStretchTiles * kKeys;
constexpr int kMinSlack = 256, kMaxSlack = 2048;
constexpr size_t kSmemTwo = 108 * 1024;  // two CTAs per SM, with margin
constexpr size_t kSmemOne = 227 * 1024;
using SelBar = GroupBarrier<1, kSelT>;

template <int G>
struct Shared {
  uint64_t full[kMaxSt], empty[kMaxSt], qfull;
  uint64_t tfull[kTBufs], tempty[kTBufs];
  uint64_t never;  // failure-path test hook: a barrier nothing signals
  uint64_t thr[G];
  uint32_t tmem;
  int abort;
  int spos[kMaxSt];   // first key position of the unit in a stage, -1: end
  int tpos[kTBufs];   // first key position of the tile in an accumulator
  int first_tiles;    // tiles of the first stretch that held keys
  int ended;          // a selector met the end of the stream
  int stop;           // the selectors leave after this check
  int cnt[G];
  int kk[G];
  int hi[G];
  uint32_t hist[G][256];  // one radix histogram per list (per cutting warp)
  float2 ml[kSelW][G];    // per warp and head: candidates' (max, sum)
};

template <int D>
struct Lay {
  static constexpr int KT = D == 64 ? 2 : 1;  // key tiles per stage
  static constexpr uint32_t kQBytes = kN * D * 2;
  static constexpr size_t q_off = 0;
  static constexpr size_t k_off = 4096;  // 1024-aligned, after q
};

// At a check point (all inserts of the stretch done): warp h cuts list h
// back to its head's k keys, which raises the admission threshold for the
// next stretch; the keys sit in registers when they fit.  The first check
// also drops the empty (0) keys of the first stretch's slots, so that later
// lists hold real keys only.  Barriers on both sides keep every selector
// from inserting while a list is being cut.  In between, one thread decides
// for all whether the selectors leave after this check (the stream ended, a
// wait gave up, or the stretch count reached its bound `last`), so every
// selector warp takes the same number of barriers.
template <int G>
__device__ __forceinline__ void check(uint64_t* buf, int cap, bool first,
                                      bool last, Shared<G>* sh, int sw,
                                      int lane) {
  SelBar::sync();
  if (sw == 0 && lane == 0)
    sh->stop = (last || sh->ended || *(volatile int*)&sh->abort) ? 1 : 0;
  if (sw < G) {
    const int n = sh->cnt[sw];  // at most kSubKeys on the first check
    const int kk = sh->kk[sw];
    if (kk > 0 && (n > kk || (first && n > 0))) {
      uint64_t* lst = buf + (size_t)sw * cap;
      uint64_t T;
      int kept = kk;
      if (n <= 128) T = warp_cut_regs<4>(lst, n, kk, lane, &kept);
      else if (n <= 256) T = warp_cut_regs<8>(lst, n, kk, lane, &kept);
      else if (n <= 512) T = warp_cut_regs<16>(lst, n, kk, lane, &kept);
      else T = warp_cut(lst, n, kk, sh->hist[sw], lane);  // keys all real
      if (lane == 0) {
        sh->cnt[sw] = kept;
        // T = 1: the list holds every real key so far, the next stretch
        // admits any real key
        sh->thr[sw] = T > 1ull ? T : 0ull;
      }
    }
  }
  SelBar::sync();
}

template <int G>
__device__ __forceinline__ void tmem_ld_g(uint32_t taddr, uint32_t (&r)[G]);
template <>
__device__ __forceinline__ void tmem_ld_g<1>(uint32_t taddr, uint32_t (&r)[1]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
               : "=r"(r[0]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_g<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_g<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_g<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
}

template <int D, int G, bool MASS>
__global__ void __launch_bounds__(kThreads, G >= 8 ? 1 : 2)
decode_score_topk_tc(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK, DecodeArgs a,
                     int maps3d) {
  using Ly = Lay<D>;
  constexpr int KT = Ly::KT;
  constexpr int kUnitKeys = KT * kKeys;  // keys per unit (one stage)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + Ly::q_off;
  unsigned char* sK = smem + Ly::k_off;
  const int NS = a.nstages;
  const int cap = a.cap;
  uint64_t* buf = reinterpret_cast<uint64_t*>(sK + (size_t)NS * kStage);
  __shared__ Shared<G> sh_;
  Shared<G>* sh = &sh_;

  // Let the merge kernel (launched as a programmatic dependent) start its
  // independent prologue on SMs this grid releases.
  asm volatile("griddepcontrol.launch_dependents;");
  const int worker = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int nworkers = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L;        // rows of this cache (a shard of the sequence)
  const int pos0 = a.pos0;  // sequence position of row 0
  if (tid == 0) {
    // per q-head of the group: last candidate position (in the sequence,
    // whose query sits at Lg - 1) and Top-k size
    for (int h = 0; h < G; ++h) {
      const int hq = g * G + h;
      const bool rep = worker == 0;
      sh->hi[h] = (a.Lg - 1) - row_window(a.W_i, b, a.W_h, hq, a.W, a.Lg,
                                          a.status, rep);
      sh->kk[h] = head_k(a.k_h, hq, a.k, a.status, rep);
      sh->cnt[h] = 0;
      sh->thr[h] = sh->kk[h] > 0 ? 0ull : ~0ull;  // k = 0 admits nothing
    }
    for (int s = 0; s < NS; ++s) {
      sm100::mbar_init(&sh->full[s], 1);
      sm100::mbar_init(&sh->empty[s], 1);
    }
    sm100::mbar_init(&sh->qfull, 1);
    sm100::mbar_init(&sh->never, 1);
    for (int t = 0; t < kTBufs; ++t) {
      // the MMA commit, and the issuer's own arrive after it wrote tpos
      sm100::mbar_init(&sh->tfull[t], 2);
      sm100::mbar_init(&sh->tempty[t], kSelW / 2);
    }
    sh->abort = 0;
    sh->first_tiles = 0;
    sh->ended = 0;
    sh->stop = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(&sh->tmem, kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = sh->tmem;
  int hi = -1;
#pragma unroll
  for (int h = 0; h < G; ++h) hi = max(hi, sh->hi[h]);
  // the group's candidate keys are positions 1..hi; in this cache, rows
  // 0..hl, in units of kUnitKeys rows from row 0 (position 0 and positions
  // past a head's window start are masked by the selectors)
  const int hl = min(hi - pos0, L - 1);
  const int nunits = (hi >= 1 && hl >= 0) ? (hl + kUnitKeys) / kUnitKeys : 0;
  volatile int* abort_flag = &sh->abort;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      sm100::prefetch_tmap(&tmQ);
      sm100::prefetch_tmap(&tmK);
      const int qrow = b * a.Hq + g * G;
      const int krow = (b * a.Hkv + g) * L;
      int* ctr = a.claims + (size_t)b * a.Hkv + g;
      sm100::mbar_arrive_expect_tx(&sh->qfull, Ly::kQBytes);
      for (int kb = 0; kb < D / 64; ++kb)
        sm100::tma_load_2d(sQ + kb * (kN * 128), &tmQ, &sh->qfull, kb * 64,
                           qrow);
      // The first NS units of a worker are fixed (worker + i * nworkers);
      // later ones come from the group's counter, each claimed one stage
      // ahead so that the atomic's latency hides behind the copies in
      // flight (claiming further ahead leaves more work committed to a
      // worker when the counter runs out).
      const int nfixed = NS * nworkers;
      auto unit_of = [&](int u, int claim) {
        return u < NS ? worker + u * nworkers : nfixed + claim;
      };
      int c_next = nunits > nfixed ? atomicAdd(ctr, 1) : 0;
      int issued = 0;
      // every pass takes a unit no other worker takes (or ends the stream),
      // so there are at most nunits + 1 passes; the bound only guards that
      for (int u = 0; u <= nunits + NS; ++u) {
        int unit = u < NS ? unit_of(u, 0) : unit_of(u, c_next);
        if (u == nunits + NS) {
          raise_flag(a.status, kErrInternal);
          unit = nunits;  // end the stream
        }
        if (u >= NS && unit < nunits) c_next = atomicAdd(ctr, 1);
        const int s = u % NS;
        const uint32_t ph = (u / NS) & 1;
        if (u >= NS &&
            !sm100::wait_or_abort(&sh->empty[s], ph ^ 1, abort_flag, a.status,
                                  a.wait_ns))
          break;
        issued = u + 1;
        if (unit >= nunits) {
          // end of the stream: a stage without data
          sh->spos[s] = -1;
          sm100::mbar_arrive(&sh->full[s]);
          break;
        }
        unsigned char* dst = sK + (size_t)s * kStage;
        const int row = krow + unit * kUnitKeys;
        sh->spos[s] = unit * kUnitKeys;
        sm100::mbar_arrive_expect_tx(&sh->full[s], kStage);
        if (D == 64) {
          sm100::tma_load_2d(dst, &tmK, &sh->full[s], 0, row);
        } else if (maps3d) {
          sm100::tma_load_3d(dst, &tmK, &sh->full[s], 0, row, 0);
        } else {
          for (int kb = 0; kb < 2; ++kb)
            sm100::tma_load_2d(dst + kb * 16384, &tmK, &sh->full[s], kb * 64,
                               row);
        }
      }
      // every copy this thread started must land before the CTA can exit
      bool drained = sm100::mbar_wait(&sh->qfull, 0, kDrainWaitNs);
      for (int u = issued - NS < 0 ? 0 : issued - NS; u < issued; ++u)
        drained &= sm100::mbar_wait(&sh->full[u % NS], (u / NS) & 1,
                                    kDrainWaitNs);
      if (!drained) raise_flag(a.status, kErrTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop (waits,
    // addresses and descriptors warp-uniform); one elected lane writes the
    // tile positions and issues each MMA, commit and arrival
    {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(kKeys, kN);
      const uint32_t aq = sm100::smem_u32(sQ);
      const uint32_t ak = sm100::smem_u32(sK);
      const bool leader = sm100::elect_one();
      int tt = 0, real = 0;
      bool ok = true;
      // the next accumulator buffer, once the selectors have released it
      auto take_buf = [&]() -> int {
        const int tb = tt & (kTBufs - 1);
        if (tt >= kTBufs &&
            !__all_sync(0xFFFFFFFFu,
                        sm100::wait_or_abort(&sh->tempty[tb],
                                             ((tt / kTBufs) & 1) ^ 1,
                                             abort_flag, a.status, a.wait_ns)))
          return -1;
        return tb;
      };
      if (a.stall_ns) {
        // Failure-path test hook: wait on a barrier that nothing signals, so
        // the wait runs out, raises the time-out flag and aborts every wait
        // of the CTA; the kernel then leaves through its normal path.
        if (leader)
          sm100::wait_or_abort(&sh->never, 0, abort_flag, a.status,
                               a.stall_ns);
        __syncwarp();
      }
      if (__all_sync(0xFFFFFFFFu,
                     sm100::wait_or_abort(&sh->qfull, 0, abort_flag, a.status,
                                          a.wait_ns))) {
        for (int u = 0; ok; ++u) {
          const int s = u % NS;
          if (!__all_sync(0xFFFFFFFFu,
                          sm100::wait_or_abort(&sh->full[s], (u / NS) & 1,
                                               abort_flag, a.status,
                                               a.wait_ns)))
            break;
          const int pos = *(volatile int*)&sh->spos[s];
          if (pos < 0) {
            // end of the stream: two empty tiles, so that both selector
            // halves (alternate tiles) meet one
            for (int e = 0; e < 2 && ok; ++e) {
              const int tb = take_buf();
              if (tb < 0) {
                ok = false;
                break;
              }
              if (leader) {
                sh->tpos[tb] = -1;
                sm100::mbar_arrive(&sh->tfull[tb]);
                sm100::mbar_arrive(&sh->tfull[tb]);
              }
              __syncwarp();
              ++tt;
            }
            break;
          }
#pragma unroll
          for (int q = 0; q < KT; ++q) {
            const int tb = take_buf();
            if (tb < 0) {
              ok = false;
              break;
            }
            sm100::tc_fence_after();
            const uint32_t kt = ak + s * kStage + q * 16384;
            if (leader) {
              sh->tpos[tb] = pos + q * kKeys;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t offk = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint32_t offq = (kk >> 2) * (kN * 128) + (kk & 3) * 32;
                sm100::mma_bf16(tmem + tb * kN, sm100::desc_k_sw128(kt + offk),
                                sm100::desc_k_sw128(aq + offq), idesc,
                                kk > 0 ? 1u : 0u);
              }
              sm100::mma_commit(&sh->tfull[tb]);
              sm100::mbar_arrive(&sh->tfull[tb]);  // releases the tpos write
            }
            __syncwarp();
            ++tt;
            real = tt;
          }
          if (leader) sm100::mma_commit(&sh->empty[s]);
          __syncwarp();
        }
      }
      // The last commit covers every MMA issued: wait for it before exit.
      if (leader && real > 0 &&
          !sm100::mbar_wait(&sh->tfull[(real - 1) & (kTBufs - 1)],
                            ((real - 1) / kTBufs) & 1, kDrainWaitNs))
        raise_flag(a.status, kErrTimeout);
    }
  } else {
    // ---------------- selectors: thread = key of the tile
    const int sw = warp - 2;           // 0..7
    const int half = sw >> 2;          // takes the tiles t with t % 2 == half
    const int quarter = warp & 3;      // TMEM lane quarter
    const int kq = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = 1.4426950408889634f / sqrtf((float)D);
    int hi_h[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hi_h[h] = sh->hi[h];
    Lse2 ml[G];
    uint64_t thr[G];
    float thr_f[G];
    bool done = false;  // this half met the end of the stream
    // A worker sees at most every unit's tiles and the two end tiles: the
    // stretch count is bounded by that (a longer run is an internal error).
    const int max_stretch = (nunits * KT + 2 + kStretchTiles - 1) / kStretchTiles;
#pragma unroll 1
    for (int m = 0;; ++m) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        thr[h] = sh->thr[h];
        thr_f[h] = thr[h] ? key_score(thr[h]) : -INFINITY;
      }
#pragma unroll 1
      for (int t = m * kStretchTiles + half;
           t < (m + 1) * kStretchTiles && !done; t += 2) {
        const int tb = t & (kTBufs - 1);
        const bool ok = __all_sync(
            0xFFFFFFFFu,
            sm100::wait_or_abort(&sh->tfull[tb], (t / kTBufs) & 1, abort_flag,
                                 a.status, a.wait_ns));
        if (!ok) {
          done = true;
          break;
        }
        const int pos = *(volatile int*)&sh->tpos[tb];
        if (pos < 0) {
          done = true;
          if (lane == 0) sh->ended = 1;
          break;
        }
        if (m == 0 && lane == 0 && (sw & 3) == 0)
          atomicMax(&sh->first_tiles, t + 1);
        uint32_t v[G];
        sm100::tc_fence_after();
        tmem_ld_g<G>(tl + tb * kN, v);
        sm100::tmem_wait_ld();
        sm100::tc_fence_before();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&sh->tempty[tb]);
        const int j = pos0 + pos + kq;  // sequence position
        const bool in = pos + kq <= hl && j >= 1;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float sc = __uint_as_float(v[h]);
          const bool cand = in && j <= hi_h[h];
          if constexpr (MASS) {
            if (cand) ml[h].add(sc * sl2);
          }
          if (m == 0) {
            // first stretch: every key of the tile goes in at its own slot
            // (a key outside this head's candidates as an empty key)
            if (in_bounds(t * kKeys + kq < cap, a.status))
              buf[(size_t)h * cap + t * kKeys + kq] =
                  cand ? make_key(sc, (uint32_t)j) : 0ull;
          } else if (cand && sc >= thr_f[h]) {
            const uint64_t key = make_key(sc, (uint32_t)j);
            if (key > thr[h]) {
              const int p = atomicAdd(&sh->cnt[h], 1);
              if (in_bounds(p < cap, a.status)) buf[(size_t)h * cap + p] = key;
            }
          }
        }
      }
      if (m == 0) {
        // the first stretch filled the slots of its tiles that held keys
        // (a prefix of the worker's tiles)
        SelBar::sync();
        if (tid - 64 < G)
          sh->cnt[tid - 64] = sh->kk[tid - 64] > 0 ? sh->first_tiles * kKeys : 0;
      }
      check<G>(buf, cap, m == 0, m >= max_stretch, sh, sw, lane);
      if (sh->stop) {
        if (m >= max_stretch && !sh->ended && !*abort_flag && tid == 64)
          raise_flag(a.status, kErrInternal);
        break;
      }
    }
    if constexpr (MASS) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float m2 = __shfl_xor_sync(0xFFFFFFFFu, ml[h].m, off);
          const float l2 = __shfl_xor_sync(0xFFFFFFFFu, ml[h].l, off);
          ml[h].merge(m2, l2);
        }
        if (lane == 0) sh->ml[sw][h] = make_float2(ml[h].m, ml[h].l);
      }
      SelBar::sync();
      if (tid - 64 < G) {
        const int h = tid - 64;
        Lse2 c;
        for (int w = 0; w < kSelW; ++w) c.merge(sh->ml[w][h].x, sh->ml[w][h].y);
        const size_t lst =
            ((size_t)b * a.Hq + (size_t)g * G + h) * a.nchunks + worker;
        a.cand_ml[lst] = make_float2(c.m, c.l);
      }
    }
    // this worker's best keys per q-head; empty slots get key 0.  With
    // k <= 128 a list starts with its r best keys, largest first, for the
    // head's m = min(k_h, candidate positions) and r = ceil(m / workers):
    // the merge takes a floor from those when r <= kDecodeTopR.
    if (a.k <= 128) {
      if (sw < G) {
        const int h = sw;
        uint64_t* out =
            a.cand + (((size_t)b * a.Hq + (size_t)g * G + h) * a.nchunks +
                      worker) * a.k;
        const int cnt = sh->cnt[h];
        // the head's candidates in this cache: positions max(1, pos0) ..
        // min(hi_h, pos0 + L - 1)
        const int nc = max(0, min(hi_h[h], pos0 + L - 1) - max(1, pos0) + 1);
        const int mh = min(sh->kk[h], nc);
        const int r = mh > 0 ? (mh + nworkers - 1) / nworkers : 0;
        uint64_t v[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int e = t * 32 + lane;
          v[t] = e < cnt ? buf[(size_t)h * cap + e] : 0ull;
        }
        int w = 0;
        if (r <= kDecodeTopR) {
#pragma unroll 1
          for (; w < r; ++w) {
            const uint64_t mx =
                warp_max_u64(max(max(v[0], v[1]), max(v[2], v[3])));
            if (lane == 0) out[w] = mx;
#pragma unroll
            for (int t = 0; t < 4; ++t) v[t] = v[t] == mx ? 0ull : v[t];
          }
        }
        const uint32_t below = (1u << lane) - 1u;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const bool keep = v[t] != 0ull;
          const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
          if (keep) out[w + __popc(bal & below)] = v[t];
          w += __popc(bal);
        }
        for (int e = w + lane; e < a.k; e += 32) out[e] = 0ull;
      }
    } else {
      for (int e = tid - 64; e < G * a.k; e += kSelT) {
        const int h = e / a.k, r = e - h * a.k;
        const size_t lst =
            ((size_t)b * a.Hq + (size_t)g * G + h) * a.nchunks + worker;
        a.cand[lst * a.k + r] =
            r < sh->cnt[h] ? buf[(size_t)h * cap + r] : 0ull;
      }
    }
  }
  __syncwarp();  // reconverge single-lane roles before the CTA barrier
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// Shared memory: q rows, the staging ring and per-list candidate buffers of
// k + 512 + slack keys.  Two CTAs per SM when they fit (two stages), else
// one CTA with up to four stages; what is left goes to insert slack.
template <int D, int G>
bool plan(int k, int* cap, int* nst, size_t* bytes) {
  const size_t fixed = Lay<D>::k_off + 1024;  // + the manual alignment
  const size_t min_lists = (size_t)G * 8 * (k + kSubKeys + kMinSlack);
  size_t budget = kSmemTwo - sizeof(Shared<G>);
  long st = 2;
  if (fixed + 2 * kStage + min_lists > budget) {
    budget = kSmemOne - sizeof(Shared<G>);
    st = (long)((budget - fixed - min_lists) / kStage);
    if (st > kMaxSt) st = kMaxSt;
  }
  if (st < 2) return false;
  const size_t rem = budget - fixed - (size_t)st * kStage;
  long slack = (long)(rem / (8 * G)) - k - kSubKeys;
  if (slack > kMaxSlack) slack = kMaxSlack;
  if (slack < kMinSlack) return false;
  *cap = k + kSubKeys + (int)slack;
  *nst = (int)st;
  *bytes = fixed + (size_t)st * kStage + (size_t)G * 8 * (size_t)(*cap);
  return true;
}

template <int D, int G>
cudaError_t launch_g(DecodeArgs a, bool mass, cudaStream_t s) {
  size_t smem;
  if (!plan<D, G>(a.k, &a.cap, &a.nstages, &smem)) return cudaErrorNotSupported;
  CUtensorMap tq, tk;
  int maps3d = 0;
  const uint64_t qrows = (uint64_t)a.B * a.Hq;
  const uint64_t krows = (uint64_t)a.B * a.Hkv * a.L;
  if (!make_tmap_2d(&tq, a.q, qrows, D, kN)) return cudaErrorInvalidValue;
  if (D == 64) {
    if (!make_tmap_2d(&tk, a.K, krows, D, 2 * kKeys)) return cudaErrorInvalidValue;
  } else if (make_tmap_3d(&tk, a.K, krows, kKeys)) {
    maps3d = 1;
  } else if (!make_tmap_2d(&tk, a.K, krows, D, kKeys)) {
    return cudaErrorInvalidValue;
  }
  auto kern = mass ? decode_score_topk_tc<D, G, true>
                   : decode_score_topk_tc<D, G, false>;
  cudaError_t e = ensure_smem(kern, smem, true);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nchunks, a.Hkv, a.B);
  prof_before(s, "decode_score_topk");
  kern<<<grid, kThreads, smem, s>>>(tq, tk, a, maps3d);
  prof_after(s);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dd(const DecodeArgs& a, bool mass, cudaStream_t s) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_g<D, 1>(a, mass, s);
    case 2: return launch_g<D, 2>(a, mass, s);
    case 4: return launch_g<D, 4>(a, mass, s);
    case 8: return launch_g<D, 8>(a, mass, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t decode_score_tc_launch(const DecodeArgs& a, int d, bool mass,
                                   cudaStream_t s) {
  if (d == 64) return launch_dd<64>(a, mass, s);
  if (d == 128) return launch_dd<128>(a, mass, s);
  return cudaErrorInvalidValue;
}

}  // namespace ca

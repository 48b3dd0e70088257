// Decode path: one query per (batch, q-head) at position L-1 against an
// L-long KV cache.  "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质",
// §2.1 Definition 1 (C_i for the last row), §2.2.3 (Dynamic Top-k), §2.4
// Corollary 3 (per-query window), §5.2.2 (select, then attend on the subset).
//
// Launch 1, decode_score_topk: grid (chunks, Hkv, B), about two CTAs per SM.
// With bf16 inputs the tensor-core pass (decode_tc.cu) runs instead, with
// the same outputs; this CUDA-core pass serves fp32 inputs.  One producer
// thread streams the chunk's contiguous K rows into a ring of 32 KiB
// shared-memory stages with bulk asynchronous copies (no multicast), so the
// loads stay deep in flight whatever the compute warps are doing.  Eight
// compute warps read each K row once from shared memory (8 lanes per row,
// 16-byte reads, conflict-free), score all G = Hq/Hkv q-heads of the group
// from the same bytes with packed fp32 FMAs, and keep a per-head candidate
// buffer in shared memory behind a threshold that only rises.  Buffers are
// cut back to exactly the best k keys by a radix select over the compute
// warps; the chunk's best k keys per q-head go to the workspace.  The union
// of the lists contains the global Top-k, since every global Top-k member
// is among the best k of its own chunk.
//
// Launch 2, decode_merge_attend: grid (Hq, B).  Every warp first gathers
// anchor and window rows into its fp32 online softmax while the score grid
// drains (they do not depend on the selection); then half of the CTA merges
// the lists into the exact Top-k (for k <= 128: a floor from each list's
// best few keys, the exact m-th best of the keys at or above it, ranks for
// ascending positions; else a radix select); then all warps accumulate the
// Top-k rows, whose scores come with their keys, and the per-warp softmax
// states are combined.
#include "common.cuh"
#include "decode.cuh"
#include "launch.cuh"
#include "profile.cuh"
#include "select.cuh"
#include "sm100.cuh"
#include "warp_sort.cuh"

namespace ca {

namespace {

constexpr int kComputeWarps = 8;
constexpr int kCompute = kComputeWarps * 32;  // compute threads
constexpr int kThreads = kCompute + 32;       // + one producer warp
// Stage size: each stage is waited for and released by every compute warp,
// so a larger stage spreads that handshake over more keys (32 KiB x 2
// stages measured 8% faster at 131K and 12% at 1M than 16 KiB x 3).
constexpr int kStageBytes = 32768;
constexpr int kTwoCtaStages = 2;  // ring depth when two CTAs share an SM
constexpr int kMaxStages = 6;  // K staging ring depth (chosen per launch)
constexpr int kSub = 512;     // keys between candidate-buffer checks
constexpr int kMinSlack = 256;      // smallest insert room kept after a cut
constexpr int kMaxSlack = 2048;     // largest useful insert room
constexpr size_t kSmemTwoCtas = 108 * 1024;   // two CTAs per SM, with margin
constexpr size_t kSmemOneCta = 227 * 1024;
constexpr int kMergeThreads = 512;
using ComputeBar = GroupBarrier<1, kCompute>;
using MergeBar = GroupBarrier<1, 256>;

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
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t never;  // failure-path test hook: a barrier nothing signals
  uint64_t thr[G];
  int cnt[G];
  int kk[G];       // Top-k size of each q-head of the group
  int hi[G];       // last candidate position of each q-head
  int abort;
  uint32_t hist[G][256];  // one radix histogram per list (per cutting warp)
  float2 ml[8][G];        // per compute warp and head: (max, sum) of the
                          // candidates' log2-scaled scores (mass reports)
};

// At a check point (all inserts of the stretch done): warp h cuts list h
// down to its head's k keys when it holds more than the limit: that k after
// the first stretch (so that a useful threshold exists early), else the
// insert room the next stretch needs (`later`: long chunks also cut once a
// list passes 4k keys, which raises the admission threshold early).
// Barriers on both sides keep every compute warp from inserting while a list
// is being cut.
template <int G>
__device__ __forceinline__ void check_lists(uint64_t* buf, int cap, bool first,
                                            bool long_chunk, TopkShared<G>* sh,
                                            int warp, int lane) {
  ComputeBar::sync();
  if (warp < G) {
    const int n = sh->cnt[warp];
    const int kk = sh->kk[warp];
    const int limit = first ? kk
                      : (long_chunk ? min(cap - kSub, 4 * kk) : cap - kSub);
    if (kk > 0 && n > limit && n > kk) {
      const uint64_t T = warp_cut(buf + (size_t)warp * cap, n, kk,
                                  sh->hist[warp], lane);
      if (lane == 0) {
        sh->cnt[warp] = kk;
        sh->thr[warp] = T;
      }
    }
  }
  ComputeBar::sync();
}

template <typename T, int D, int G>
struct ScoreCfg {
  static constexpr int VEC = Elem<T>::kPer16B;   // elements per 16 bytes
  static constexpr int ROWB = D * (int)sizeof(T);
  static constexpr int CPL = ROWB / 16 / 8;       // 16-byte pieces per lane
  static constexpr int PPL = CPL * VEC / 2;       // element pairs per lane
  static constexpr int KPR = 4 * kComputeWarps;   // keys per round
  // a stage holds a whole number of rounds, about kStageBytes
  static constexpr int RB = KPR * ROWB;           // bytes per round
  static constexpr int STAGE = (kStageBytes / RB > 0 ? kStageBytes / RB : 1) * RB;
  static constexpr int R = STAGE / ROWB;          // K rows per stage
  static constexpr int ROUNDS = R / KPR;
  static constexpr int SUB_ST = kSub / R;         // stages per buffer check
  static_assert(CPL >= 1 && R % KPR == 0 && kSub % R == 0, "tiling");
};

// Unpack one 16-byte piece into element pairs.
template <typename T>
__device__ __forceinline__ void pairs16(const uint4& v, float2* p);
template <>
__device__ __forceinline__ void pairs16<__nv_bfloat16>(const uint4& v,
                                                       float2* p) {
  p[0] = make_float2(bf16lo(v.x), bf16hi(v.x));
  p[1] = make_float2(bf16lo(v.y), bf16hi(v.y));
  p[2] = make_float2(bf16lo(v.z), bf16hi(v.z));
  p[3] = make_float2(bf16lo(v.w), bf16hi(v.w));
}
template <>
__device__ __forceinline__ void pairs16<float>(const uint4& v, float2* p) {
  p[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
  p[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}

template <typename T, int D, int G, bool MASS>
__global__ void __launch_bounds__(kThreads, G >= 8 ? 1 : 2)
decode_score_topk(DecodeArgs a) {
  using C = ScoreCfg<T, D, G>;
  constexpr int VEC = C::VEC, CPL = C::CPL, PPL = C::PPL, R = C::R;
  extern __shared__ __align__(128) unsigned char smem[];
  const int k = a.k;
  const int cap = a.cap;  // per-list buffer: k + kSub + slack keys
  const int kStages = a.nstages;
  unsigned char* stages = smem;                                  // ring
  uint64_t* buf = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * C::STAGE);
  TopkShared<G>* sh = reinterpret_cast<TopkShared<G>*>(buf + (size_t)G * cap);

  // Let the merge kernel (launched as a programmatic dependent) start its
  // independent prologue on SMs this grid releases.
  asm volatile("griddepcontrol.launch_dependents;");
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L;  // positions fit in 31 bits (int L in the ABI)
  // per q-head of the group: window (W_i per batch, else W_h per head, else
  // W), last candidate position and Top-k size; the CTA streams up to the
  // largest last candidate position of the group
  int hi = -1;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const int hq = g * G + h;
    const bool rep = chunk == 0 && tid == 0;
    const int hh = (L - 1) - row_window(a.W_i, b, a.W_h, hq, a.W, L,
                                        a.status, rep);
    hi = max(hi, hh);
    if (tid == 0) {
      sh->hi[h] = hh;
      sh->kk[h] = head_k(a.k_h, hq, a.k, a.status, rep);
    }
  }
  const int j0 = chunk * a.chunk_len;
  const int c0 = j0 < 1 ? 1 : j0;
  const int c1 = (j0 + a.chunk_len < hi + 1) ? j0 + a.chunk_len : hi + 1;
  const int nrows = c1 > c0 ? c1 - c0 : 0;
  const int nst = (nrows + R - 1) / R;
  const T* Kg = reinterpret_cast<const T*>(a.K) +
                ((size_t)b * a.Hkv + g) * (size_t)L * D;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      sm100::mbar_init(&sh->full[s], 1);
      sm100::mbar_init(&sh->empty[s], kComputeWarps);
    }
    sm100::mbar_init(&sh->never, 1);
    for (int h = 0; h < G; ++h) {
      sh->cnt[h] = 0;
      // a head with k = 0 admits nothing
      sh->thr[h] = sh->kk[h] > 0 ? 0ull : ~0ull;
    }
    sh->abort = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &sh->abort;

  if (warp == kComputeWarps) {
    // ------------------------------------------------ producer
    if (lane == 0 && nst > 0) {
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;  // parity of the ring pass of stage s
      for (int t = 0; t < nst; ++t) {
        if (t >= kStages &&
            !sm100::wait_or_abort(&sh->empty[s], ph ^ 1, abort_flag, a.status,
                                  a.wait_ns))
          break;
        const int r0 = c0 + t * R;
        const int left = nrows - t * R;
        const int rows = left < R ? left : R;
        const uint32_t bytes = (uint32_t)rows * C::ROWB;
        sm100::mbar_arrive_expect_tx(&sh->full[s], bytes);
        sm100::bulk_load(stages + s * C::STAGE, Kg + (size_t)r0 * D, bytes,
                         &sh->full[s]);
        issued = t + 1;
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
      // every copy this thread started must land before the CTA exits
      for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
        if (!sm100::mbar_wait(&sh->full[t % kStages], (t / kStages) & 1,
                              kDrainWaitNs))
          raise_flag(a.status, kErrTimeout);
    }
    return;
  }

  // -------------------------------------------------- compute warps
  if (a.stall_ns && warp == 0) {
    // Failure-path test hook: wait on a barrier that nothing signals, so the
    // wait runs out, raises the time-out flag and aborts every wait of the
    // CTA; the kernel then leaves through its normal path.
    sm100::wait_or_abort(&sh->never, 0, abort_flag, a.status, a.stall_ns);
  }
  const int l8 = lane & 7, ks = lane >> 3;
  float2 q2[G][PPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const T* qh = reinterpret_cast<const T*>(a.q) +
                  ((size_t)b * a.Hq + (size_t)g * G + h) * D;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(qh + (l8 + 8 * c) * VEC);
      pairs16<T>(v, &q2[h][c * (VEC / 2)]);
    }
  }
  const int myh = reduce_head<G>(l8);
  const bool owner = reduce_owner<G>(l8);
  const int my_hi = sh->hi[myh];
  // Long chunks cut their lists again once they pass 4k keys, which raises
  // the admission threshold early (measured: 1M context 5% faster); short
  // chunks cut only when a list runs out of room (131K: the extra cuts cost
  // more than they save).
  const bool long_chunk = a.chunk_len >= 16 * kSub;
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);  // log2(e)/sqrt(d)
  Lse2 ml;                   // candidates' scaled scores (mass reports)
  uint64_t thr = 0ull;       // admission threshold key (0: admit all)
  float thr_f = -INFINITY;   // its score, for a cheap float pre-filter
  const int first_keys = nrows < kSub ? nrows : kSub;

  int s = 0;
  uint32_t ph = 0;  // parity of the ring pass of stage s
#pragma unroll 1
  for (int t = 0; t < nst; ++t) {
    if (t % C::SUB_ST == 0) {
      thr = sh->thr[myh];
      thr_f = thr ? key_score(thr) : -INFINITY;
    }
    const bool ok = __all_sync(
        0xFFFFFFFFu, sm100::wait_or_abort(&sh->full[s], ph, abort_flag,
                                          a.status, a.wait_ns));
    if (ok) {
      const unsigned char* st = stages + s * C::STAGE;
      const int rbase = c0 + t * R;
#pragma unroll
      for (int rd = 0; rd < C::ROUNDS; ++rd) {
        const int rloc = rd * C::KPR + warp * 4 + ks;
        const int j = rbase + rloc;
        uint4 piece[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          piece[c] = *reinterpret_cast<const uint4*>(st + rloc * C::ROWB +
                                                     (l8 + 8 * c) * 16);
        float2 acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          float2 kp[VEC / 2];
          pairs16<T>(piece[c], kp);
#pragma unroll
          for (int p = 0; p < VEC / 2; ++p)
#pragma unroll
            for (int h = 0; h < G; ++h)
              acc[h] = __ffma2_rn(q2[h][c * (VEC / 2) + p], kp[p], acc[h]);
        }
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = acc[h].x + acc[h].y;
        const float sc = group_reduce<G>(part, lane);
        if constexpr (MASS) {
          if (owner && j < c1 && j <= my_hi) ml.add(sc * sl2);
        }
        if (t < C::SUB_ST) {
          // first stretch: every key goes in, at its own slot (a position
          // past this head's window start goes in as an empty key)
          if (owner && j < c1)
            buf[(size_t)myh * cap + (j - c0)] =
                j <= my_hi ? make_key(sc, (uint32_t)j) : 0ull;
        } else {
          // rare once a threshold exists (a warp vote in front of this
          // branch measured slower)
          const bool cand = owner && j < c1 && j <= my_hi && sc >= thr_f;
          if (cand) {
            const uint64_t key = make_key(sc, (uint32_t)j);
            if (key > thr) {
              const int pos = atomicAdd(&sh->cnt[myh], 1);
              buf[(size_t)myh * cap + pos] = key;
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&sh->empty[s]);
    if (++s == kStages) {
      s = 0;
      ph ^= 1;
    }
    if (t % C::SUB_ST == C::SUB_ST - 1 || t == nst - 1) {
      if (t < C::SUB_ST) {
        // the first stretch filled slots 0..first_keys-1 of every list
        ComputeBar::sync();
        if (tid < G) sh->cnt[tid] = sh->kk[tid] > 0 ? first_keys : 0;
      }
      // the first cut sets a useful threshold; later cuts keep room for the
      // next stretch of keys
      check_lists<G>(buf, cap, t < C::SUB_ST, long_chunk, sh, warp, lane);
    }
  }
  check_lists<G>(buf, cap, true, long_chunk, sh, warp, lane);
  if constexpr (MASS) {
    // lanes of one head (the same l8 in each key slot ks) combine, then the
    // warps
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
      const float m2 = __shfl_xor_sync(0xFFFFFFFFu, ml.m, off);
      const float l2 = __shfl_xor_sync(0xFFFFFFFFu, ml.l, off);
      ml.merge(m2, l2);
    }
    if (owner && ks == 0) sh->ml[warp][myh] = make_float2(ml.m, ml.l);
    ComputeBar::sync();
    if (tid < G) {
      Lse2 c;
      for (int w = 0; w < kComputeWarps; ++w)
        c.merge(sh->ml[w][tid].x, sh->ml[w][tid].y);
      const size_t lst =
          ((size_t)b * a.Hq + (size_t)g * G + tid) * a.nchunks + chunk;
      a.cand_ml[lst] = make_float2(c.m, c.l);
    }
  }

  // write this chunk's best keys per q-head; empty slots get key 0
#pragma unroll 1
  for (int h = 0; h < G; ++h) {
    const size_t lst = ((size_t)b * a.Hq + (size_t)g * G + h) * a.nchunks + chunk;
    uint64_t* out = a.cand + lst * k;
    const int cnt = sh->cnt[h];
    for (int e = tid; e < k; e += kCompute)
      out[e] = e < cnt ? buf[(size_t)h * cap + e] : 0ull;
  }
}

// Online-softmax state of one warp: running max m (log2 domain), sum l and
// the lane's DL output dims.
template <int DL>
struct Online {
  float m = -INFINITY, l = 0.f, o[DL];
  __device__ __forceinline__ Online() {
#pragma unroll
    for (int e = 0; e < DL; ++e) o[e] = 0.f;
  }
  __device__ __forceinline__ void add(float s, const float* v) {
    const float mn = fmaxf(m, s);
    const float corr = exp2f(m - mn);
    const float p = exp2f(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int e = 0; e < DL; ++e) o[e] = fmaf(p, v[e], o[e] * corr);
    m = mn;
  }
};

// How many of a[beg..end) exceed x: eight independent loads per step, so
// that one thread's count is not a chain of dependent shared-memory reads.
__device__ __forceinline__ int count_above(const uint64_t* a, int beg, int end,
                                           uint64_t x) {
  int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
  int f = beg;
#pragma unroll 1
  for (; f + 8 <= end; f += 8) {
    const uint64_t v0 = a[f], v1 = a[f + 1], v2 = a[f + 2], v3 = a[f + 3];
    const uint64_t v4 = a[f + 4], v5 = a[f + 5], v6 = a[f + 6], v7 = a[f + 7];
    c0 += (v0 > x) + (v4 > x);
    c1 += (v1 > x) + (v5 > x);
    c2 += (v2 > x) + (v6 > x);
    c3 += (v3 > x) + (v7 > x);
  }
#pragma unroll 1
  for (; f < end; ++f) c0 += a[f] > x;
  return c0 + c1 + c2 + c3;
}

// How many keys of a[0..n) have a position below j (the same eight-wide
// steps as count_above).
__device__ __forceinline__ int count_pos_below(const uint64_t* a, int n,
                                               uint32_t j) {
  int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
  int f = 0;
#pragma unroll 1
  for (; f + 8 <= n; f += 8) {
    const uint32_t v0 = key_index(a[f]), v1 = key_index(a[f + 1]);
    const uint32_t v2 = key_index(a[f + 2]), v3 = key_index(a[f + 3]);
    const uint32_t v4 = key_index(a[f + 4]), v5 = key_index(a[f + 5]);
    const uint32_t v6 = key_index(a[f + 6]), v7 = key_index(a[f + 7]);
    c0 += (v0 < j) + (v4 < j);
    c1 += (v1 < j) + (v5 < j);
    c2 += (v2 < j) + (v6 < j);
    c3 += (v3 < j) + (v7 < j);
  }
#pragma unroll 1
  for (; f < n; ++f) c0 += key_index(a[f]) < j;
  return c0 + c1 + c2 + c3;
}

// The r best keys of one worker list lst[0..k) (k <= 128, read by one warp)
// to out[0..r), largest first, 0 once the list runs out.
__device__ __forceinline__ void list_top_r(const uint64_t* lst, int k, int r,
                                           uint64_t* out, int lane) {
  uint64_t v[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int e = t * 32 + lane;
    v[t] = e < k ? lst[e] : 0ull;
  }
#pragma unroll 1
  for (int q = 0; q < r; ++q) {
    const uint64_t mx = warp_max_u64(max(max(v[0], v[1]), max(v[2], v[3])));
    if (lane == 0) out[q] = mx;
#pragma unroll
    for (int t = 0; t < 4; ++t) v[t] = v[t] == mx ? 0ull : v[t];
  }
}

template <typename T, int D, typename TO>
__global__ void __launch_bounds__(kMergeThreads)
decode_merge_attend(DecodeArgs a) {
  constexpr int DL = D / 32;  // head dims per lane in the gathers
  constexpr int NW = kMergeThreads / 32;
  static_assert(NW <= 32, "one lane per warp in the final combine");
  constexpr int UG = 4;       // rows in flight per warp
  extern __shared__ __align__(128) unsigned char smem[];
  const int k = a.k;
  const int ncand = a.nchunks * k;
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem);           // [ncand]
  uint64_t* surv = cand + ncand;                                // [ncand]
  uint64_t* pairs = surv + ncand;                               // [128]
  uint32_t* topj = reinterpret_cast<uint32_t*>(pairs + 128);    // [kpow2]
  float* tops = reinterpret_cast<float*>(topj + a.kpow2);       // [kpow2]
  SelectState<1>* st = reinterpret_cast<SelectState<1>*>(tops + a.kpow2);
  int* s_cnt = reinterpret_cast<int*>(st + 1);                  // [512]
  __shared__ int s_n, s_kk, s_m;
  __shared__ uint64_t s_T, s_t0[8];
  __shared__ float s_mw[NW], s_lw[NW];
  __shared__ float s_ow[NW][D];
  __shared__ float s_wm[NW], s_wl[NW], s_s0;  // window+anchor states; anchor score
  __shared__ int s_seg[8];                     // survivors per merge warp

  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int gtid = tid & 255, gw = warp & 7;
  const int g = h / (a.Hq / a.Hkv);
  // this cache holds the sequence positions [p0, p1); the query is at i
  const int64_t L = a.L, i = (int64_t)a.Lg - 1;
  const int64_t p0 = a.pos0, p1 = p0 + L;
  const bool select_only = a.mode == kShardSelect;
  const bool shard_part = a.mode == kShardAttend;
  const int Wb = row_window(a.W_i, b, a.W_h, h, a.W, a.Lg, a.status,
                            tid == 0);
  const int kh = head_k(a.k_h, h, k, a.status, tid == 0);
  const bool want_mass = a.mass != nullptr || a.lse != nullptr;
  const int64_t lo = (i - Wb + 1) > 0 ? (i - Wb + 1) : 0;
  const int64_t ncand_pos = (i - Wb) > 0 ? (i - Wb) : 0;  // |[1, i-W]|
  // selected keys: m of the sequence's candidates, or, when selecting for
  // one shard, of the candidates in this cache
  const int64_t ncand_here =
      select_only ? max((int64_t)0, min(i - Wb, p1 - 1) - max((int64_t)1, p0) + 1)
                  : ncand_pos;
  const int m = (int)(kh < ncand_here ? kh : ncand_here);
  const int anc = lo > 0 ? 1 : 0;
  const int64_t count = anc + m + (i - lo + 1);
  // the anchor and window rows in this cache: the anchor when p0 = 0, then
  // positions [wlo, whi]
  const int anc_here = (anc && p0 == 0) ? 1 : 0;
  const int64_t wlo = lo > p0 ? lo : p0, whi = i < p1 - 1 ? i : p1 - 1;
  const int64_t nwin_here =
      select_only ? 0 : anc_here + (whi >= wlo ? whi - wlo + 1 : 0);

  const T* qh = reinterpret_cast<const T*>(a.q) + ((size_t)b * a.Hq + h) * D;
  float qv[DL];
  load_f32<T, DL>(qh + lane * DL, qv);
  // row r of this cache is sequence position p0 + r
  const T* Kg = reinterpret_cast<const T*>(a.K) +
                ((size_t)b * a.Hkv + g) * (size_t)L * D + lane * DL;
  const T* Vg = reinterpret_cast<const T*>(a.V) +
                ((size_t)b * a.Hkv + g) * (size_t)L * D + lane * DL;
  auto row_of = [&](int64_t j) -> size_t { return (size_t)(j - p0) * D; };
  const float sl2 = 1.4426950408889634f / sqrtf((float)D);  // log2(e)/sqrt(d)
  Online<DL> acc;
  {
    // ask L2 for the anchor and (the first 512) window rows of K and V at
    // once, so that the window gathers below wait for one L2 round trip
    // rather than one HBM round trip per batch of rows
    constexpr int kLines = D * (int)sizeof(T) / 128;
    const int64_t nwin = min(nwin_here, (int64_t)512);
    const char* kb = reinterpret_cast<const char*>(Kg - lane * DL);
    const char* vb = reinterpret_cast<const char*>(Vg - lane * DL);
    for (int64_t e = tid; e < nwin * kLines; e += kMergeThreads) {
      const int64_t row = e / kLines, ln = e % kLines;
      const int64_t j = (anc_here && row == 0) ? 0 : wlo + (row - anc_here);
      const size_t o = row_of(j) * sizeof(T) + (size_t)ln * 128;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(kb + o));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(vb + o));
    }
  }

  // A shard selection attends to nothing: warps 8-15 leave before any
  // CTA-wide barrier (warps 0-7 leave after the selection).
  if (select_only && warp >= 8) return;
  if (!select_only) {
    // ---------------- anchor and window rows, every warp: they do not
    // depend on the selection, and the score grid is still draining
    const int64_t nwin = nwin_here;
#pragma unroll 1
    for (int64_t e0 = warp; e0 < nwin; e0 += NW * UG) {
      float kf[UG][DL], vf[UG][DL];
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        const int64_t e = e0 + NW * u;
        int64_t j = p0;
        if (e < nwin) j = (anc_here && e == 0) ? 0 : wlo + (e - anc_here);
        load_f32<T, DL>(Kg + row_of(j), kf[u]);
        load_f32<T, DL>(Vg + row_of(j), vf[u]);
      }
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        if (e0 + NW * u >= nwin) break;  // warp-uniform
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) dot = fmaf(qv[e], kf[u][e], dot);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
        acc.add(dot * sl2, vf[u]);
      }
    }
    if (want_mass) {
      // the window + anchor part alone, and the anchor's own score (inside
      // the window when the window reaches position 0)
      if (lane == 0) {
        s_wm[warp] = acc.m;
        s_wl[warp] = acc.l;
      }
      if (warp == NW - 1) {
        float k0[DL];
        load_f32<T, DL>(Kg, k0);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) dot = fmaf(qv[e], k0[e], dot);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
        if (lane == 0) s_s0 = dot * sl2;
      }
    }
  }
  if (warp < 8) {
    // ---------------- merge the worker lists into the exact Top-k
    // list c of this q-head: k keys at src + c * list_stride (the workspace
    // lists of the score pass, or every shard's keys)
    const uint64_t* src = a.cand + ((size_t)b * a.Hq + h) * a.head_stride;
    const size_t lstride = a.list_stride;
    const bool async_ok = lstride == (size_t)k && (((uintptr_t)src) & 15u) == 0;
    // k <= 128: a floor first.  With each list's r = ceil(m / lists) best
    // keys, the m-th largest of those, F, has m keys at or above it, so the
    // global m-th best key is >= F and only keys >= F can be selected
    // (about m survive).  The tensor-core pass writes those r keys at the
    // front of each list.  F and the exact selection among the survivors
    // are found by ranks (a key's number of larger keys), counted by
    // several threads per key: no barrier per step, and loops that stay
    // rolled.
    const bool fast = a.kpow2 <= 128;
    const int r = m > 0 ? (m + a.nchunks - 1) / a.nchunks : 0;
    const int nt = a.nchunks * r;
    const bool use_floor = fast && m > 0 && r <= kDecodeTopR && nt <= 512;
    const bool lead = use_floor && a.top_first;
    {
      // The lists are written by the score kernel, which may still be
      // finishing: wait for it (programmatic dependent launch).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      // every list into shared memory at once: 16-byte asynchronous copies
      // when the lists are contiguous (the list area of a head starts
      // 16-byte aligned: k keys per list, 8 bytes each, and the workspace
      // lists start at a 256-byte boundary; an odd k leaves the head's area
      // 8-byte aligned: then plain loads)
      if (lstride != (size_t)k) {
        for (int e = gtid; e < ncand; e += 256)
          cand[e] = src[(size_t)(e / k) * lstride + e % k];
      } else if (async_ok) {
        for (int e = 2 * gtid; e + 1 < ncand; e += 512) {
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                           (uint32_t)__cvta_generic_to_shared(cand + e)),
                       "l"(src + e)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if ((ncand & 1) && gtid == 0) cand[ncand - 1] = src[ncand - 1];
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      } else {
        for (int e = gtid; e < ncand; e += 256) cand[e] = src[e];
      }
    }
    if (gtid == 0) {
      s_n = 0;
      s_m = 0;
      s_kk = m > 0 ? m : 1;
      s_T = fast ? 1ull : 0ull;  // 1: no floor, real keys only
    }
    MergeBar::sync();
    if (fast) {
      if (use_floor) {
        // the leading keys: list c's q-th at lk[c * ls + q]
        if (!lead) {
          for (int c = gw; c < a.nchunks; c += 8)
            list_top_r(cand + (size_t)c * k, k, r, surv + (size_t)c * r, lane);
          MergeBar::sync();
        }
        // the nt leading keys, contiguous in surv (list_top_r wrote them so)
        if (lead)
          for (int e = gtid; e < nt; e += 256)
            surv[e] = cand[(size_t)(e / r) * k + e % r];
        for (int e = gtid; e < nt; e += 256) s_cnt[e] = 0;
        MergeBar::sync();
        // each key's rank counted in S slices of the others, by S threads
        const int S = nt < 256 ? 256 / nt : 1;
        const int slice = (nt + S - 1) / S;
        for (int u = gtid; u < nt * S; u += 256) {
          const int e = u % nt, sl = u / nt;
          const uint64_t my = surv[e];
          if (my == 0ull) continue;
          const int part =
              count_above(surv, sl * slice, min(nt, (sl + 1) * slice), my);
          if (part) atomicAdd(&s_cnt[e], part);
        }
        MergeBar::sync();
        for (int e = gtid; e < nt; e += 256) {
          const uint64_t my = surv[e];
          if (my != 0ull && s_cnt[e] == m - 1) s_T = my;  // m - 1 above it
        }
        MergeBar::sync();
      }
      const uint64_t F = s_T;
      // survivors (keys >= F): warp gw packs those of its slice to the same
      // slice of surv, and asks L2 for their V rows, which the Top-k
      // accumulation reads next
      const int per = (ncand + 7) / 8;
      if (m > 0) {
        const int beg = min(ncand, gw * per), end = min(ncand, beg + per);
        int w = 0;
        for (int e0 = beg; e0 < end; e0 += 32) {
          const int e = e0 + lane;
          const uint64_t key = e < end ? cand[e] : 0ull;
          const bool keep = key >= F;  // F >= 1: real keys only
          const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
          if (keep) {
            const int slot = beg + w + __popc(bal & ((1u << lane) - 1u));
            if (in_bounds(slot < end, a.status)) surv[slot] = key;
            if (!select_only) {
              const char* row = reinterpret_cast<const char*>(
                  Vg - lane * DL + row_of(key_index(key)));
              for (int o = 0; o < D * (int)sizeof(T); o += 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(row + o));
            }
          }
          w += __popc(bal);
        }
        if (lane == 0) s_seg[gw] = w;
      }
      MergeBar::sync();
      if (m > 0) {
        int off[8], ns = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          off[c] = ns;
          ns += s_seg[c];
        }
        // survivor e (in segment order): segment c holds s_seg[c] keys at
        // surv + c * per
        auto gather = [&](int e) -> uint64_t {
          int c = 0;
#pragma unroll
          for (int q = 1; q < 8; ++q) c = e >= off[q] ? q : c;
          return surv[(size_t)c * per + (e - off[c])];
        };
        // the survivors, contiguous, into cand (no longer read)
        for (int e = gtid; e < ns; e += 256) {
          cand[e] = gather(e);
          if (e < 512) s_cnt[e] = 0;
        }
        if (gtid == 0) s_n = ns;
        MergeBar::sync();
        if (ns <= 512) {
          // a survivor with fewer than m larger survivors is selected, at
          // the slot of its rank (so pairs holds them largest first); each
          // rank is counted by S threads over slices of the survivors
          const int S = ns < 256 ? 256 / ns : 1;
          const int slice = (ns + S - 1) / S;
          for (int u = gtid; u < ns * S; u += 256) {
            const int e = u % ns, sl = u / ns;
            const int part = count_above(cand, sl * slice,
                                         min(ns, (sl + 1) * slice), cand[e]);
            if (part) atomicAdd(&s_cnt[e], part);
          }
          MergeBar::sync();
          for (int e = gtid; e < ns; e += 256)
            if (s_cnt[e] < m) pairs[s_cnt[e]] = cand[e];
          if (gtid == 0) s_m = min(ns, m);
        } else {
          // many survivors: radix select over the eight warps
          cta_select_thresholds<256, 1, MergeBar>(cand, 0, &s_n, &s_kk, &s_T,
                                                  st, gtid);
          for (int e = gtid; e < ns; e += 256) {
            const uint64_t key = cand[e];
            if (key >= s_T && key != 0ull) {
              const int p = atomicAdd(&s_m, 1);
              if (p < 128) pairs[p] = key;
            }
          }
        }
      }
      MergeBar::sync();
      // pairs[0..got) holds the selected keys
      const int got = min(min(s_m, m), 128);
      if (select_only) {
        // the shard's best keys, largest first (so that a list's leading
        // keys are its best), 0 after them
        uint64_t* out = a.keys_out + ((size_t)b * a.Hq + h) * k;
        if (gtid < got) {
          const uint64_t my = pairs[gtid];
          out[count_above(pairs, 0, got, my)] = my;
        }
        for (int e = got + gtid; e < k; e += 256) out[e] = 0ull;
        if (m > 0 && s_m != m && gtid == 0) raise_flag(a.status, kErrInternal);
        return;
      }
      // ascending positions: each selected key goes to its position's rank
      if (gtid < got) {
        const uint64_t my = pairs[gtid];
        const uint32_t jm = key_index(my);
        const int rank = count_pos_below(pairs, got, jm);
        topj[rank] = jm;
        tops[rank] = key_score(my);
      }
    } else {
      // Every chunk list holds its chunk's best k keys, so the largest of the
      // lists' smallest keys, T0, is at most the global k-th best key (the
      // chunk that has it alone holds k keys >= T0): only keys >= T0 can be
      // selected.  A list of a chunk with fewer than k candidates has empty
      // (0) slots and contributes 0.
      uint64_t t0 = 0ull;
      for (int c = gw; c < a.nchunks; c += 8) {
        uint64_t mn = ~0ull;
        for (int e = lane; e < kh; e += 32) mn = min(mn, cand[(size_t)c * k + e]);
  #pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        t0 = max(t0, mn);
      }
      if (lane == 0) s_t0[gw] = t0;
      MergeBar::sync();
      t0 = s_t0[0];
  #pragma unroll
      for (int w = 1; w < 8; ++w) t0 = max(t0, s_t0[w]);
      // keep the keys >= T0 (and real), packed to the front in any order: in
      // place, one round of 256 keys at a time (a round's keys are all read
      // before any of them is written, and the kept count never passes the
      // keys read so far)
      for (int e0 = 0; e0 < ncand; e0 += 256) {
        const int e = e0 + gtid;
        const uint64_t key = e < ncand ? cand[e] : 0ull;
        const bool keep = key != 0ull && key >= t0;
        MergeBar::sync();
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&s_n, __popc(bal));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        if (keep) cand[base + __popc(bal & ((1u << lane) - 1u))] = key;
      }
      MergeBar::sync();
      cta_select_thresholds<256, 1, MergeBar>(cand, 0, &s_n, &s_kk, &s_T, st,
                                              gtid);
      if (select_only) {
        // the shard's best keys, in no particular order, 0 after them
        uint64_t* out = a.keys_out + ((size_t)b * a.Hq + h) * k;
        if (m > 0) {
          for (int e = gtid; e < s_n; e += 256) {
            const uint64_t key = cand[e];
            if (key >= s_T && key != 0ull) {
              const int p = atomicAdd(&s_m, 1);
              if (p < m) out[p] = key;
              else raise_flag(a.status, kErrInternal);
            }
          }
        }
        MergeBar::sync();
        for (int e = min(s_m, m) + gtid; e < k; e += 256) out[e] = 0ull;
        if (m > 0 && s_m != m && gtid == 0) raise_flag(a.status, kErrInternal);
        return;
      }
      if (m > 0) {
        for (int e = gtid; e < s_n; e += 256) {
          const uint64_t key = cand[e];
          if (key >= s_T && key != 0ull) {
            const uint32_t j = key_index(key);
            const int p = atomicAdd(&s_m, 1);
            if (p < m && j >= 1 && (int64_t)j <= i - Wb) {
              topj[p] = j;
              tops[p] = key_score(key);
            } else {
              raise_flag(a.status, kErrInternal);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  const int got = s_m < m ? s_m : m;
  if (m > 0 && s_m != m && tid == 0) raise_flag(a.status, kErrInternal);
  // idx: C_i = {0} U sorted Top-k U [lo, i], ascending, -1 padded, and |C_i|
  auto write_idx = [&]() {
    int32_t* idx_row = a.idx + ((size_t)b * a.Hq + h) * a.C_max;
    if (count > a.C_max && tid == 0) raise_flag(a.status, kErrCmax);
    const int64_t wcount = count < a.C_max ? count : a.C_max;
    for (int64_t r = tid; r < a.C_max; r += kMergeThreads) {
      int32_t v;
      if (r >= wcount) v = -1;
      else if (r < anc) v = 0;
      else if (r < anc + m) v = (r - anc < got) ? (int32_t)topj[r - anc] : 0;
      else v = (int32_t)(lo + (r - anc - m));
      idx_row[r] = v;
    }
    if (tid == 0) a.idx_count[(size_t)b * a.Hq + h] = (int32_t)count;
  };
  // (k <= 128: topj is sorted already, so the writes overlap the gathers)
  if (a.kpow2 <= 128) write_idx();
  // Top-k rows, spread over all warps: the score travels with the key, so
  // only V is read (of the rows in this cache)
#pragma unroll 1
  for (int e0 = warp; e0 < got; e0 += NW * UG) {
    float vf[UG][DL];
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      const int e = e0 + NW * u;
      int64_t j = e < got ? (int64_t)topj[e] : p0;
      if (j < p0 || j >= p1) j = p0;
      load_f32<T, DL>(Vg + row_of(j), vf[u]);
    }
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      const int e = e0 + NW * u;
      if (e >= got) break;  // warp-uniform
      const int64_t j = topj[e];
      if (j >= p0 && j < p1) acc.add(tops[e] * sl2, vf[u]);
    }
  }
  if (lane == 0) {
    s_mw[warp] = acc.m;
    s_lw[warp] = acc.l;
  }
#pragma unroll
  for (int e = 0; e < DL; ++e) s_ow[warp][lane * DL + e] = acc.o[e];
  __syncthreads();  // every warp is done reading topj
  // C_i = {0} U sorted Top-k U [lo, i], ascending, for the idx output
  // (the k <= 128 path wrote it sorted already)
  if (warp == 0 && a.kpow2 > 128) warp_sort_prefix(topj, got, a.kpow2, lane);
  if (tid >= 32 && tid < 32 + D) {
    // lane w < NW of each combining warp holds warp w's scale 2^(m_w - M)
    // (0 for a warp that saw no row)
    const int dd = tid - 32;
    const float mw = lane < NW ? s_mw[lane] : -INFINITY;
    const float lw = lane < NW ? s_lw[lane] : 0.f;
    float M = mw;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, off));
    const float cw = lw != 0.f ? exp2f(mw - M) : 0.f;
    float l = lw * cw;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      o = fmaf(s_ow[w][dd], __shfl_sync(0xFFFFFFFFu, cw, w), o);
    if (shard_part) {
      // this shard's softmax state over its part of C_i: (max, sum, o) in
      // the log2 domain, o not yet divided by the sum (max = -inf, sum = 0
      // when no member of C_i lies here)
      float* pt = a.partial + ((size_t)b * a.Hq + h) * (D + 2);
      if (dd == 0) {
        pt[0] = M;
        pt[1] = l;
      }
      pt[2 + dd] = o;
    } else {
      TO* out = reinterpret_cast<TO*>(a.O) + ((size_t)b * a.Hq + h) * D;
      store_out<TO>(out + dd, o / l);
    }
  }
  if (want_mass && tid == 32 + D) {
    // masses over the full causal softmax: C (all warps), window + anchor
    // (every warp before the Top-k rows), and every candidate (the score
    // pass's per-chunk sums), in one frame
    Lse2 c, wa, cand;
    for (int w = 0; w < NW; ++w) c.merge(s_mw[w], s_lw[w]);
    for (int w = 0; w < NW; ++w) wa.merge(s_wm[w], s_wl[w]);
    const float2* cml = a.cand_ml + ((size_t)b * a.Hq + h) * a.nchunks;
    for (int ch = 0; ch < a.nchunks; ++ch) cand.merge(cml[ch].x, cml[ch].y);
    mass_report(a.mass, a.lse, (size_t)b * a.Hq + h, c.m, c.l, wa.m, wa.l,
                cand.m, cand.l, s_s0, anc != 0);
  }
  // the radix path's Top-k, sorted by warp 0 above, once every thread sees it
  if (a.kpow2 > 128) {
    __syncthreads();
    write_idx();
  }
}


// Sequence-sharded decode, last step: combine the shards' softmax states
// (max, sum, o) into O = sum_p o_p 2^(m_p - M) / sum_p l_p 2^(m_p - M),
// M = max_p m_p over the shards that hold members of C_i.  One CTA per
// (batch, q-head), one thread per output dimension.
template <typename TO>
__global__ void decode_shard_combine(const float* parts, int P, int rows,
                                     int D, void* O) {
  const int row = blockIdx.x, dd = threadIdx.x;
  if (dd >= D) return;
  float M = -INFINITY;
  for (int p = 0; p < P; ++p) {
    const float* pt = parts + ((size_t)p * rows + row) * (D + 2);
    if (pt[1] > 0.f) M = fmaxf(M, pt[0]);
  }
  float l = 0.f, o = 0.f;
  for (int p = 0; p < P; ++p) {
    const float* pt = parts + ((size_t)p * rows + row) * (D + 2);
    if (pt[1] > 0.f) {
      const float c = exp2f(pt[0] - M);
      l += pt[1] * c;
      o += pt[2 + dd] * c;
    }
  }
  store_out<TO>(reinterpret_cast<TO*>(O) + (size_t)row * D + dd, o / l);
}

// Shared memory of the score kernel: a K staging ring of 2..kMaxStages
// stages and per-list candidate buffers of k + kSub + slack keys.  Prefer
// two CTAs per SM; spend what is left after the ring on insert slack.
template <typename T, int D, int G>
void score_smem(int k, int* cap, int* nstages, size_t* bytes) {
  constexpr size_t kStage = ScoreCfg<T, D, G>::STAGE;
  const size_t fixed = sizeof(TopkShared<G>);
  const size_t min_lists = (size_t)G * 8 * (k + kSub + kMinSlack);
  size_t budget = kSmemTwoCtas;
  if (fixed + min_lists + kTwoCtaStages * kStage > budget) budget = kSmemOneCta;
  // With two CTAs per SM, kTwoCtaStages stages; the rest goes to insert
  // slack, which makes list cuts rarer (a deeper ring with less slack
  // measured slower at 131K).
  long st = budget == kSmemTwoCtas
                ? kTwoCtaStages
                : (long)((budget - fixed - min_lists) / kStage);
  if (st > kMaxStages) st = kMaxStages;
  if (st < 2) st = 2;
  const size_t rem = budget - fixed - (size_t)st * kStage;
  long slack = (long)(rem / (8 * G)) - k - kSub;
  if (slack > kMaxSlack) slack = kMaxSlack;
  if (slack < kMinSlack) slack = kMinSlack;
  *cap = k + kSub + (int)slack;
  *nstages = (int)st;
  *bytes = (size_t)st * kStage + (size_t)G * 8 * (size_t)(*cap) + fixed;
}

template <typename T, int D, int G>
cudaError_t launch_typed(DecodeArgs a, cudaStream_t stream) {
  a.top_first = 0;
  if (a.mode == kShardAttend) {
    // the lists are the shards' selections, best keys first when k <= 128
    a.top_first = a.kpow2 <= 128;
  } else {
    a.list_stride = (size_t)a.k;
    a.head_stride = (size_t)a.nchunks * a.k;
  }
  size_t smem1;
  score_smem<T, D, G>(a.k, &a.cap, &a.nstages, &smem1);
  cudaError_t e = cudaSuccess;
  const bool mass = a.mass != nullptr || a.lse != nullptr;
  // with k = 0 the set is anchor and window only: the score pass runs only
  // for the mass reports (the candidates' sums); a shard's attend step has
  // its lists already
  if (a.mode != kShardAttend && (a.k > 0 || mass)) {
    bool done = false;
    if constexpr (sizeof(T) == 2) {
      // bf16: the dot products on the tensor pipe
      e = decode_score_tc_launch(a, D, mass, stream);
      if (e != cudaErrorNotSupported) {
        if (e != cudaSuccess) return e;
        done = true;
        a.top_first = 1;
      }
    }
    if (!done) {
      // the CUDA-core pass scores a whole cache only
      if (a.mode == kShardSelect) return cudaErrorNotSupported;
      auto k1 = mass ? decode_score_topk<T, D, G, true>
                     : decode_score_topk<T, D, G, false>;
      // the largest shared-memory carve-out, so that two CTAs fit per SM
      e = ensure_smem(k1, smem1, true);
      if (e != cudaSuccess) return e;
      dim3 grid1(a.nchunks, a.Hkv, a.B);
      prof_before(stream, "decode_score_topk");
      k1<<<grid1, kThreads, smem1, stream>>>(a);
      prof_after(stream);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  const size_t smem2 = (size_t)a.nchunks * a.k * 16 + 128 * 8 +
                       (size_t)a.kpow2 * 8 + sizeof(SelectState<1>) + 512 * 4;
  dim3 grid2(a.Hq, a.B);
  auto k2 = a.o_bf16 ? decode_merge_attend<T, D, __nv_bfloat16>
                     : decode_merge_attend<T, D, float>;
  e = ensure_smem(k2, smem2);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: the merge grid may start while the score
  // grid drains; it waits (griddepcontrol.wait) before reading the lists.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid2;
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = smem2;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_before(stream, "decode_merge_attend");
  e = cudaLaunchKernelEx(&cfg, k2, a);
  prof_after(stream);
  if (e != cudaSuccess) return e;
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
  // About two CTAs per SM of the current device, each chunk a multiple of
  // 64 keys, and at most 8192 merged candidates per q-head.
  const int units = B * Hkv;
  const int target = kDecodeCtasPerSm * sm_count();
  int per = (target + units - 1) / units;
  int cap_merge = kDecodeMaxMerge / (k > 0 ? k : 1);
  if (per > cap_merge) per = cap_merge;
  int max_by_len = (L + 255) / 256;
  if (per > max_by_len) per = max_by_len;
  if (per < 1) per = 1;
  return per;
}

int decode_chunk_len(int L, int nchunks) {
  // a whole number of 128-key tiles of the tensor-core score pass
  int len = (L + nchunks - 1) / nchunks;
  return (len + 127) / 128 * 128;
}

cudaError_t decode_shard_combine_launch(const float* parts, int P, int rows,
                                        int d, void* O, bool o_bf16,
                                        cudaStream_t s) {
  prof_before(s, "decode_shard_combine");
  if (o_bf16)
    decode_shard_combine<__nv_bfloat16><<<rows, d, 0, s>>>(parts, P, rows, d, O);
  else
    decode_shard_combine<float><<<rows, d, 0, s>>>(parts, P, rows, d, O);
  prof_after(s);
  return cudaGetLastError();
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

// C ABI of the Condensate attention library: argument checks, workspace
// layout and dispatch to the decode and prefill launchers.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/condensate_attn.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill.cuh"

namespace {

// Failure-path test hook (condensate_attn_test_stall): 0 = off.
std::atomic<unsigned long long> g_stall_ns{0};

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

bool group_ok(int Hq, int Hkv) {
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return false;
  int G = Hq / Hkv;
  return G == 1 || G == 2 || G == 4 || G == 8;
}

// Decode workspace: status area | unit counters [B, Hkv] (int32) | worker
// lists [B, Hq, workers, k] (64-bit keys) | per-worker candidate (max, sum)
// [B, Hq, workers] (float2).  The status area and the counters are cleared
// by each call.
size_t decode_claims_bytes(int B, int Hkv) {
  return round_up((size_t)B * Hkv * 4, 256);
}
size_t decode_lists_bytes(int B, int Hq, int nch, int k) {
  return round_up((size_t)B * Hq * nch * (k > 0 ? k : 1) * 8, 256);
}
size_t decode_ws(int B, int L, int Hq, int Hkv, int k) {
  const int nch = ca::decode_chunks(B, L, Hkv, k);
  return ca::kStatusBytes + decode_claims_bytes(B, Hkv) +
         decode_lists_bytes(B, Hq, nch, k) +
         round_up((size_t)B * Hq * nch * 8, 256);
}

size_t prefill_ws(int B, int nq, int Hq, int k) {
  return ca::kStatusBytes + ca::prefill_workspace((int64_t)B * Hq * nq, k);
}

bool sizes_ok(ca_dtype dtype, int B, int nq, int L, int Hq, int Hkv, int d,
              int W_max, int k) {
  return B >= 1 && nq >= 1 && L >= nq && group_ok(Hq, Hkv) && W_max >= 1 &&
         k >= 0 && (d == 64 || d == 128) &&
         (dtype == CA_F32 || dtype == CA_BF16);
}

const ca_extras kNoExtras = {nullptr, nullptr, nullptr, nullptr};

// Checks shared by every entry point, in the order the header lists them.
ca_status check_common(const void* q, const void* K, const void* V,
                       ca_dtype dtype, int B, int nq, int L, int Hq, int Hkv,
                       int d, int W, int k, const int32_t* W_i,
                       const ca_extras& x, void* O, ca_dtype o_dtype,
                       int32_t* idx, int32_t* idx_count, int C_max, void* ws) {
  if (!q || !K || !V || !O || !idx || !idx_count) return CA_ERR_INVALID_ARG;
  if (B < 1 || nq < 1 || L < nq || k < 0 || C_max < 1)
    return CA_ERR_INVALID_ARG;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return CA_ERR_INVALID_ARG;
  const bool device_windows = W_i || x.W_h;
  if (!device_windows && W < 1) return CA_ERR_INVALID_ARG;
  if (!device_windows) {
    // the largest set is the last row's: min(L, 1 + W + k)
    long long need = 1LL + W + k;
    if (need > L) need = L;
    if (C_max < need) return CA_ERR_INVALID_ARG;
  }
  if (dtype != CA_F32 && dtype != CA_BF16) return CA_ERR_UNSUPPORTED;
  if (o_dtype != CA_F32 && o_dtype != CA_BF16) return CA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return CA_ERR_UNSUPPORTED;
  if (!group_ok(Hq, Hkv)) return CA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      !aligned16(idx) || !aligned16(idx_count) || !aligned16(ws) ||
      (W_i && ((uintptr_t)W_i & 3u)) || (x.W_h && ((uintptr_t)x.W_h & 3u)) ||
      (x.k_h && ((uintptr_t)x.k_h & 3u)) ||
      (x.mass && ((uintptr_t)x.mass & 15u)) ||
      (x.lse && ((uintptr_t)x.lse & 3u)))
    return CA_ERR_ALIGNMENT;
  return CA_OK;
}


// Checks shared by the two per-shard steps.
ca_status check_shard(const void* q, const void* K, ca_dtype dtype, int B,
                      int L_shard, int pos0, int L, int Hq, int Hkv, int d,
                      int W, int k, const int32_t* W_i, void* ws) {
  if (!q || !K) return CA_ERR_INVALID_ARG;
  if (B < 1 || L_shard < 1 || pos0 < 0 || L < 1 ||
      (long long)pos0 + L_shard > L || k < 0 || (!W_i && W < 1))
    return CA_ERR_INVALID_ARG;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return CA_ERR_INVALID_ARG;
  if (dtype != CA_F32 && dtype != CA_BF16) return CA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return CA_ERR_UNSUPPORTED;
  if (!group_ok(Hq, Hkv)) return CA_ERR_UNSUPPORTED;
  if (k > ca::kDecodeMaxK) return CA_ERR_UNSUPPORTED;
  if (!ws) return CA_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(K) || !aligned16(ws) ||
      (W_i && ((uintptr_t)W_i & 3u)))
    return CA_ERR_ALIGNMENT;
  return CA_OK;
}

void shard_args(ca::DecodeArgs& a, const void* q, const void* K,
                const void* V, int B, int L_shard, int pos0, int L, int Hq,
                int Hkv, int W, int k, const int32_t* W_i, void* ws) {
  a.q = q; a.K = K; a.V = V;
  a.B = B; a.L = L_shard; a.Hq = Hq; a.Hkv = Hkv; a.W = W; a.k = k;
  a.Lg = L; a.pos0 = pos0;
  a.W_i = W_i; a.W_h = nullptr; a.k_h = nullptr;
  a.mass = nullptr; a.lse = nullptr; a.cand_ml = nullptr;
  a.O = nullptr; a.o_bf16 = 0;
  a.idx = nullptr; a.idx_count = nullptr; a.C_max = 0;
  a.keys_out = nullptr; a.partial = nullptr;
  a.kpow2 = next_pow2(k > 1 ? k : 2);
  a.status = (uint32_t*)ws;
  a.claims = (int*)((char*)ws + ca::kStatusBytes);
  a.wait_ns = ca::kPipelineWaitNs;
  a.stall_ns = g_stall_ns.load();
}

ca_status launch_status(cudaError_t e) {
  if (e == cudaSuccess) return CA_OK;
  return e == cudaErrorNotSupported ? CA_ERR_UNSUPPORTED : CA_ERR_CUDA;
}

}  // namespace

extern "C" {

int condensate_attn_version(void) { return 301; }

int condensate_attn_build_flags(void) {
#ifdef CA_DEBUG
  return CA_BUILD_DEBUG;
#else
  return 0;
#endif
}

const char* condensate_attn_status_string(ca_status s) {
  switch (s) {
    case CA_OK: return "ok";
    case CA_ERR_INVALID_ARG: return "invalid argument";
    case CA_ERR_UNSUPPORTED: return "unsupported configuration";
    case CA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case CA_ERR_WORKSPACE: return "workspace missing or too small";
    case CA_ERR_CUDA: return "CUDA error";
    case CA_ERR_TIMEOUT: return "device wait timed out";
    case CA_ERR_DEVICE_ARG: return "device-side argument out of range";
    case CA_ERR_INTERNAL: return "internal consistency check failed on the device";
    case CA_ERR_BOUNDS: return "index check of the debug build failed on the device";
  }
  return "unknown status";
}

size_t condensate_attn_workspace_size_ex(int is_decode, ca_dtype dtype, int B,
                                         int nq, int L, int Hq, int Hkv, int d,
                                         int W_max, int k) {
  if (is_decode) nq = 1;
  if (!sizes_ok(dtype, B, nq, L, Hq, Hkv, d, W_max, k)) return 0;
  if (is_decode) return decode_ws(B, L, Hq, Hkv, k);
  return prefill_ws(B, nq, Hq, k);
}

size_t condensate_attn_workspace_size(int is_decode, ca_dtype dtype, int B,
                                      int n_or_L, int Hq, int Hkv, int d,
                                      int W_max, int k) {
  return condensate_attn_workspace_size_ex(is_decode, dtype, B, n_or_L,
                                           n_or_L, Hq, Hkv, d, W_max, k);
}

int condensate_attn_decode_chunks(int B, int L, int Hkv, int k) {
  if (B < 1 || L < 1 || Hkv < 1 || k < 0) return 0;
  return ca::decode_chunks(B, L, Hkv, k);
}

ca_status condensate_attn_decode_ex(const void* q, const void* K,
                                    const void* V, ca_dtype dtype, int B,
                                    int L, int Hq, int Hkv, int d, int W,
                                    int k, const int32_t* W_i,
                                    const ca_extras* extras, void* O,
                                    ca_dtype o_dtype, int32_t* idx,
                                    int32_t* idx_count, int C_max,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (!workspace) return CA_ERR_WORKSPACE;
  const ca_extras& x = extras ? *extras : kNoExtras;
  ca_status st = check_common(q, K, V, dtype, B, 1, L, Hq, Hkv, d, W, k, W_i,
                              x, O, o_dtype, idx, idx_count, C_max, workspace);
  if (st != CA_OK) return st;
  if (k > ca::kDecodeMaxK) return CA_ERR_UNSUPPORTED;
  if (workspace_bytes < decode_ws(B, L, Hq, Hkv, k)) return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t cleared = ca::kStatusBytes + decode_claims_bytes(B, Hkv);
  if (cudaMemsetAsync(workspace, 0, cleared, s) != cudaSuccess)
    return CA_ERR_CUDA;
  ca::DecodeArgs a;
  a.q = q; a.K = K; a.V = V;
  a.B = B; a.L = L; a.Hq = Hq; a.Hkv = Hkv; a.W = W; a.k = k;
  a.W_i = W_i; a.W_h = x.W_h; a.k_h = x.k_h; a.mass = x.mass; a.lse = x.lse;
  a.O = O; a.o_bf16 = o_dtype == CA_BF16;
  a.idx = idx; a.idx_count = idx_count; a.C_max = C_max;
  a.nchunks = ca::decode_chunks(B, L, Hkv, k);
  a.chunk_len = ca::decode_chunk_len(L, a.nchunks);
  a.kpow2 = next_pow2(k > 1 ? k : 2);
  a.status = (uint32_t*)workspace;
  a.claims = (int*)((char*)workspace + ca::kStatusBytes);
  a.cand = (uint64_t*)((char*)workspace + cleared);
  a.cand_ml = (float2*)((char*)a.cand +
                        decode_lists_bytes(B, Hq, a.nchunks, k));
  a.Lg = L;
  a.pos0 = 0;
  a.mode = ca::kDecodeAttend;
  a.keys_out = nullptr;
  a.partial = nullptr;
  a.wait_ns = ca::kPipelineWaitNs;
  a.stall_ns = g_stall_ns.load();
  cudaError_t e = ca::decode_launch(a, dtype == CA_BF16, d, s);
  return e == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

// ------------------------------------------------- sequence-sharded decode

size_t condensate_attn_decode_shard_workspace_size(ca_dtype dtype, int B,
                                                   int L_shard, int Hq,
                                                   int Hkv, int d, int k) {
  if (!sizes_ok(dtype, B, 1, L_shard, Hq, Hkv, d, 1, k)) return 0;
  return decode_ws(B, L_shard, Hq, Hkv, k);
}

ca_status condensate_attn_decode_shard_select(
    const void* q, const void* K, ca_dtype dtype, int B, int L_shard,
    int pos0, int L, int Hq, int Hkv, int d, int W, int k,
    const int32_t* W_i, uint64_t* keys_out, void* workspace,
    size_t workspace_bytes, void* stream) {
  ca_status st = check_shard(q, K, dtype, B, L_shard, pos0, L, Hq, Hkv, d, W,
                             k, W_i, workspace);
  if (st != CA_OK) return st;
  if (!keys_out && k > 0) return CA_ERR_INVALID_ARG;
  if (keys_out && !aligned16(keys_out)) return CA_ERR_ALIGNMENT;
  if (dtype != CA_BF16) return CA_ERR_UNSUPPORTED;  // tensor-core pass only
  if (workspace_bytes < decode_ws(B, L_shard, Hq, Hkv, k))
    return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t cleared = ca::kStatusBytes + decode_claims_bytes(B, Hkv);
  if (cudaMemsetAsync(workspace, 0, cleared, s) != cudaSuccess)
    return CA_ERR_CUDA;
  ca::DecodeArgs a;
  shard_args(a, q, K, K, B, L_shard, pos0, L, Hq, Hkv, W, k, W_i, workspace);
  a.mode = ca::kShardSelect;
  a.keys_out = keys_out;
  a.nchunks = ca::decode_chunks(B, L_shard, Hkv, k);
  a.chunk_len = ca::decode_chunk_len(L_shard, a.nchunks);
  a.cand = (uint64_t*)((char*)workspace + cleared);
  if (k == 0) return CA_OK;  // nothing to select: keys_out is empty
  return launch_status(ca::decode_launch(a, true, d, s));
}

ca_status condensate_attn_decode_shard_attend(
    const void* q, const void* K, const void* V, ca_dtype dtype, int B,
    int L_shard, int pos0, int L, int Hq, int Hkv, int d, int W, int k,
    const int32_t* W_i, const uint64_t* keys_all, int P, float* partial,
    int32_t* idx, int32_t* idx_count, int C_max, void* workspace,
    size_t workspace_bytes, void* stream) {
  ca_status st = check_shard(q, K, dtype, B, L_shard, pos0, L, Hq, Hkv, d, W,
                             k, W_i, workspace);
  if (st != CA_OK) return st;
  if (!V || !partial || !idx || !idx_count || (k > 0 && !keys_all) || P < 1 ||
      C_max < 1)
    return CA_ERR_INVALID_ARG;
  if (!W_i) {
    long long need = 1LL + W + k;
    if (need > L) need = L;
    if (C_max < need) return CA_ERR_INVALID_ARG;
  }
  if (!aligned16(V) || !aligned16(partial) || !aligned16(idx) ||
      !aligned16(idx_count) || (keys_all && !aligned16(keys_all)))
    return CA_ERR_ALIGNMENT;
  if ((long long)P * (k > 0 ? k : 1) > ca::kDecodeMaxMerge)
    return CA_ERR_UNSUPPORTED;
  if (workspace_bytes < ca::kStatusBytes) return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, ca::kStatusBytes, s) != cudaSuccess)
    return CA_ERR_CUDA;
  ca::DecodeArgs a;
  shard_args(a, q, K, V, B, L_shard, pos0, L, Hq, Hkv, W, k, W_i, workspace);
  a.mode = ca::kShardAttend;
  a.partial = partial;
  a.idx = idx; a.idx_count = idx_count; a.C_max = C_max;
  a.nchunks = P;
  a.chunk_len = 0;
  a.cand = const_cast<uint64_t*>(keys_all);
  a.list_stride = (size_t)B * Hq * k;  // shard p's keys: keys_all[p][b][h]
  a.head_stride = (size_t)k;
  return launch_status(ca::decode_launch(a, dtype == CA_BF16, d, s));
}

ca_status condensate_attn_decode_shard_combine(const float* partials, int P,
                                               int B, int Hq, int d, void* O,
                                               ca_dtype o_dtype,
                                               void* stream) {
  if (!partials || !O || P < 1 || B < 1 || Hq < 1) return CA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return CA_ERR_UNSUPPORTED;
  if (o_dtype != CA_F32 && o_dtype != CA_BF16) return CA_ERR_UNSUPPORTED;
  if (!aligned16(partials) || !aligned16(O)) return CA_ERR_ALIGNMENT;
  return launch_status(ca::decode_shard_combine_launch(
      partials, P, B * Hq, d, O, o_dtype == CA_BF16, (cudaStream_t)stream));
}

ca_status condensate_attn_decode(const void* q, const void* K, const void* V,
                                 ca_dtype dtype, int B, int L, int Hq, int Hkv,
                                 int d, int W, int k, const int32_t* W_i,
                                 void* O, ca_dtype o_dtype, int32_t* idx,
                                 int32_t* idx_count, int C_max,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream) {
  return condensate_attn_decode_ex(q, K, V, dtype, B, L, Hq, Hkv, d, W, k, W_i,
                                   nullptr, O, o_dtype, idx, idx_count, C_max,
                                   workspace, workspace_bytes, stream);
}

ca_status condensate_attn_prefill_ex(const void* Q, const void* K,
                                     const void* V, ca_dtype dtype, int B,
                                     int nq, int L, int Hq, int Hkv, int d,
                                     int W, int k, const int32_t* W_i,
                                     const ca_extras* extras, void* O,
                                     ca_dtype o_dtype, int32_t* idx,
                                     int32_t* idx_count, int C_max,
                                     void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!workspace) return CA_ERR_WORKSPACE;
  const ca_extras& x = extras ? *extras : kNoExtras;
  ca_status st = check_common(Q, K, V, dtype, B, nq, L, Hq, Hkv, d, W, k, W_i,
                              x, O, o_dtype, idx, idx_count, C_max, workspace);
  if (st != CA_OK) return st;
  if (k > ca::kPrefillMaxK) return CA_ERR_UNSUPPORTED;
  if (workspace_bytes < prefill_ws(B, nq, Hq, k)) return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, ca::kStatusBytes, s) != cudaSuccess)
    return CA_ERR_CUDA;
  const int64_t rows = (int64_t)B * Hq * nq;
  ca::PrefillArgs a;
  a.Q = Q; a.K = K; a.V = V;
  a.B = B; a.nq = nq; a.L = L; a.p0 = L - nq;
  a.Hq = Hq; a.Hkv = Hkv; a.W = W; a.k = k;
  a.W_i = W_i; a.W_h = x.W_h; a.k_h = x.k_h; a.mass = x.mass; a.lse = x.lse;
  a.O = O; a.o_bf16 = o_dtype == CA_BF16;
  a.idx = idx; a.idx_count = idx_count; a.C_max = C_max;
  a.status = (uint32_t*)workspace;
  a.ovf_count = (uint32_t*)workspace + 4;  // inside the cleared status area
  a.topk = (uint64_t*)((char*)workspace + ca::kStatusBytes);
  a.ovf_rows = (uint32_t*)((char*)a.topk + ca::prefill_topk_bytes(rows, k));
  a.cand_ml = (float2*)((char*)a.ovf_rows + round_up((size_t)rows * 4, 256));
  a.wait_ns = ca::kPipelineWaitNs;
  a.stall_ns = g_stall_ns.load();
  cudaError_t e = ca::prefill_launch(a, dtype == CA_BF16, d, s);
  if (e == cudaErrorNotSupported) return CA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? CA_OK : CA_ERR_CUDA;
}

ca_status condensate_attn_prefill(const void* Q, const void* K, const void* V,
                                  ca_dtype dtype, int B, int n, int Hq,
                                  int Hkv, int d, int W, int k,
                                  const int32_t* W_i, void* O,
                                  ca_dtype o_dtype, int32_t* idx,
                                  int32_t* idx_count, int C_max,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return condensate_attn_prefill_ex(Q, K, V, dtype, B, n, n, Hq, Hkv, d, W, k,
                                    W_i, nullptr, O, o_dtype, idx, idx_count,
                                    C_max, workspace, workspace_bytes, stream);
}

ca_status condensate_attn_status(void* workspace, void* stream) {
  if (!workspace) return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CA_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return CA_ERR_CUDA;
  if (word != 0 && cudaMemset(workspace, 0, 4) != cudaSuccess)
    return CA_ERR_CUDA;
  if (word & ca::kErrTimeout) return CA_ERR_TIMEOUT;
  if (word & (ca::kErrWindow | ca::kErrCmax)) return CA_ERR_DEVICE_ARG;
  if (word & ca::kErrInternal) return CA_ERR_INTERNAL;
  if (word & ca::kErrBounds) return CA_ERR_BOUNDS;
  return CA_OK;
}

ca_status condensate_attn_test_stall(unsigned long long limit_ns) {
  if (limit_ns > 60ull * 1000000000ull) return CA_ERR_INVALID_ARG;
  g_stall_ns.store(limit_ns);
  return CA_OK;
}

}  // extern "C"

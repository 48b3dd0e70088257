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

size_t decode_ws(int B, int L, int Hq, int Hkv, int k) {
  int nch = ca::decode_chunks(B, L, Hkv, k);
  return ca::kStatusBytes +
         round_up((size_t)B * Hq * nch * (k > 0 ? k : 1) * 8, 256);
}

}  // namespace

extern "C" {

int condensate_attn_version(void) { return 100; }

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
  }
  return "unknown status";
}

size_t condensate_attn_workspace_size(int is_decode, ca_dtype dtype, int B,
                                      int n_or_L, int Hq, int Hkv, int d,
                                      int W_max, int k) {
  if (B < 1 || n_or_L < 1 || !group_ok(Hq, Hkv) || W_max < 1 || k < 0 ||
      (d != 64 && d != 128) || (dtype != CA_F32 && dtype != CA_BF16))
    return 0;
  if (is_decode) return decode_ws(B, n_or_L, Hq, Hkv, k);
  return ca::kStatusBytes + ca::prefill_workspace(dtype == CA_BF16, B, n_or_L,
                                                  Hq, Hkv, d, k);
}

static ca_status check_common(const void* q, const void* K, const void* V,
                              ca_dtype dtype, int B, int n, int Hq, int Hkv,
                              int d, int W, int k, const int32_t* W_i, void* O,
                              ca_dtype o_dtype, int32_t* idx,
                              int32_t* idx_count, int C_max, void* ws) {
  if (!q || !K || !V || !O || !idx || !idx_count) return CA_ERR_INVALID_ARG;
  if (B < 1 || n < 1 || k < 0 || C_max < 1) return CA_ERR_INVALID_ARG;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return CA_ERR_INVALID_ARG;
  if (!W_i && W < 1) return CA_ERR_INVALID_ARG;
  if (!W_i) {
    long long need = 1LL + W + k;
    if (need > n) need = n;
    if (C_max < need) return CA_ERR_INVALID_ARG;
  }
  if (dtype != CA_F32 && dtype != CA_BF16) return CA_ERR_UNSUPPORTED;
  if (o_dtype != CA_F32 && o_dtype != CA_BF16) return CA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return CA_ERR_UNSUPPORTED;
  if (!group_ok(Hq, Hkv)) return CA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      !aligned16(idx) || !aligned16(idx_count) || !aligned16(ws) ||
      (W_i && ((uintptr_t)W_i & 3u)))
    return CA_ERR_ALIGNMENT;
  return CA_OK;
}

ca_status condensate_attn_decode(const void* q, const void* K, const void* V,
                                 ca_dtype dtype, int B, int L, int Hq, int Hkv,
                                 int d, int W, int k, const int32_t* W_i,
                                 void* O, ca_dtype o_dtype, int32_t* idx,
                                 int32_t* idx_count, int C_max,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!workspace) return CA_ERR_WORKSPACE;
  ca_status st = check_common(q, K, V, dtype, B, L, Hq, Hkv, d, W, k, W_i, O,
                              o_dtype, idx, idx_count, C_max, workspace);
  if (st != CA_OK) return st;
  if (k > ca::kDecodeMaxK) return CA_ERR_UNSUPPORTED;
  if (workspace_bytes < decode_ws(B, L, Hq, Hkv, k)) return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, ca::kStatusBytes, s) != cudaSuccess)
    return CA_ERR_CUDA;
  ca::DecodeArgs a;
  a.q = q; a.K = K; a.V = V;
  a.B = B; a.L = L; a.Hq = Hq; a.Hkv = Hkv; a.W = W; a.k = k;
  a.W_i = W_i; a.O = O; a.o_bf16 = o_dtype == CA_BF16;
  a.idx = idx; a.idx_count = idx_count; a.C_max = C_max;
  a.nchunks = ca::decode_chunks(B, L, Hkv, k);
  a.chunk_len = ca::decode_chunk_len(L, a.nchunks);
  a.kpow2 = next_pow2(k > 1 ? k : 2);
  a.status = (uint32_t*)workspace;
  a.cand = (uint64_t*)((char*)workspace + ca::kStatusBytes);
  a.wait_ns = ca::kPipelineWaitNs;
  a.stall_ns = g_stall_ns.load();
  cudaError_t e = ca::decode_launch(a, dtype == CA_BF16, d, s);
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
  if (!workspace) return CA_ERR_WORKSPACE;
  ca_status st = check_common(Q, K, V, dtype, B, n, Hq, Hkv, d, W, k, W_i, O,
                              o_dtype, idx, idx_count, C_max, workspace);
  if (st != CA_OK) return st;
  if (k > ca::kPrefillMaxK) return CA_ERR_UNSUPPORTED;
  size_t need = ca::kStatusBytes +
                ca::prefill_workspace(dtype == CA_BF16, B, n, Hq, Hkv, d, k);
  if (workspace_bytes < need) return CA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, ca::kStatusBytes, s) != cudaSuccess)
    return CA_ERR_CUDA;
  ca::PrefillArgs a;
  a.Q = Q; a.K = K; a.V = V;
  a.B = B; a.n = n; a.Hq = Hq; a.Hkv = Hkv; a.W = W; a.k = k;
  a.W_i = W_i; a.O = O; a.o_bf16 = o_dtype == CA_BF16;
  a.idx = idx; a.idx_count = idx_count; a.C_max = C_max;
  a.status = (uint32_t*)workspace;
  a.ovf_count = (uint32_t*)workspace + 4;  // inside the cleared status area
  a.topk = (uint64_t*)((char*)workspace + ca::kStatusBytes);
  a.ovf_rows = (uint32_t*)((char*)a.topk + ca::prefill_topk_bytes(B, n, Hq, k));
  a.wait_ns = ca::kPipelineWaitNs;
  a.stall_ns = g_stall_ns.load();
  cudaError_t e = ca::prefill_launch(a, dtype == CA_BF16, d, s);
  if (e == cudaErrorNotSupported) return CA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? CA_OK : CA_ERR_CUDA;
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
  return CA_OK;
}

ca_status condensate_attn_test_stall(unsigned long long limit_ns) {
  if (limit_ns > 60ull * 1000000000ull) return CA_ERR_INVALID_ARG;
  g_stall_ns.store(limit_ns);
  return CA_OK;
}

}  // extern "C"

// Prefill path launch interface (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ca {

// Largest Top-k the prefill selector holds per row (shared-memory heap).
constexpr int kPrefillMaxK = 128;

struct PrefillArgs {
  const void* Q;   // [B, Hq, nq, d]
  const void* K;   // [B, Hkv, L, d]
  const void* V;
  // nq query rows per (batch, head) at positions p0 .. p0+nq-1 (p0 = L-nq)
  // against L keys
  int B, nq, L, p0, Hq, Hkv, W, k;
  const int32_t* W_i;   // [B, nq] or NULL
  const int32_t* W_h;   // [Hq] or NULL
  const int32_t* k_h;   // [Hq] or NULL
  float* mass;          // [B*Hq*nq, 4] or NULL
  float* lse;           // [B*Hq*nq] or NULL
  float2* cand_ml;      // [B*Hq*nq] log2-domain (max, sum) over the
                        // candidates, when mass or lse is asked (workspace)
  void* O;
  int o_bf16;
  int32_t* idx;
  int32_t* idx_count;
  int C_max;
  uint32_t* status;  // device status word (workspace)
  uint64_t* topk;    // [B*Hq*n, k] selected keys per row (workspace)
  uint32_t* ovf_count;  // rows listed for the exact fallback (status area)
  uint32_t* ovf_rows;   // [B*Hq*n] their row indices (workspace)
  uint64_t wait_ns;     // limit of each pipeline wait (kPipelineWaitNs)
  uint64_t stall_ns;    // failure-path test hook (0: off)
};

// Bytes of the per-row Top-k key area at the start of the workspace body
// (rows = B*Hq*nq).
size_t prefill_topk_bytes(int64_t rows, int k);
// Workspace bytes beyond the status area: Top-k keys, the fallback row
// list, the candidates' (max, sum) per row.
size_t prefill_workspace(int64_t rows, int k);
cudaError_t prefill_launch(const PrefillArgs& a, bool bf16, int d,
                           cudaStream_t stream);
// The tensor-core score + Top-k pass (bf16 inputs; prefill_tc.cu).
cudaError_t launch_select_tc(const PrefillArgs& a, int d, cudaStream_t stream);

}  // namespace ca

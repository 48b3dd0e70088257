// Prefill path launch interface (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ca {

// Largest Top-k the prefill selector holds per row (shared-memory heap).
constexpr int kPrefillMaxK = 64;

struct PrefillArgs {
  const void* Q;
  const void* K;
  const void* V;
  int B, n, Hq, Hkv, W, k;
  const int32_t* W_i;
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

// Bytes of the per-row Top-k key area at the start of the workspace body.
size_t prefill_topk_bytes(int B, int n, int Hq, int k);
// Workspace bytes beyond the status area.
size_t prefill_workspace(bool bf16, int B, int n, int Hq, int Hkv, int d,
                         int k);
cudaError_t prefill_launch(const PrefillArgs& a, bool bf16, int d,
                           cudaStream_t stream);

}  // namespace ca

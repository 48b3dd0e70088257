// Host-side launch helpers shared by the launchers (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ca {

// Raise `func`'s dynamic shared-memory limit to at least `bytes` on the
// current device (and ask for the largest shared-memory carve-out when
// `max_carveout`).  The attribute calls are made once per (device, kernel,
// size): later launches only look the value up.
cudaError_t ensure_smem(const void* func, size_t bytes, bool max_carveout);

// Number of SMs of the current device (looked up once per device; 148 if
// the query fails).
int sm_count();

template <typename F>
cudaError_t ensure_smem(F* func, size_t bytes, bool max_carveout = false) {
  return ensure_smem(reinterpret_cast<const void*>(func), bytes, max_carveout);
}

}  // namespace ca

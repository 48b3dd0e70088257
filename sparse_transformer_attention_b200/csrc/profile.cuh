// Optional per-launch timing: when enabled through the C ABI, every kernel
// launch of the library is bracketed by CUDA events recorded on the launch
// stream, so a caller can read each kernel's device time.  Off by default;
// meant for single-threaded benchmarking.
#pragma once

#include <cuda_runtime.h>

namespace ca {

void prof_before(cudaStream_t s, const char* name);
void prof_after(cudaStream_t s);

}  // namespace ca

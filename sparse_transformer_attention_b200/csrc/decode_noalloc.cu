// Decode entry point for callers that cannot allocate device memory.
//
// The regular decode entry point needs a caller-provided workspace for its
// per-chunk candidate lists.  Some callers have no way to provide one: a
// plugin loaded by a host program that exposes no allocator to it, code
// whose device memory is fully budgeted and handed out before it runs, or a
// fixed foreign interface with no scratch-pointer argument.  This entry
// point serves them from a scratch buffer compiled into the library instead.
//
// The buffer is a file-scope __device__ array of kScratchBytes.  Every GPU
// that loads this library's code keeps those bytes reserved until the
// process exits.  In host code the array's name is only a host-side
// stand-in, never a device address, so its device address is looked up once
// per device with cudaGetSymbolAddress (with that device current) and
// cached; the first call on a device does that set-up, so make that first
// call before any stream capture.
//
// All calls on a device share the one buffer and it keeps the previous
// call's contents: the status word at its start is cleared by every call,
// and the candidate lists are fully rewritten before they are read.  The
// flags a call raises on the device (a bad W_i, an overflowing C_max, a
// bounded wait that ran out, a failed internal check) are read and cleared
// by condensate_attn_decode_noalloc_status.  The cached address is valid for
// the life of the device's primary context: after cudaDeviceReset the
// process must not call these entry points again.  Calls
// that overlap on the GPU (on different streams, or from several host
// threads) race on the buffer and must be serialised by the caller.  The
// call allocates nothing: no cudaMalloc, no cudaFree, no allocating library
// routine.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/condensate_attn.h"

namespace {

constexpr size_t kScratchBytes = (size_t)4 << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch buffer on the current device.
ca_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return CA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p)
      return CA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return CA_OK;
}

}  // namespace

extern "C" ca_status condensate_attn_decode_noalloc(
    const void* q, const void* K, const void* V, ca_dtype dtype, int B, int L,
    int Hq, int Hkv, int d, int W, int k, const int32_t* W_i, void* O,
    ca_dtype o_dtype, int32_t* idx, int32_t* idx_count, int C_max,
    void* stream) {
  void* scratch = nullptr;
  ca_status st = scratch_address(&scratch);
  if (st != CA_OK) return st;
  // Same checks and kernels as the workspace entry point; a problem whose
  // workspace exceeds the built-in buffer is rejected with CA_ERR_WORKSPACE
  // before anything is launched.
  return condensate_attn_decode(q, K, V, dtype, B, L, Hq, Hkv, d, W, k, W_i,
                                O, o_dtype, idx, idx_count, C_max, scratch,
                                kScratchBytes, stream);
}

// The device status word of the built-in buffer lives at its start, like a
// workspace's; reading it reuses the cached address and allocates nothing.
extern "C" ca_status condensate_attn_decode_noalloc_status(void* stream) {
  void* scratch = nullptr;
  ca_status st = scratch_address(&scratch);
  if (st != CA_OK) return st;
  return condensate_attn_status(scratch, stream);
}

// Once-per-device kernel attributes (see launch.cuh).
#include <mutex>
#include <vector>

#include "launch.cuh"

namespace ca {

namespace {

struct AttrEntry {
  int dev;
  const void* func;
  size_t bytes;
  bool carveout;
};

std::mutex g_attr_mu;
std::vector<AttrEntry> g_attr;

}  // namespace

cudaError_t ensure_smem(const void* func, size_t bytes, bool max_carveout) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  AttrEntry* hit = nullptr;
  for (auto& a : g_attr)
    if (a.dev == dev && a.func == func) hit = &a;
  if (hit && hit->bytes >= bytes && (hit->carveout || !max_carveout))
    return cudaSuccess;
  const size_t want = hit && hit->bytes > bytes ? hit->bytes : bytes;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)want);
  if (e != cudaSuccess) return e;
  const bool carve = max_carveout || (hit && hit->carveout);
  if (carve) {
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
  }
  if (hit) {
    hit->bytes = want;
    hit->carveout = carve;
  } else {
    g_attr.push_back({dev, func, want, carve});
  }
  return cudaSuccess;
}

int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        n < 1)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace ca

#include <stdint.h>
#include <string.h>

#include "../../include/condensate_attn.h"
#include "profile.cuh"

namespace ca {
namespace {

struct Record {
  const char* name;
  cudaEvent_t start, stop;
};

Record* g_rec = nullptr;
int g_cap = 0;
int g_n = 0;
bool g_on = false;

}  // namespace

void prof_before(cudaStream_t s, const char* name) {
  if (!g_on || g_n >= g_cap) return;
  g_rec[g_n].name = name;
  cudaEventRecord(g_rec[g_n].start, s);
}

void prof_after(cudaStream_t s) {
  if (!g_on || g_n >= g_cap) return;
  cudaEventRecord(g_rec[g_n].stop, s);
  ++g_n;
}

}  // namespace ca

extern "C" {

ca_status condensate_attn_profile_start(int capacity) {
  using namespace ca;
  if (capacity < 1 || capacity > (1 << 20)) return CA_ERR_INVALID_ARG;
  if (g_rec) {
    for (int i = 0; i < g_cap; ++i) {
      cudaEventDestroy(g_rec[i].start);
      cudaEventDestroy(g_rec[i].stop);
    }
    delete[] g_rec;
    g_rec = nullptr;
    g_cap = 0;
  }
  g_rec = new Record[capacity];
  for (int i = 0; i < capacity; ++i) {
    if (cudaEventCreate(&g_rec[i].start) != cudaSuccess ||
        cudaEventCreate(&g_rec[i].stop) != cudaSuccess) {
      g_cap = i;
      return CA_ERR_CUDA;
    }
  }
  g_cap = capacity;
  g_n = 0;
  g_on = true;
  return CA_OK;
}

int condensate_attn_profile_stop(const char** names, float* ms, int cap) {
  using namespace ca;
  g_on = false;
  int n = g_n < cap ? g_n : cap;
  for (int i = 0; i < n; ++i) {
    float t = -1.f;
    if (cudaEventSynchronize(g_rec[i].stop) == cudaSuccess)
      cudaEventElapsedTime(&t, g_rec[i].start, g_rec[i].stop);
    if (names) names[i] = g_rec[i].name;
    if (ms) ms[i] = t;
  }
  g_n = 0;
  return n;
}

}  // extern "C"

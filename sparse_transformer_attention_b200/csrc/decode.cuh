// Decode path launch interface (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ca {

// CTAs per SM of the K-streaming pass (the grid is this times the SM count
// of the current device, split over batch x kv-heads x chunks).
constexpr int kDecodeCtasPerSm = 2;
// Largest Top-k of the decode path (the per-head candidate buffers of the
// score pass must fit in shared memory next to the K staging ring).
constexpr int kDecodeMaxK = 1024;
// Upper bound on merged candidates per q-head (chunks x k), so the merge
// fits in shared memory.
constexpr int kDecodeMaxMerge = 8192;
// With k <= 128, each worker list of the tensor-core score pass starts with
// its r = ceil(m / workers) best keys when r is at most this.
constexpr int kDecodeTopR = 8;

// What the merge launch does with the exact Top-k it selects.
enum DecodeMode {
  kDecodeAttend = 0,  // attend over C_i and write O (the whole cache here)
  kShardSelect = 1,   // write the shard's best keys to keys_out, no attend
  kShardAttend = 2,   // lists are every shard's keys; attend over the part
                      // of C_i in this shard and write the partial state
};

struct DecodeArgs {
  const void* q;
  const void* K;
  const void* V;
  int B, L, Hq, Hkv, W, k;
  int Lg;               // cache length of the whole sequence (L unless the
                        // cache is sharded along L); the query is at Lg - 1
  int pos0;             // position of this cache's row 0 in the sequence
  int mode;             // DecodeMode
  uint64_t* keys_out;   // kShardSelect: [B, Hq, k] best keys of the shard
  float* partial;       // kShardAttend: [B, Hq, d + 2] = (max, sum, o[d])
  size_t list_stride;   // keys between consecutive lists of a q-head
  size_t head_stride;   // keys between the lists of consecutive q-heads
  const int32_t* W_i;   // [B] or NULL
  const int32_t* W_h;   // [Hq] or NULL
  const int32_t* k_h;   // [Hq] or NULL
  float* mass;          // [B*Hq, 4] or NULL
  float* lse;           // [B*Hq] or NULL
  float2* cand_ml;      // [B, Hq, nchunks] log2-domain (max, sum) of each
                        // chunk's candidates, when mass or lse is asked
  void* O;
  int o_bf16;
  int32_t* idx;
  int32_t* idx_count;
  int C_max;
  int chunk_len, nchunks, kpow2;
  int top_first;        // 1: each list starts with its r best keys (see
                        // kDecodeTopR), written by the tensor-core pass
  int cap;              // per-list candidate buffer of the score kernel
  int nstages;          // K staging ring depth of the score kernel
  uint64_t* cand;       // [B, Hq, nchunks, k] chunk-best keys (workspace)
  int* claims;          // [B, Hkv] unit counters of the tensor-core score
                        // pass (workspace, zero at launch)
  uint32_t* status;   // device status word (workspace)
  uint64_t wait_ns;   // limit of each pipeline wait (kPipelineWaitNs)
  uint64_t stall_ns;  // failure-path test hook (0: off)
};

int decode_chunks(int B, int L, int Hkv, int k);
// The bf16 score pass on tensor cores (decode_tc.cu); cudaErrorNotSupported
// when its shared-memory plan does not fit (the CUDA-core pass runs then).
cudaError_t decode_score_tc_launch(const DecodeArgs& a, int d, bool mass,
                                   cudaStream_t stream);
int decode_chunk_len(int L, int nchunks);
cudaError_t decode_launch(const DecodeArgs& a, bool bf16, int d,
                          cudaStream_t stream);
// O[row] from the P shards' (max, sum, o[d]) states parts[P, rows, d + 2].
cudaError_t decode_shard_combine_launch(const float* parts, int P, int rows,
                                        int d, void* O, bool o_bf16,
                                        cudaStream_t stream);

}  // namespace ca

/*
 * condensate_attn.h - C ABI of the Condensate attention library (B200, sm_100a).
 *
 * The operation ("Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质",
 * §2.1 Definition 1, §2.2.1-§2.2.3, §2.4 Corollary 3, §5.2.2): for every
 * query position i of a (batch, q-head),
 *
 *     t_ij = q_i . k_j                      (j <= i, causal)
 *     C_i  = {0} U [max(0, i-W_i+1), i] U Top-k_i
 *     o_i  = softmax(t_ij / sqrt(d), j in C_i) . V
 *
 * Top-k_i holds the m_i = min(k, max(0, i-W_i)) best candidates of
 * [1, i-W_i] (the causal positions outside anchor and window), ranked by
 * t_ij descending with ties going to the lower index, so that
 * |C_i| = min(i+1, 1+W_i+k) (§2.4 Corollary 2 as an equality).  With a
 * per-query window array W_i (§2.4 Corollary 3, W_i = 64 + 192 RepScore_i)
 * the scalar W is ignored.  A window at least as long as the sequence (or
 * cache) covers every causal position.
 *
 * Layouts (row-major, head dimension innermost, no padding):
 *   prefill  Q [B, Hq, n, d]; K, V [B, Hkv, n, d]; O [B, Hq, n, d]
 *            idx [B, Hq, n, C_max] int32; idx_count [B, Hq, n] int32;
 *            W_i [B, n] int32 (optional)
 *   decode   q [B, Hq, d]; K, V [B, Hkv, L, d] (the cache, holding the current
 *            token at position L-1, which is the query position);
 *            O [B, Hq, d]; idx [B, Hq, C_max]; idx_count [B, Hq];
 *            W_i [B] int32 (optional)
 * q-head h reads kv-head h / (Hq/Hkv) (grouped-query attention).
 * idx rows hold C_i in ascending order, padded with -1 up to C_max.
 * Supported: d in {64, 128}; dtype CA_F32 or CA_BF16 for Q/K/V (all three
 * alike); O may be CA_F32 or CA_BF16; Hq/Hkv in {1, 2, 4, 8}; k <= 128 for
 * prefill and k <= 1024 for decode (CA_ERR_UNSUPPORTED beyond).
 * Scores and the softmax are accumulated in fp32; selection uses the
 * unscaled fp32 dot product with the tie rule above.
 *
 * Ownership: every pointer is a device pointer owned by the caller, and no
 * entry point allocates device memory.  `stream` is a cudaStream_t (NULL =
 * legacy default stream).  Calls are asynchronous; the returned status
 * covers argument checks and launch errors only.
 *
 * Process-wide state (everything else is per call): a per-device cache of
 * kernel attributes and of the SM count (filled on first use, behind a
 * mutex); the profiling switch (condensate_attn_profile_start/stop) and the
 * failure-path test hook (condensate_attn_test_stall), both for benchmarks
 * and tests, not for use while other threads call the library; and the
 * built-in buffer of condensate_attn_decode_noalloc with its per-device
 * address cache.  The decode chunking follows the current device's SM count,
 * so query condensate_attn_workspace_size with the device current that the
 * call will run on.
 *
 * Errors: arguments are validated before anything is launched (null
 * pointers, sizes, d, group size, 16-byte alignment, C_max >= 1+W+k for the
 * scalar window, workspace size).  Values read on the device (a W_i below
 * 1, a W_i whose set overflows C_max, a bounded wait that ran out)
 * set flags in the workspace's status word; condensate_attn_status() waits
 * for the stream and reports them.  The status word is cleared at the start
 * of every call that uses the workspace.  Inputs must be finite.
 *
 * Debug build: `python -m sparse_transformer_attention_b200.build --debug`
 * compiles the same sources with CA_DEBUG into libcondensate_attn_debug.so
 * (same entry points).  Its kernels also check the indexes that the release
 * build keeps in range by construction (shared-memory segment cursors, list
 * slots, survivor slots, rows listed for the exact fallback); a failed check
 * skips the access and raises CA_ERR_BOUNDS instead of a memory fault.
 */
#ifndef CONDENSATE_ATTN_H
#define CONDENSATE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CA_API __attribute__((visibility("default")))
#else
#define CA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CA_OK = 0,
  CA_ERR_INVALID_ARG = 1, /* null pointer, bad size, C_max too small        */
  CA_ERR_UNSUPPORTED = 2, /* d, dtype or group size outside the list above  */
  CA_ERR_ALIGNMENT = 3,   /* a tensor pointer is not 16-byte aligned         */
  CA_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than required         */
  CA_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed            */
  CA_ERR_TIMEOUT = 6,     /* a bounded device wait gave up (status query)    */
  CA_ERR_DEVICE_ARG = 7,  /* W_i out of range or set overflowing C_max      */
  CA_ERR_INTERNAL = 8,    /* an internal check failed on the device: the
                             results of that call are invalid (a bug)      */
  CA_ERR_BOUNDS = 9       /* debug build only: an index check failed on the
                             device and the access was skipped (a bug)     */
} ca_status;

typedef enum { CA_F32 = 0, CA_BF16 = 1 } ca_dtype;

/*
 * Bytes of device workspace needed by one prefill (is_decode = 0; n_or_L = n)
 * or decode (is_decode = 1; n_or_L = L) call with these sizes.  W_max is the
 * largest window the call may use.  Pure host function; returns 0 for
 * invalid sizes.
 */
CA_API size_t condensate_attn_workspace_size(int is_decode, ca_dtype dtype, int B,
                                      int n_or_L, int Hq, int Hkv, int d,
                                      int W_max, int k);

/*
 * Optional inputs and outputs of the _ex entry points (all device pointers,
 * each may be NULL; the struct itself may be NULL).
 *
 *   W_h   [Hq] int32: window of each q-head ("Condensate Theorem" page 1
 *         §6 layer-wise window schedule and §10.2 per-head parameters: a
 *         schedule over layers is one call per layer with its own W or W_h).
 *         The window of row (b, h, i) is W_i[b, i] when W_i is given, else
 *         W_h[h] when given, else W.  Values below 1 raise
 *         CA_ERR_DEVICE_ARG and are read as 1.
 *   k_h   [Hq] int32: Top-k size of each q-head, each in [0, k] (k, the
 *         scalar argument, is the largest and sizes the workspace; k_h = 0
 *         is the static anchor + window variant).  Values outside [0, k]
 *         raise CA_ERR_DEVICE_ARG and are clamped.
 *   mass  [rows, 4] fp32: per query row, over the full causal softmax
 *         A_ij = softmax_j<=i(t_ij / sqrt(d)) (§2.2.1, §2.2.2, §3.2.2):
 *           [0] anchor mass   A_i0
 *           [1] window mass   sum over j in [max(0, i-W_i+1), i] of A_ij
 *           [2] Top-k mass    sum over the selected Top-k of A_ij
 *           [3] excluded mass epsilon_i = sum over causal j not in C_i
 *   lse   [rows] fp32: log sum_j<=i exp(t_ij / sqrt(d)) (natural log).
 * rows = B*Hq*nq for prefill, B*Hq for decode.  Asking for mass or lse adds
 * one exponential per causal score to the score pass.
 */
typedef struct {
  const int32_t* W_h;
  const int32_t* k_h;
  float* mass;
  float* lse;
} ca_extras;

/*
 * Causal prefill over n positions (§2.1 Definition 1 applied to every row,
 * §5.2.2 select-then-attend).  Two launches: a fused score + Top-k pass
 * (tcgen05 tensor cores for bf16, FFMA for fp32) and a gather + fp32 online
 * softmax pass.  W_i may be NULL.
 */
CA_API ca_status condensate_attn_prefill(const void* Q, const void* K, const void* V,
                                  ca_dtype dtype, int B, int n, int Hq,
                                  int Hkv, int d, int W, int k,
                                  const int32_t* W_i, void* O,
                                  ca_dtype o_dtype, int32_t* idx,
                                  int32_t* idx_count, int C_max,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * Prefill of the last nq positions against an L-long cache (a chunk of a
 * longer prefill, or several decode queries at once; §2.1 Definition 1 for
 * rows L-nq .. L-1, §5.2.2).  Q [B, Hq, nq, d]; K, V [B, Hkv, L, d] with
 * 1 <= nq <= L; query row r sits at position i = L - nq + r and attends to
 * keys 0..i.  W_i is [B, nq]; outputs are [B, Hq, nq, ...].  nq = L is
 * condensate_attn_prefill.  The workspace is
 * condensate_attn_workspace_size_ex(0, dtype, B, nq, L, Hq, Hkv, d, W_max, k).
 */
CA_API ca_status condensate_attn_prefill_ex(
    const void* Q, const void* K, const void* V, ca_dtype dtype, int B, int nq,
    int L, int Hq, int Hkv, int d, int W, int k, const int32_t* W_i,
    const ca_extras* extras, void* O, ca_dtype o_dtype, int32_t* idx,
    int32_t* idx_count, int C_max, void* workspace, size_t workspace_bytes,
    void* stream);

/*
 * Workspace bytes of condensate_attn_prefill_ex (is_decode = 0) or
 * condensate_attn_decode_ex (is_decode = 1, nq = 1) with these sizes.
 */
CA_API size_t condensate_attn_workspace_size_ex(int is_decode, ca_dtype dtype,
                                                int B, int nq, int L, int Hq,
                                                int Hkv, int d, int W_max,
                                                int k);

/*
 * Decode of one query per (batch, q-head) at position L-1 against an L-long
 * cache (§2.1 Definition 1 for the last row).  Two launches: a K-streaming
 * score pass with a per-chunk Top-k, and a merge + gather + softmax pass.
 * W_i may be NULL.
 */
CA_API ca_status condensate_attn_decode(const void* q, const void* K, const void* V,
                                 ca_dtype dtype, int B, int L, int Hq, int Hkv,
                                 int d, int W, int k, const int32_t* W_i,
                                 void* O, ca_dtype o_dtype, int32_t* idx,
                                 int32_t* idx_count, int C_max,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Number of workers (CTAs per batch and kv-head) of the decode score pass on
 * the current device (about two CTAs per SM); each keeps one candidate list
 * per q-head over the part of the cache it streamed.  The decode workspace
 * holds, after its 256-byte status area and a 256-byte-rounded area of
 * B * Hkv 32-bit work counters, the best k selection keys of every worker
 * and q-head, [B, Hq, workers, k] 64-bit keys (fp32 score bits in an
 * order-preserving form in the high word, 0xFFFFFFFF - position in the low
 * word, 0 for an empty slot), in a 256-byte-rounded area.  For tests and
 * debugging; 0 for invalid sizes.
 */
CA_API int condensate_attn_decode_chunks(int B, int L, int Hkv, int k);

/* condensate_attn_decode with the optional inputs and outputs above. */
CA_API ca_status condensate_attn_decode_ex(
    const void* q, const void* K, const void* V, ca_dtype dtype, int B, int L,
    int Hq, int Hkv, int d, int W, int k, const int32_t* W_i,
    const ca_extras* extras, void* O, ca_dtype o_dtype, int32_t* idx,
    int32_t* idx_count, int C_max, void* workspace, size_t workspace_bytes,
    void* stream);

/*
 * Sequence-sharded decode: the cache of one sequence (length L, query at
 * position L-1) split along L over P ranks, rank p holding the contiguous
 * rows [pos0, pos0 + L_shard) as its own K and V of shape
 * [B, Hkv, L_shard, d].  The set C_i and the output are those of
 * condensate_attn_decode on the whole cache (§2.1 Definition 1 for the
 * last row, §2.2.3 Top-k, §5.2.2 select then attend); the split and the two
 * exchanges are this library's, not the paper's.  Per rank, in order:
 *   1. condensate_attn_decode_shard_select: the best min(k, candidates in
 *      the shard) selection keys of the shard per (batch, q-head), to
 *      keys_out [B, Hq, k] (64-bit keys as described for
 *      condensate_attn_decode_chunks, positions in the sequence; best first
 *      when k <= 128; 0 after them).  bf16 only (the tensor-core score
 *      pass); CA_ERR_UNSUPPORTED otherwise.
 *   2. the caller gathers every rank's keys_out into keys_all [P, B, Hq, k]
 *      in rank order (an all-gather);
 *   3. condensate_attn_decode_shard_attend: the exact Top-k of the sequence
 *      from keys_all (the same on every rank), idx / idx_count as
 *      condensate_attn_decode writes them, and this shard's softmax state
 *      over its members of C_i to partial [B, Hq, d + 2] fp32: the running
 *      maximum (log2 domain, scores scaled by log2(e)/sqrt(d)), the sum of
 *      2^(s - max), then the d sums of 2^(s - max) v (max = -inf and sum 0
 *      when no member lies in the shard);
 *   4. the caller gathers every rank's partial into partials [P, B, Hq,
 *      d + 2] (an all-gather);
 *   5. condensate_attn_decode_shard_combine: O [B, Hq, d] in o_dtype.
 * W_i may be NULL; per-head windows, mass and lse outputs are not offered
 * here.  Workspace: condensate_attn_decode_shard_workspace_size for step 1,
 * 256 bytes for step 3 (each call clears what it uses).  Pointers are
 * device pointers, 16-byte aligned (W_i 4-byte); the caller owns every
 * buffer; errors as for condensate_attn_decode, with pos0 < 0, L_shard < 1
 * or pos0 + L_shard > L an invalid argument and P * k > 8192 unsupported.
 */
CA_API size_t condensate_attn_decode_shard_workspace_size(ca_dtype dtype,
                                                          int B, int L_shard,
                                                          int Hq, int Hkv,
                                                          int d, int k);
CA_API ca_status condensate_attn_decode_shard_select(
    const void* q, const void* K, ca_dtype dtype, int B, int L_shard,
    int pos0, int L, int Hq, int Hkv, int d, int W, int k,
    const int32_t* W_i, uint64_t* keys_out, void* workspace,
    size_t workspace_bytes, void* stream);
CA_API ca_status condensate_attn_decode_shard_attend(
    const void* q, const void* K, const void* V, ca_dtype dtype, int B,
    int L_shard, int pos0, int L, int Hq, int Hkv, int d, int W, int k,
    const int32_t* W_i, const uint64_t* keys_all, int P, float* partial,
    int32_t* idx, int32_t* idx_count, int C_max, void* workspace,
    size_t workspace_bytes, void* stream);
CA_API ca_status condensate_attn_decode_shard_combine(const float* partials,
                                                      int P, int B, int Hq,
                                                      int d, void* O,
                                                      ca_dtype o_dtype,
                                                      void* stream);

/*
 * Decode without a workspace argument, for callers that cannot allocate
 * device memory or pass a scratch pointer (a plugin whose host exposes no
 * allocator, a fully pre-budgeted memory plan, a fixed interface with no
 * scratch argument).  The paper has no counterpart to this entry point.
 * Same arguments, results and checks as condensate_attn_decode on the
 * current device, but the scratch comes from a 4 MiB buffer compiled into
 * the library (held on every GPU that loads it until exit).  Problems whose
 * decode workspace (condensate_attn_workspace_size) exceeds 4 MiB are
 * rejected with CA_ERR_WORKSPACE before any launch.  Allocates nothing.  The
 * first call on a device looks up the buffer's device address; make it
 * before any stream capture.  That address is cached for the life of the
 * device's primary context: do not call this entry point again after
 * cudaDeviceReset.  All calls on a device share the buffer: calls that
 * overlap on the GPU race and must be serialised by the caller.  Flags the
 * kernels raise on the device land in the shared buffer's status word; read
 * them with condensate_attn_decode_noalloc_status.
 */
CA_API ca_status condensate_attn_decode_noalloc(
    const void* q, const void* K, const void* V, ca_dtype dtype, int B, int L,
    int Hq, int Hkv, int d, int W, int k, const int32_t* W_i, void* O,
    ca_dtype o_dtype, int32_t* idx, int32_t* idx_count, int C_max,
    void* stream);

/*
 * Status of the last condensate_attn_decode_noalloc call(s) on the current
 * device: waits for `stream`, then reads and clears the status word of the
 * built-in buffer, with the codes of condensate_attn_status.  Allocates
 * nothing.  The paper has no counterpart to this entry point.
 */
CA_API ca_status condensate_attn_decode_noalloc_status(void* stream);

/*
 * Waits for `stream`, then reads and clears the device status word of
 * `workspace`.  The kernels raise four flags there (five in the debug
 * build):
 *   W_i below 1                      -> CA_ERR_DEVICE_ARG (the row is run
 *                                       with a window of 1)
 *   |C_i| larger than C_max          -> CA_ERR_DEVICE_ARG (idx holds the
 *                                       first C_max entries, idx_count the
 *                                       true size)
 *   a bounded device wait ran out    -> CA_ERR_TIMEOUT (outputs invalid)
 *   an internal check failed         -> CA_ERR_INTERNAL (outputs invalid)
 *   (debug build) an index check     -> CA_ERR_BOUNDS (outputs invalid)
 *   failed
 * The time-out outranks the argument flags, which outrank the internal one,
 * which outranks the index check.
 * CA_OK when no flag is set; CA_ERR_CUDA if the wait or copy itself failed.
 */
CA_API ca_status condensate_attn_status(void* workspace, void* stream);

/*
 * Failure-path test hook, not for production use.  With limit_ns > 0 every
 * later prefill or decode call makes one pipeline consumer of its score
 * kernel wait, for at most limit_ns, on a barrier that nothing signals: the
 * wait runs out, the kernel raises the time-out flag, every other wait of
 * the CTA gives up at once, and the kernel leaves through its normal path
 * (copies and tensor-core operations it issued are drained first), so the
 * CUDA context stays usable and condensate_attn_status reports
 * CA_ERR_TIMEOUT.  0 turns the hook off.  Process-wide switch; limit_ns
 * above 60 s is CA_ERR_INVALID_ARG.
 */
CA_API ca_status condensate_attn_test_stall(unsigned long long limit_ns);

/* Static, human-readable name of a status code. */
CA_API const char* condensate_attn_status_string(ca_status s);

/*
 * Per-launch timing for benchmarks (not part of the computation).  Between
 * start and stop, every kernel the library launches is bracketed by CUDA
 * events on its stream, up to `capacity` launches.  stop() waits for the
 * recorded events and writes, per launch in issue order, the kernel's name
 * (a static string) and its device time in milliseconds; returns the number
 * of records written (at most cap).  Process-wide switch: not for use while
 * other threads call the library.
 */
CA_API ca_status condensate_attn_profile_start(int capacity);
CA_API int condensate_attn_profile_stop(const char** names, float* ms,
                                        int cap);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
CA_API int condensate_attn_version(void);

/* Flags of the loaded build: CA_BUILD_DEBUG when it was compiled with
 * CA_DEBUG (the index-checking debug build), 0 for the release build. */
#define CA_BUILD_DEBUG 1
CA_API int condensate_attn_build_flags(void);

#ifdef __cplusplus
}
#endif

#endif /* CONDENSATE_ATTN_H */

// jfa_internal.cuh — declarations shared by the kernel files and the C ABI.
#pragma once

#include "jfa_common.cuh"

#include <utility>

namespace jfa {

// Launch with programmatic stream serialization, so the kernel may be
// scheduled while the previous kernel of the stream drains; the kernel calls
// pdl_wait() before touching anything the previous kernel writes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Workspace layout for (geometry, max_topk); host and device agree on it.
int workspace_layout(const jfa_geom& g, int max_topk, jfa_workspace_layout* out);

// A decode step's query: device (or managed) memory is used as it is; pinned
// host memory is copied into the workspace's staging region by one kernel
// (launched here) and *q is pointed there.  JFA_ERR_INVALID_ARG for pageable
// host memory.
int stage_query(const jfa_geom& g, const uint16_t** q, uint8_t* ws, const jfa_workspace_layout& L,
                cudaStream_t st);

// Per-sequence lengths of one call (the same for every KV head of a
// sequence) and the offset of each sequence's first group in the flattened
// (segment, group) list the scan splits: sequence b, KV head h, group g is
// entry gpre[b] + h * ng(b) + g, ng(b) = N_q(b) / 64.  Passed by value in
// the launch parameters (2 KB).
constexpr int kMaxBatch = JFA_MAX_BATCH;
struct SeqTable {
  int32_t n_ctx[kMaxBatch];
  int32_t gpre[kMaxBatch + 1];
};
// Fill the table for a geometry: lens[b] (host array) or, when lens is null,
// geom.n_ctx for every sequence.  Returns false when a length is outside
// [1, capacity] or the batch exceeds kMaxBatch.
bool fill_seq_table(const jfa_geom& g, const int32_t* lens, SeqTable* t);
__host__ __device__ __forceinline__ int seq_groups(const SeqTable& t, int b) {
  return split_point(t.n_ctx[b]) / kKG;
}
// Largest quantized-token count over the batch.
int max_nq(const jfa_geom& g, const SeqTable& t);

// Scan decomposition: W warps each take a balanced contiguous range of the
// flattened (segment, group) list; warp w writes one partial per segment it
// touches into slot (w + segment).
struct ScanPlan {
  long long total_groups;  // entries of the flattened list
  int n_warps;             // warps with work
  int n_ctas;
};
ScanPlan scan_plan(const jfa_geom& g, const SeqTable& t, int num_sms);
int num_sms_current();

// First warp whose range contains flattened group x (W warps, T groups).
__host__ __device__ __forceinline__ long long scan_warp_of(long long x, long long W, long long T) {
  return ((x + 1) * W - 1) / T;
}
__host__ __device__ __forceinline__ long long scan_range_begin(long long w, long long W,
                                                               long long T) {
  return w * T / W;
}

int launch_pack(const jfa_geom& g, const jfa_cache& c, const uint16_t* k_new,
                const uint16_t* v_new, int n_new, uint32_t* flag, cudaStream_t st);
// One new token per sequence at position t.n_ctx[b] - 1 (t holds the lengths
// after the append; a full tail is first flushed as one group); the new rows
// also go to the exact copy when it is given.
int launch_append1(const jfa_geom& g, const SeqTable& t, const jfa_cache& c, const uint16_t* k_new,
                   const uint16_t* v_new, uint16_t* k_exact, uint16_t* v_exact, uint32_t* flag,
                   cudaStream_t st);
// pdl: launch as a programmatic dependent of the previous kernel (its first
// record copies may then start before that kernel has finished); defer_last:
// the previous kernel may be writing each sequence's last group (the append
// kernel), so that record is requested only after the dependency wait.
int launch_scores(const jfa_geom& g, const SeqTable& t, const jfa_cache& c, const uint16_t* q,
                  float scale, uint8_t* ws, const jfa_workspace_layout& L, cudaStream_t st,
                  bool pdl = true, bool defer_last = false);
int launch_topk(const jfa_geom& g, int k, uint8_t* ws, const jfa_workspace_layout& L,
                int32_t* idx, cudaStream_t st);
int count_topk_launches(const jfa_geom& g, int k);
// Block selection: at most kMaxSelBlocks blocks of 128 quantized tokens per
// segment (N_q <= 1M tokens).
constexpr int kMaxSelBlocks = 8192;
// bkeys: the block keys already computed (the FP4 scan leaves them), else
// null to take every block's largest stored score.
int launch_topk_blocks(const jfa_geom& g, int n_blocks, uint8_t* ws, const jfa_workspace_layout& L,
                       int32_t* idx, cudaStream_t st, const uint32_t* bkeys = nullptr);
// Selection (idx_in == nullptr: top-k written to idx_out) or a given index
// set (idx_in), then correction and merge: one cluster per segment.
int launch_finish(const jfa_geom& g, const SeqTable& t, const jfa_cache& c, const uint16_t* q,
                  float scale, int k,
                  int32_t* idx_out, const int32_t* idx_in, const uint16_t* k_exact,
                  const uint16_t* v_exact, uint8_t* ws, const jfa_workspace_layout& L, float* out,
                  cudaStream_t st);

}  // namespace jfa

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

// Scan decomposition: W warps each take a balanced contiguous range of the
// flattened (segment, group) list; warp w writes one partial per segment it
// touches into slot (w + segment).
struct ScanPlan {
  long long total_groups;  // n_seg * NG
  int ng;                  // groups per segment in this call (N_q / 64)
  int n_warps;             // warps with work
  int n_ctas;
};
ScanPlan scan_plan(const jfa_geom& g, int num_sms);
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
int launch_scores(const jfa_geom& g, const jfa_cache& c, const uint16_t* q, float scale,
                  uint8_t* ws, const jfa_workspace_layout& L, cudaStream_t st);
int launch_topk(const jfa_geom& g, int k, uint8_t* ws, const jfa_workspace_layout& L,
                int32_t* idx, cudaStream_t st);
int count_topk_launches(const jfa_geom& g, int k);
// Block selection: at most kMaxSelBlocks blocks of 128 quantized tokens per
// segment (N_q <= 1M tokens).
constexpr int kMaxSelBlocks = 8192;
int launch_topk_blocks(const jfa_geom& g, int n_blocks, uint8_t* ws, const jfa_workspace_layout& L,
                       int32_t* idx, cudaStream_t st);
// Selection (idx_in == nullptr: top-k written to idx_out) or a given index
// set (idx_in), then correction and merge: one cluster per segment.
int launch_finish(const jfa_geom& g, const jfa_cache& c, const uint16_t* q, float scale, int k,
                  int32_t* idx_out, const int32_t* idx_in, const uint16_t* k_exact,
                  const uint16_t* v_exact, uint8_t* ws, const jfa_workspace_layout& L, float* out,
                  cudaStream_t st);

}  // namespace jfa

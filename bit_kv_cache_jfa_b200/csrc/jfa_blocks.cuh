// jfa_blocks.cuh — block-level building blocks shared by the selection and
// finishing kernels: block scans and the radix-bin search.
#pragma once

#include "jfa_internal.cuh"

namespace jfa {

constexpr unsigned kAll = 0xFFFFFFFFu;

// Block-wide exclusive sum over threads in DESCENDING thread order:
// returns the sum of v over threads with a larger index.
__device__ __forceinline__ uint32_t block_suffix_excl(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_down_sync(kAll, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) scratch[warp] = x;
  __syncthreads();
  uint32_t after = 0;
  for (int w = warp + 1; w < nw; ++w) after += scratch[w];
  __syncthreads();
  return after + (x - v);
}

// Block-wide exclusive prefix sum in thread order; *total gets the sum.
__device__ __forceinline__ uint32_t block_prefix_excl(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(kAll, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
  for (int w = 0; w < nw; ++w) {
    const uint32_t t = scratch[w];
    before += w < warp ? t : 0u;
    all += t;
  }
  __syncthreads();
  *total = all;
  return before + (x - v);
}

// Given per-bin counts h[0..nbins), find the bin where the count taken from
// the top reaches r (1 <= r <= total); returns the bin and the count above it.
__device__ __forceinline__ void find_from_top(const uint32_t* h, int nbins, uint32_t r, uint32_t* scratch,
                              int* out_bin, uint32_t* out_above) {
  const int per = nbins / blockDim.x;  // nbins is a multiple of blockDim
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += h[b0 + i];
  uint32_t cum = block_suffix_excl(local, scratch);
  for (int i = per - 1; i >= 0; --i) {
    const uint32_t c = h[b0 + i];
    if (cum < r && cum + c >= r) {
      *out_bin = b0 + i;
      *out_above = cum;
    }
    cum += c;
  }
  __syncthreads();
}


}  // namespace jfa

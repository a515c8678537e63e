// topk.cu — jfa_topk: per (sequence, KV head) the k tokens with the largest
// selection score S (JetFire README, introduction: the top-k tokens are
// corrected; Jet-QSparse abstract: selection per KV head).
//
// Order (S descending, index ascending); the chosen indices are written in
// ascending index order.  Scores map to order-preserving 32-bit keys.
//   1. histogram kernel: many CTAs per segment build a histogram of the top
//      11 key bits; the last CTA of a segment finds the bin b* holding the
//      k-th key and the count of keys above it.
//   2. collect kernel: every 4096-score chunk writes the (key, index) of each
//      score with bin >= b* to its own list, in index order (ordered
//      compaction with a block scan).
//   3. final kernel, one CTA per segment: two radix refinements (next 11,
//      then 10 key bits) over the short lists give the exact k-th key K*;
//      ties at K* go to the lowest indices, which come first in list order;
//      one ordered pass writes the chosen indices, already ascending.
#include "jfa_internal.cuh"

namespace jfa {

constexpr unsigned kFullMask = 0xFFFFFFFFu;
constexpr int kTopkChunk = 4096;  // scores per CTA of the histogram / collect kernels
constexpr int kCtrStride = 8;     // per segment: [2] b*, [3] count above b*, [4] hist CTAs done

// Block-wide exclusive sum over threads in DESCENDING thread order:
// returns the sum of v over threads with a larger index.
__device__ uint32_t block_suffix_excl(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_down_sync(kFullMask, x, o);
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
__device__ uint32_t block_prefix_excl(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(kFullMask, x, o);
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
__device__ void find_from_top(const uint32_t* h, int nbins, uint32_t r, uint32_t* scratch,
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

struct TopkBufs {
  const float* scores;
  uint32_t* hist;      // [n_seg][2048]
  uint32_t* counters;  // [n_seg][kCtrStride]
  uint2* lists;        // [n_seg][n_chunks_cap][kTopkChunk] (key, index)
  uint32_t* counts;    // [n_seg][n_chunks_cap]
  int capacity, nq, k, n_chunks, n_chunks_cap;
};

__global__ void __launch_bounds__(256) topk_hist_kernel(TopkBufs b) {
  __shared__ uint32_t sh[kHistBins];
  __shared__ uint32_t scratch[32];
  __shared__ bool s_last;
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int seg = blockIdx.y;
  const int lo = blockIdx.x * kTopkChunk;
  const float* s = b.scores + (size_t)seg * b.capacity;
  float4 v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {  // nq is a multiple of 64: a float4 is all in or all out
    const int i = lo + 4 * (threadIdx.x + 256 * r);
    v[r] = i < b.nq ? *reinterpret_cast<const float4*>(s + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (lo + 4 * (threadIdx.x + 256 * r) < b.nq) {
      atomicAdd(&sh[float_key(v[r].x) >> 21], 1u);
      atomicAdd(&sh[float_key(v[r].y) >> 21], 1u);
      atomicAdd(&sh[float_key(v[r].z) >> 21], 1u);
      atomicAdd(&sh[float_key(v[r].w) >> 21], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh = b.hist + (size_t)seg * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
  // the last CTA of the segment finds the bin holding the k-th key
  uint32_t* ctr = b.counters + (size_t)seg * kCtrStride;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&ctr[4], 1u) == gridDim.x - 1;
    s_bin = 0;
    s_above = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = __ldcg(&gh[i]);
  __syncthreads();
  find_from_top(sh, kHistBins, (uint32_t)b.k, scratch, &s_bin, &s_above);
  if (threadIdx.x == 0) {
    ctr[2] = (uint32_t)s_bin;
    ctr[3] = s_above;
  }
}

// Thread t owns the 16 consecutive scores lo + 16t .. lo + 16t + 15, so a
// block prefix sum of per-thread counts gives index-ordered positions.
__global__ void __launch_bounds__(256) topk_collect_kernel(TopkBufs b) {
  __shared__ uint32_t scratch[32];
  const int seg = blockIdx.y, chunk = blockIdx.x;
  const int lo = chunk * kTopkChunk;
  const int base = lo + 16 * threadIdx.x;
  const float* s = b.scores + (size_t)seg * b.capacity;
  float4 v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
    v[r] = base + 4 * r < b.nq ? *reinterpret_cast<const float4*>(s + base + 4 * r)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
  const uint32_t bstar = b.counters[(size_t)seg * kCtrStride + 2];
  uint32_t keys[16];
  uint32_t mask = 0, n = 0;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float vals[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = 4 * r + e;
      keys[i] = float_key(vals[e]);
      const bool in = (base + i < b.nq) && (keys[i] >> 21) >= bstar;
      mask |= (in ? 1u : 0u) << i;
      n += in ? 1u : 0u;
    }
  }
  uint32_t total;
  uint32_t pos = block_prefix_excl(n, scratch, &total);
  uint2* out = b.lists + ((size_t)seg * b.n_chunks_cap + chunk) * kTopkChunk;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (mask & (1u << i)) out[pos++] = make_uint2(keys[i], (uint32_t)(base + i));
  if (threadIdx.x == 0) b.counts[(size_t)seg * b.n_chunks_cap + chunk] = total;
}

// One CTA (256 threads) per segment.
__global__ void __launch_bounds__(256) topk_final_kernel(TopkBufs b, int32_t* idx) {
  __shared__ uint32_t h[kHistBins];
  __shared__ uint32_t scratch[32];
  __shared__ uint32_t cnt[64];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int seg = blockIdx.x;
  const int tid = threadIdx.x;
  const uint32_t* ctr = b.counters + (size_t)seg * kCtrStride;
  const uint32_t bstar = ctr[2];
  const uint32_t r = (uint32_t)b.k - ctr[3];  // keys to take from bin b* (>= 1)
  const uint2* lists = b.lists + (size_t)seg * b.n_chunks_cap * kTopkChunk;
  const uint32_t* counts = b.counts + (size_t)seg * b.n_chunks_cap;
  const bool small = b.n_chunks <= 64;
  if (small && tid < b.n_chunks) cnt[tid] = counts[tid];
  __syncthreads();
  auto count_of = [&](int c) -> uint32_t { return small ? cnt[c] : counts[c]; };

  // refinement 1: bits 20..10 of keys in bin b*
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
  if (tid == 0) {
    s_bin = 0;
    s_above = 0;
  }
  __syncthreads();
  for (int c = 0; c < b.n_chunks; ++c) {
    const uint32_t n = count_of(c);
    const uint2* L = lists + (size_t)c * kTopkChunk;
    for (uint32_t i = tid; i < n; i += blockDim.x) {
      const uint32_t key = L[i].x;
      if ((key >> 21) == bstar) atomicAdd(&h[(key >> 10) & 2047u], 1u);
    }
  }
  __syncthreads();
  find_from_top(h, 2048, r, scratch, &s_bin, &s_above);
  const uint32_t d2 = (uint32_t)s_bin;
  const uint32_t r2 = r - s_above;
  // refinement 2: bits 9..0 of keys with prefix (b*, d2)
  const uint32_t pre = (bstar << 11) | d2;
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (int c = 0; c < b.n_chunks; ++c) {
    const uint32_t n = count_of(c);
    const uint2* L = lists + (size_t)c * kTopkChunk;
    for (uint32_t i = tid; i < n; i += blockDim.x) {
      const uint32_t key = L[i].x;
      if ((key >> 10) == pre) atomicAdd(&h[key & 1023u], 1u);
    }
  }
  __syncthreads();
  find_from_top(h, 1024, r2, scratch, &s_bin, &s_above);
  const uint32_t kstar = (pre << 10) | (uint32_t)s_bin;
  const uint32_t r3 = r2 - s_above;  // keys equal to K* to take, lowest indices first

  // ordered pass: chosen = key > K*, or key == K* among the first r3 such
  uint32_t out_base = 0, eq_base = 0;
  int32_t* o = idx + (size_t)seg * b.k;
  for (int c = 0; c < b.n_chunks; ++c) {
    const uint32_t n = count_of(c);
    const uint2* L = lists + (size_t)c * kTopkChunk;
    for (uint32_t i0 = 0; i0 < n; i0 += blockDim.x) {
      const uint32_t i = i0 + tid;
      uint2 e = make_uint2(0u, 0u);
      if (i < n) e = L[i];
      const uint32_t is_eq = (i < n && e.x == kstar) ? 1u : 0u;
      uint32_t eq_tot;
      const uint32_t eq_rank = eq_base + block_prefix_excl(is_eq, scratch, &eq_tot);
      const uint32_t chosen = (i < n && (e.x > kstar || (is_eq && eq_rank < r3))) ? 1u : 0u;
      uint32_t ch_tot;
      const uint32_t pos = out_base + block_prefix_excl(chosen, scratch, &ch_tot);
      if (chosen && pos < (uint32_t)b.k) o[pos] = (int32_t)e.y;
      out_base += ch_tot;
      eq_base += eq_tot;
    }
  }
}

__global__ void topk_fill_kernel(int32_t* idx, int k, int nq) {
  const int seg = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < k; i += gridDim.x * blockDim.x)
    idx[(size_t)seg * k + i] = i < nq ? i : -1;
}

int count_topk_launches(const jfa_geom& g, int k) {
  const int nq = split_point(g.n_ctx);
  return k >= nq ? 1 : 3;  // fill | hist + collect + final (plus one memset)
}

int launch_topk(const jfa_geom& g, int k, uint8_t* ws, const jfa_workspace_layout& L,
                int32_t* idx, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  if (k >= nq) {
    topk_fill_kernel<<<dim3((k + 255) / 256, n_seg), 256, 0, st>>>(idx, k, nq);
    return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
  }
  TopkBufs b;
  b.scores = reinterpret_cast<const float*>(ws + L.off_scores);
  b.hist = reinterpret_cast<uint32_t*>(ws + L.off_hist);
  b.counters = reinterpret_cast<uint32_t*>(ws + L.off_counters);
  b.lists = reinterpret_cast<uint2*>(ws + L.off_cand);
  b.counts = reinterpret_cast<uint32_t*>(ws + L.off_sel);
  b.capacity = g.capacity;
  b.nq = nq;
  b.k = k;
  b.n_chunks = (nq + kTopkChunk - 1) / kTopkChunk;
  b.n_chunks_cap = (g.capacity + kTopkChunk - 1) / kTopkChunk;
  // histograms and counters are contiguous: clear both at once
  if (cudaMemsetAsync(ws + L.off_hist, 0, L.off_cand - L.off_hist, st) != cudaSuccess)
    return JFA_ERR_CUDA;
  topk_hist_kernel<<<dim3(b.n_chunks, n_seg), 256, 0, st>>>(b);
  topk_collect_kernel<<<dim3(b.n_chunks, n_seg), 256, 0, st>>>(b);
  topk_final_kernel<<<n_seg, 256, 0, st>>>(b, idx);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

}  // namespace jfa

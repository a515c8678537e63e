// topk.cu — jfa_topk: per (sequence, KV head) the k tokens with the largest
// selection score S (JetFire README, introduction: the top-k tokens are
// corrected; Jet-QSparse abstract: selection per KV head).
//
// Order (S descending, index ascending); the chosen indices are written in
// ascending index order.  Scores map to order-preserving 32-bit keys.
//   0. histogram kernel: many CTAs per segment count the top 11 key bits; the
//      last CTA of a segment turns the counts into suffix counts (keys with
//      bin >= b);
//   1. collect kernel: every CTA finds the bin b* holding the k-th key from
//      those counts, and every 4096-score chunk writes the (key, index) of
//      each score with bin >= b* to its own list, in index order (ordered
//      compaction with a block scan).
//   2. final kernel, one CTA per segment: the short lists are staged in shared
//      memory; two radix refinements (next 11, then 10 key bits) give the
//      exact k-th key K*; ties at K* go to the lowest indices, which come
//      first in list order; one ordered pass writes the chosen indices,
//      already ascending; it then clears the segment's histogram and counters
//      for the next call (the workspace starts zero-filled).
#include <mutex>

#include "jfa_blocks.cuh"

namespace jfa {

constexpr int kTopkChunk = 4096;  // scores per CTA of the histogram / collect kernels
constexpr int kStageCap = 4096;   // list entries the final kernel stages in shared memory

struct TopkBufs {
  const float* scores;
  const uint32_t* hist;  // [n_seg][2048] suffix counts: keys with bin >= b
  uint32_t* counters;  // [n_seg][kCtrStride]
  uint2* lists;        // [n_seg][n_chunks_cap][kTopkChunk] (key, index)
  uint32_t* counts;    // [n_seg][n_chunks_cap]
  int capacity, nq, k, n_chunks, n_chunks_cap;
};

// Thread t owns the 16 consecutive scores lo + 16t .. lo + 16t + 15, so a
// block prefix sum of per-thread counts gives index-ordered positions.
__global__ void __launch_bounds__(256) topk_collect_kernel(TopkBufs b) {
  __shared__ uint32_t scratch[32];
  pdl_wait();
  pdl_launch_dependents();
  const int seg = blockIdx.y, chunk = blockIdx.x;
  const int lo = chunk * kTopkChunk;
  const int base = lo + 16 * threadIdx.x;
  const float* s = b.scores + (size_t)seg * b.capacity;
  float4 v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
    v[r] = base + 4 * r < b.nq ? *reinterpret_cast<const float4*>(s + base + 4 * r)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
  // b* = the largest bin whose suffix count reaches k (counts fall with b)
  const uint32_t* suf = b.hist + (size_t)seg * kHistBins;
  uint32_t sv[kHistBins / 256];
#pragma unroll
  for (int i = 0; i < kHistBins / 256; ++i) sv[i] = suf[(kHistBins / 256) * threadIdx.x + i];
  int best = -1;
#pragma unroll
  for (int i = 0; i < kHistBins / 256; ++i)
    if (sv[i] >= (uint32_t)b.k) best = (kHistBins / 256) * threadIdx.x + i;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(kAll, best, o));
  __shared__ int s_best[8];
  if ((threadIdx.x & 31) == 0) s_best[threadIdx.x >> 5] = best;
  __syncthreads();
  best = s_best[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) best = max(best, s_best[w]);
  const uint32_t bstar = (uint32_t)max(best, 0);
  if (chunk == 0 && threadIdx.x == 0) {
    uint32_t* ctr = b.counters + (size_t)seg * kCtrStride;
    ctr[2] = bstar;
    ctr[3] = bstar + 1 < (uint32_t)kHistBins ? suf[bstar + 1] : 0u;
  }
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

// Zero a segment's histogram and counters (all their readers are done).
__device__ __forceinline__ void clear_segment(uint32_t* hist, uint32_t* counters, int seg) {
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[(size_t)seg * kHistBins + i] = 0u;
  if (threadIdx.x < kCtrStride) counters[(size_t)seg * kCtrStride + threadIdx.x] = 0u;
}

// One CTA (256 threads) per segment.
__global__ void __launch_bounds__(256) topk_final_kernel(TopkBufs b, int32_t* idx,
                                                         uint32_t* hist_clear) {
  __shared__ uint32_t h[kHistBins];
  pdl_wait();
  pdl_launch_dependents();
  __shared__ uint2 st[kStageCap];
  __shared__ uint32_t scratch[32];
  __shared__ uint32_t off[65];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int seg = blockIdx.x;
  const int tid = threadIdx.x;
  const uint32_t* ctr = b.counters + (size_t)seg * kCtrStride;
  const uint32_t bstar = ctr[2];
  const uint32_t r = (uint32_t)b.k - ctr[3];  // keys to take from bin b* (>= 1)
  const uint2* lists = b.lists + (size_t)seg * b.n_chunks_cap * kTopkChunk;
  const uint32_t* counts = b.counts + (size_t)seg * b.n_chunks_cap;
  // chunk offsets in the concatenated (index-ordered) list
  if (tid < 32) {
    uint32_t run = 0;
    for (int c0 = 0; c0 < b.n_chunks; c0 += 32) {
      const int c = c0 + tid;
      const uint32_t v = c < b.n_chunks ? counts[c] : 0u;
      uint32_t x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kAll, x, o);
        if (tid >= o) x += y;
      }
      if (c < b.n_chunks && c < 64) off[c] = run + x - v;
      run += __shfl_sync(kAll, x, 31);
    }
    if (tid == 0) off[min(b.n_chunks, 64)] = run;
  }
  if (tid == 0) {
    s_bin = 0;
    s_above = 0;
  }
  __syncthreads();
  const uint32_t total = off[min(b.n_chunks, 64)];
  const bool staged = b.n_chunks <= 64 && total <= (uint32_t)kStageCap;
  int32_t* o = idx + (size_t)seg * b.k;

  if (staged) {
    // stage every list entry (loads independent of the shared-memory stores)
#pragma unroll 4
    for (uint32_t j = tid; j < total; j += 256) {
      int lo = 0, hi = b.n_chunks;  // last chunk with off[c] <= j
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= j) lo = mid;
        else hi = mid;
      }
      st[j] = lists[(size_t)lo * kTopkChunk + (j - off[lo])];
    }
    for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    // refinement 1: bits 20..10 of keys in bin b*
    for (uint32_t i = tid; i < total; i += blockDim.x) {
      const uint32_t key = st[i].x;
      if ((key >> 21) == bstar) atomicAdd(&h[(key >> 10) & 2047u], 1u);
    }
    __syncthreads();
    find_from_top(h, 2048, r, scratch, &s_bin, &s_above);
    const uint32_t d2 = (uint32_t)s_bin;
    const uint32_t r2 = r - s_above;
    const uint32_t pre = (bstar << 11) | d2;
    for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    // refinement 2: bits 9..0 of keys with prefix (b*, d2)
    for (uint32_t i = tid; i < total; i += blockDim.x) {
      const uint32_t key = st[i].x;
      if ((key >> 10) == pre) atomicAdd(&h[key & 1023u], 1u);
    }
    __syncthreads();
    find_from_top(h, 1024, r2, scratch, &s_bin, &s_above);
    const uint32_t kstar = (pre << 10) | (uint32_t)s_bin;
    const uint32_t r3 = r2 - s_above;
    // ordered pass; thread t owns entries [t*per, (t+1)*per) so one block scan
    // per counter orders the whole list
    const uint32_t per = (total + 255) / 256;
    const uint32_t i0 = tid * per, i1 = min(total, i0 + per);
    uint32_t n_eq = 0;
    for (uint32_t i = i0; i < i1; ++i) n_eq += st[i].x == kstar;
    uint32_t tot;
    uint32_t eq_rank = block_prefix_excl(n_eq, scratch, &tot);
    uint32_t n_ch = 0;
    for (uint32_t i = i0; i < i1; ++i) {
      const uint32_t key = st[i].x;
      const bool eq = key == kstar;
      n_ch += (key > kstar || (eq && eq_rank < r3)) ? 1u : 0u;
      eq_rank += eq;
    }
    uint32_t pos = block_prefix_excl(n_ch, scratch, &tot);
    eq_rank -= n_eq;  // back to this thread's first entry
    for (uint32_t i = i0; i < i1; ++i) {
      const uint2 e = st[i];
      const bool eq = e.x == kstar;
      if (e.x > kstar || (eq && eq_rank < r3)) {
        if (pos < (uint32_t)b.k) o[pos] = (int32_t)e.y;
        ++pos;
      }
      eq_rank += eq;
    }
    clear_segment(hist_clear, b.counters, seg);
    return;
  }

  // general path (long lists): the same steps reading the lists in place
  auto count_of = [&](int c) -> uint32_t { return counts[c]; };
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
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
  const uint32_t r3 = r2 - s_above;
  uint32_t out_base = 0, eq_base = 0;
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
  clear_segment(hist_clear, b.counters, seg);
}

// Histogram of the selection-score keys, turned into per-segment suffix
// counts (keys with bin >= b) by the last CTA of each segment.
__global__ void __launch_bounds__(256) score_hist_kernel(const float* scores, int capacity, int nq,
                                                         uint32_t* hist, uint32_t* counters) {
  __shared__ uint32_t sh[kHistBins];
  __shared__ bool s_last;
  pdl_wait();
  pdl_launch_dependents();
  const int seg = blockIdx.y;
  const int lo = blockIdx.x * kTopkChunk;
  const float* s = scores + (size_t)seg * capacity;
  float4 v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = lo + 4 * (threadIdx.x + 256 * r);
    v[r] = i < nq ? *reinterpret_cast<const float4*>(s + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (lo + 4 * (threadIdx.x + 256 * r) < nq) {
      atomicAdd(&sh[float_key(v[r].x) >> 21], 1u);
      atomicAdd(&sh[float_key(v[r].y) >> 21], 1u);
      atomicAdd(&sh[float_key(v[r].z) >> 21], 1u);
      atomicAdd(&sh[float_key(v[r].w) >> 21], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh = hist + (size_t)seg * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&counters[(size_t)seg * kCtrStride], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // thread t owns bins [8t, 8t + 8): all loads first, one block suffix scan
  constexpr int kPer = kHistBins / 256;
  uint32_t hv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) hv[i] = __ldcg(&gh[kPer * threadIdx.x + i]);
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) local += hv[i];
  __shared__ uint32_t scratch[32];
  uint32_t run = block_suffix_excl(local, scratch);  // keys in bins above this range
#pragma unroll
  for (int i = kPer - 1; i >= 0; --i) {
    run += hv[i];
    gh[kPer * threadIdx.x + i] = run;
  }
}

__global__ void topk_fill_kernel(int32_t* idx, int k, int nq) {
  const int seg = blockIdx.y;
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < k; i += gridDim.x * blockDim.x)
    idx[(size_t)seg * k + i] = i < nq ? i : -1;
}

int count_topk_launches(const jfa_geom& g, int k) {
  const int nq = split_point(g.n_ctx);
  return k >= nq ? 1 : 3;  // fill | histogram + collect + final
}

int launch_topk(const jfa_geom& g, int k, uint8_t* ws, const jfa_workspace_layout& L,
                int32_t* idx, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  if (k >= nq) {
    return launch_pdl(topk_fill_kernel, dim3((k + 255) / 256, n_seg), dim3(256), 0, st, idx, k,
                      nq) == cudaSuccess
               ? JFA_OK
               : JFA_ERR_CUDA;
  }
  TopkBufs b;
  b.scores = reinterpret_cast<const float*>(ws + L.off_scores);
  b.hist = reinterpret_cast<const uint32_t*>(ws + L.off_hist);
  b.counters = reinterpret_cast<uint32_t*>(ws + L.off_counters);
  b.lists = reinterpret_cast<uint2*>(ws + L.off_cand);
  b.counts = reinterpret_cast<uint32_t*>(ws + L.off_sel);
  b.capacity = g.capacity;
  b.nq = nq;
  b.k = k;
  b.n_chunks = (nq + kTopkChunk - 1) / kTopkChunk;
  b.n_chunks_cap = (g.capacity + kTopkChunk - 1) / kTopkChunk;
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + L.off_hist);
  // the histogram and counters start zero: the workspace is zero-filled at
  // allocation and every final kernel clears its segment when done
  cudaError_t e = launch_pdl(score_hist_kernel, dim3(b.n_chunks, n_seg), dim3(256), 0, st,
                             b.scores, g.capacity, nq, hist, b.counters);
  if (e == cudaSuccess)
    e = launch_pdl(topk_collect_kernel, dim3(b.n_chunks, n_seg), dim3(256), 0, st, b);
  if (e == cudaSuccess)
    e = launch_pdl(topk_final_kernel, dim3(n_seg), dim3(256), 0, st, b, idx, hist);
  return e == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

}  // namespace jfa

// ---------------------------------------------------------------------------
// Allocation-free top-k (jfa_topk_noalloc): the same three kernels, with their
// histogram, counters and lists in a fixed file-scope device array instead of
// a caller-allocated workspace.
// ---------------------------------------------------------------------------
namespace {
constexpr int kNoAllocMaxSeg = 64;     // segments per call
constexpr int kNoAllocMaxChunks = 64;  // segments x ceil(scores / 4096) per call
constexpr size_t kNoAllocHistWords = (size_t)kNoAllocMaxSeg * jfa::kHistBins;
constexpr size_t kNoAllocCtrWords = (size_t)kNoAllocMaxSeg * jfa::kCtrStride;
constexpr size_t kNoAllocCountOff = kNoAllocHistWords + kNoAllocCtrWords;
constexpr size_t kNoAllocListOff = (kNoAllocCountOff + kNoAllocMaxChunks + 63) / 64 * 64;
constexpr size_t kNoAllocWords = kNoAllocListOff + (size_t)kNoAllocMaxChunks * 4096 * 2;
}  // namespace

// About 2.5 MB; every device that loads the library holds it until exit.
static __device__ __align__(256) uint32_t g_topk_scratch[kNoAllocWords];

namespace jfa {

// Device address of g_topk_scratch on the current device (resolved once per
// device; the host-side name is only a stand-in, never a device address).
static uint32_t* noalloc_scratch() {
  static uint32_t* addr[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}

}  // namespace jfa

extern "C" int jfa_topk_noalloc(const float* scores, int32_t n_seg, int32_t stride,
                                int32_t n_scores, int32_t k, int32_t* idx, void* stream) {
  using namespace jfa;
  if (!scores || !idx || (reinterpret_cast<uintptr_t>(scores) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) != 0)
    return JFA_ERR_INVALID_ARG;
  if (n_seg < 1 || n_scores < 1 || n_scores % 4 != 0 || stride < n_scores || stride % 4 != 0 ||
      k < 1 || k > JFA_MAX_TOPK)
    return JFA_ERR_INVALID_ARG;
  const int n_chunks = (n_scores + kTopkChunk - 1) / kTopkChunk;
  if (n_seg > kNoAllocMaxSeg || (long long)n_seg * n_chunks > kNoAllocMaxChunks)
    return JFA_ERR_UNSUPPORTED;  // beyond the fixed scratch
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (k >= n_scores) {
    topk_fill_kernel<<<dim3((k + 255) / 256, n_seg), 256, 0, st>>>(idx, k, n_scores);
    return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
  }
  uint32_t* scratch = noalloc_scratch();
  if (scratch == nullptr) return JFA_ERR_CUDA;
  // the histogram and counters of the rows this call uses must start at zero
  // (the final kernel clears its row after use; an earlier call that stopped
  // short may not have): only those rows are cleared
  if (cudaMemsetAsync(scratch, 0, (size_t)n_seg * jfa::kHistBins * sizeof(uint32_t), st) != cudaSuccess ||
      cudaMemsetAsync(scratch + kNoAllocHistWords, 0, (size_t)n_seg * jfa::kCtrStride * sizeof(uint32_t),
                      st) != cudaSuccess)
    return JFA_ERR_CUDA;
  TopkBufs b;
  b.scores = scores;
  b.hist = scratch;
  b.counters = scratch + kNoAllocHistWords;
  b.counts = scratch + kNoAllocCountOff;
  b.lists = reinterpret_cast<uint2*>(scratch + kNoAllocListOff);
  b.capacity = stride;
  b.nq = n_scores;
  b.k = k;
  b.n_chunks = n_chunks;
  b.n_chunks_cap = n_chunks;
  score_hist_kernel<<<dim3(n_chunks, n_seg), 256, 0, st>>>(scores, stride, n_scores, scratch,
                                                          b.counters);
  topk_collect_kernel<<<dim3(n_chunks, n_seg), 256, 0, st>>>(b);
  topk_final_kernel<<<n_seg, 256, 0, st>>>(b, idx, scratch);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

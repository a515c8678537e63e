// topk.cu — jfa_topk: per (sequence, KV head) the k tokens with the largest
// selection score S (JetFire README, introduction: the top-k tokens are
// corrected; Jet-QSparse abstract: selection per KV head).
//
// Order (S descending, index ascending); output indices sorted ascending.
// Scores map to order-preserving 32-bit keys.  Three kernels:
//   1. histogram of the top 11 key bits per segment (many CTAs per segment);
//   2. every CTA finds the bin holding the k-th key, appends indices of keys
//      in higher bins to the segment's selected list and (key, index) pairs in
//      that bin to a candidate list;
//   3. one CTA per segment refines the candidates by the next 11 and 10 key
//      bits (radix select) to the exact k-th key, resolves ties by index,
//      and sorts the k chosen indices (bitonic, in shared memory).
// A candidate list that overflows its capacity falls back to reading S.
#include "jfa_internal.cuh"

namespace jfa {

constexpr unsigned kFullMask = 0xFFFFFFFFu;
constexpr uint32_t kRankCap = 1024;  // candidates handled by the counting-rank path

// Block-wide exclusive sum over threads in DESCENDING thread order:
// returns sum of v over threads with a larger index.  scratch: >= 32 uints.
__device__ uint32_t block_suffix_excl(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  // inclusive suffix within the warp
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_down_sync(kFullMask, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) scratch[warp] = x;  // warp total
  __syncthreads();
  uint32_t after = 0;
  for (int w = warp + 1; w < nw; ++w) after += scratch[w];
  __syncthreads();
  return after + (x - v);
}

// Given per-bin counts in h[0..nbins), find the bin where the count taken
// from the top reaches r.  Returns bin and count strictly above it.
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
// Same from the bottom (smallest bins first): bin where the count reaches r.
__device__ void find_from_bottom(const uint32_t* h, int nbins, uint32_t r, uint32_t* scratch,
                                 int* out_bin, uint32_t* out_below) {
  const int per = nbins / blockDim.x;
  // reverse the bin order so the suffix helper gives "count below"
  const int b0 = nbins - (threadIdx.x + 1) * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += h[b0 + i];
  uint32_t cum = block_suffix_excl(local, scratch);
  for (int i = 0; i < per; ++i) {
    const uint32_t c = h[b0 + i];
    if (cum < r && cum + c >= r) {
      *out_bin = b0 + i;
      *out_below = cum;
    }
    cum += c;
  }
  __syncthreads();
}

constexpr int kTopkChunk = 4096;  // scores per CTA of the histogram / collect kernels
constexpr int kCtrStride = 8;     // counters per segment: n_sel, n_cand, bstar, above, done

__global__ void __launch_bounds__(256) topk_hist_kernel(const float* scores, int capacity,
                                                        int nq, int k, uint32_t* hist,
                                                        uint32_t* counters) {
  __shared__ uint32_t sh[kHistBins];
  const int seg = blockIdx.y;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
  const int lo = blockIdx.x * kTopkChunk;
  const float* s = scores + (size_t)seg * capacity;
  float4 v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {  // nq is a multiple of 64: a float4 is all in or all out
    const int i = lo + 4 * (threadIdx.x + 256 * r);
    v[r] = i < nq ? *reinterpret_cast<const float4*>(s + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
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
  // the last CTA of the segment finds the bin holding the k-th key
  __shared__ bool s_last;
  __shared__ uint32_t scratch[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  uint32_t* ctr = counters + (size_t)seg * kCtrStride;
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
  find_from_top(sh, kHistBins, (uint32_t)k, scratch, &s_bin, &s_above);
  if (threadIdx.x == 0) {
    ctr[2] = (uint32_t)s_bin;
    ctr[3] = s_above;
  }
}

struct TopkBufs {
  const float* scores;
  uint32_t* hist;      // [n_seg][2048]
  uint32_t* counters;  // [n_seg][8]: n_sel, n_cand, bstar, above, hist CTAs done
  uint2* cand;         // [n_seg][cand_cap] (key, index)
  int32_t* sel;        // [n_seg][max_topk]
  int capacity, nq, k, cand_cap, max_topk;
};

__global__ void __launch_bounds__(256) topk_collect_kernel(TopkBufs b) {
  const int seg = blockIdx.y;
  const int lo = blockIdx.x * kTopkChunk;
  const float* s = b.scores + (size_t)seg * b.capacity;
  float4 v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = lo + 4 * (threadIdx.x + 256 * r);
    v[r] = i < b.nq ? *reinterpret_cast<const float4*>(s + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  uint32_t* ctr = b.counters + (size_t)seg * kCtrStride;
  const uint32_t bstar = ctr[2];
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int32_t* sel = b.sel + (size_t)seg * b.max_topk;
  uint2* cand = b.cand + (size_t)seg * b.cand_cap;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i0 = lo + 4 * (threadIdx.x + 256 * r);
    const float vals[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + e;
      const bool valid = i0 < b.nq;
      const uint32_t key = float_key(vals[e]);
      const uint32_t bin = key >> 21;
      const bool is_sel = valid && bin > bstar;
      const bool is_cand = valid && bin == bstar;
      const unsigned ms = __ballot_sync(kFullMask, is_sel);
      if (ms) {
        uint32_t pos = 0;
        if (lane == __ffs(ms) - 1) pos = atomicAdd(&ctr[0], (uint32_t)__popc(ms));
        pos = __shfl_sync(kFullMask, pos, __ffs(ms) - 1);
        if (is_sel) sel[pos + __popc(ms & lt)] = i;
      }
      const unsigned mc = __ballot_sync(kFullMask, is_cand);
      if (mc) {
        uint32_t pos = 0;
        if (lane == __ffs(mc) - 1) pos = atomicAdd(&ctr[1], (uint32_t)__popc(mc));
        pos = __shfl_sync(kFullMask, pos, __ffs(mc) - 1);
        const uint32_t mine = pos + __popc(mc & lt);
        if (is_cand && mine < (uint32_t)b.cand_cap) cand[mine] = make_uint2(key, (uint32_t)i);
      }
    }
  }
}

// One CTA (1024 threads) per segment.
__global__ void __launch_bounds__(1024) topk_final_kernel(TopkBufs b, int32_t* idx) {
  __shared__ uint32_t h[kHistBins];
  __shared__ int32_t out[JFA_MAX_TOPK];
  __shared__ uint32_t scratch[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_cnt, s_nout;
  const int seg = blockIdx.x;
  const int tid = threadIdx.x;
  const uint32_t* ctr = b.counters + (size_t)seg * kCtrStride;
  const uint32_t n_sel = ctr[0], n_cand = ctr[1], bstar = ctr[2];
  const uint32_t r = (uint32_t)b.k - n_sel;  // >= 1
  const int32_t* sel = b.sel + (size_t)seg * b.max_topk;
  for (uint32_t i = tid; i < n_sel; i += blockDim.x) out[i] = sel[i];
  const bool from_cand = n_cand <= (uint32_t)b.cand_cap;
  if (from_cand && n_cand <= kRankCap && b.k <= (int)blockDim.x) {
    // small case: rank every candidate by counting (no refinement passes),
    // then rank the k chosen indices by counting to sort them
    uint32_t* ck = h;                                  // keys   [<= 1024]
    int32_t* cx = reinterpret_cast<int32_t*>(h) + kRankCap;  // indices
    const uint2* cand = b.cand + (size_t)seg * b.cand_cap;
    for (uint32_t i = tid; i < n_cand; i += blockDim.x) {
      const uint2 c = cand[i];
      ck[i] = c.x;
      cx[i] = (int32_t)c.y;
    }
    __syncthreads();
    if (tid < n_cand) {
      const uint32_t key = ck[tid];
      const int32_t ix = cx[tid];
      uint32_t rank = 0;
      for (uint32_t j = 0; j < n_cand; ++j) {
        const uint32_t kj = ck[j];
        rank += (kj > key) || (kj == key && cx[j] < ix);
      }
      if (rank < r) out[n_sel + rank] = ix;
    }
    __syncthreads();
    int32_t mine = 0;
    uint32_t pos = 0;
    if (tid < b.k) {
      mine = out[tid];
      for (int j = 0; j < b.k; ++j) pos += out[j] < mine;
    }
    __syncthreads();
    if (tid < b.k) out[pos] = mine;
    __syncthreads();
    int32_t* o = idx + (size_t)seg * b.k;
    if (tid < b.k) o[tid] = out[tid];
    return;
  }
  const uint2* cand = b.cand + (size_t)seg * b.cand_cap;
  const float* s = b.scores + (size_t)seg * b.capacity;
  const uint32_t n_src = from_cand ? n_cand : (uint32_t)b.nq;
  // element j of the source: (key, index, member of the threshold bin?)
  auto src = [&](uint32_t j, uint32_t& key, int32_t& ix) -> bool {
    if (from_cand) {
      const uint2 c = cand[j];
      key = c.x;
      ix = (int32_t)c.y;
      return true;
    }
    key = float_key(s[j]);
    ix = (int32_t)j;
    return (key >> 21) == bstar;
  };

  // refine bits 20..10
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
  if (tid == 0) s_nout = n_sel;
  __syncthreads();
  for (uint32_t j = tid; j < n_src; j += blockDim.x) {
    uint32_t key;
    int32_t ix;
    if (src(j, key, ix)) atomicAdd(&h[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  int d2 = 0;
  uint32_t above2 = 0;
  find_from_top(h, 2048, r, scratch, &s_bin, &s_cnt);
  d2 = s_bin;
  above2 = s_cnt;
  const uint32_t r2 = r - above2;
  // refine bits 9..0
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (uint32_t j = tid; j < n_src; j += blockDim.x) {
    uint32_t key;
    int32_t ix;
    if (src(j, key, ix) && ((key >> 10) & 2047u) == (uint32_t)d2) atomicAdd(&h[key & 1023u], 1u);
  }
  __syncthreads();
  find_from_top(h, 1024, r2, scratch, &s_bin, &s_cnt);
  const int d3 = s_bin;
  const uint32_t r3 = r2 - s_cnt;        // ties to take at the exact k-th key
  const uint32_t n_eq = h[d3];
  const uint32_t kstar = (bstar << 21) | ((uint32_t)d2 << 10) | (uint32_t)d3;
  __syncthreads();

  // smallest r3 indices among keys == kstar: index threshold istar
  int32_t istar = 0x7FFFFFFF;
  if (r3 < n_eq) {
    uint32_t need = r3;
    uint32_t prefix = 0;  // high index bits fixed so far
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = 22 - 11 * pass;   // bits 32..22, 21..11, 10..0
      const uint32_t nb = 2048;
      for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
      __syncthreads();
      for (uint32_t j = tid; j < n_src; j += blockDim.x) {
        uint32_t key;
        int32_t ix;
        if (src(j, key, ix) && key == kstar) {
          const uint32_t ux = (uint32_t)ix;
          const bool match = pass == 0 || (ux >> (shift + 11)) == prefix;
          if (match) atomicAdd(&h[(ux >> shift) & (nb - 1)], 1u);
        }
      }
      __syncthreads();
      find_from_bottom(h, 2048, need, scratch, &s_bin, &s_cnt);
      need -= s_cnt;
      prefix = (prefix << 11) | (uint32_t)s_bin;
      __syncthreads();
    }
    istar = (int32_t)prefix;
  }

  // collect the rest of the selection from the source
  for (uint32_t j = tid; j < n_src; j += blockDim.x) {
    uint32_t key;
    int32_t ix;
    if (!src(j, key, ix)) continue;
    if (key > kstar || (key == kstar && ix <= istar)) {
      const uint32_t pos = atomicAdd(&s_nout, 1u);
      if (pos < (uint32_t)b.k) out[pos] = ix;
    }
  }
  __syncthreads();
  // bitonic sort out[0..npow) ascending
  int npow = 1;
  while (npow < b.k) npow <<= 1;
  for (int i = b.k + tid; i < npow; i += blockDim.x) out[i] = 0x7FFFFFFF;
  __syncthreads();
  if (npow <= (int)blockDim.x) {
    // one element per thread; strides below 32 exchange through shuffles
    int32_t x = tid < npow ? out[tid] : 0x7FFFFFFF;
    for (int size = 2; size <= npow; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        int32_t y;
        if (stride >= 32) {
          __syncthreads();
          if (tid < npow) out[tid] = x;
          __syncthreads();
          y = tid < npow ? out[tid ^ stride] : 0x7FFFFFFF;
        } else {
          y = __shfl_xor_sync(kFullMask, x, stride);
        }
        const bool up = (tid & size) == 0;
        const bool lower = (tid & stride) == 0;
        // the lower element of a pair keeps the min when sorting up
        x = (lower == up) ? min(x, y) : max(x, y);
      }
    }
    __syncthreads();
    if (tid < npow) out[tid] = x;
  } else {
    for (int size = 2; size <= npow; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < npow / 2; i += blockDim.x) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool up = (lo & size) == 0;
          const int32_t a = out[lo], c = out[hi];
          if ((a > c) == up) {
            out[lo] = c;
            out[hi] = a;
          }
        }
        __syncthreads();
      }
    }
  }
  __syncthreads();
  int32_t* o = idx + (size_t)seg * b.k;
  for (int i = tid; i < b.k; i += blockDim.x) o[i] = out[i];
}

__global__ void topk_fill_kernel(int32_t* idx, int k, int nq) {
  const int seg = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < k; i += gridDim.x * blockDim.x)
    idx[(size_t)seg * k + i] = i < nq ? i : -1;
}

static int topk_chunks(int nq, int n_seg) {
  (void)n_seg;
  return (nq + kTopkChunk - 1) / kTopkChunk;
}

int count_topk_launches(const jfa_geom& g, int k) {
  const int nq = split_point(g.n_ctx);
  return k >= nq ? 1 : 4;  // fill | memset + hist + collect + final
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
  b.cand = reinterpret_cast<uint2*>(ws + L.off_cand);
  b.sel = reinterpret_cast<int32_t*>(ws + L.off_sel);
  b.capacity = g.capacity;
  b.nq = nq;
  b.k = k;
  b.cand_cap = L.cand_cap;
  b.max_topk = L.max_topk;
  // histograms and counters are contiguous: clear both at once
  if (cudaMemsetAsync(ws + L.off_hist, 0, L.off_cand - L.off_hist, st) != cudaSuccess)
    return JFA_ERR_CUDA;
  const int chunks = topk_chunks(nq, n_seg);
  topk_hist_kernel<<<dim3(chunks, n_seg), 256, 0, st>>>(b.scores, g.capacity, nq, k, b.hist,
                                                       b.counters);
  topk_collect_kernel<<<dim3(chunks, n_seg), 256, 0, st>>>(b);
  topk_final_kernel<<<n_seg, 1024, 0, st>>>(b, idx);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

}  // namespace jfa

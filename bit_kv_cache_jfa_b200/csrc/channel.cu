// channel.cu — critical-channel scores (TailorKV review: the importance of a
// channel is the query's magnitude in it times the largest key magnitude in
// it, s_i = |q_i| * max|K_i|; approximate attention scores over the critical
// channels pick the tokens that are then fetched and attended exactly).
//
//   channel_pack_kernel    one CTA per (64-token group, segment): writes the
//                          group's keys channel-major (k_t [seg][128][cap],
//                          bf16) and raises the segment's per-channel max|K|;
//   channel_select_kernel  one CTA per segment: ranks the 128 channels by
//                          importance (largest |q_i| over the KV head's query
//                          heads times max|K_i|, both bf16 values so the fp32
//                          product is exact) and keeps the r best (ties to the
//                          lower channel), with the scaled query at them;
//   channel_scores_kernel  one CTA per (1024 tokens, segment): streams the r
//                          kept channel rows of k_t, 4 tokens per thread: the
//                          selection score of a token is the largest over the
//                          query heads of scale * sum_i q_{h,i} K_{t,i}.
// HBM-bound: 2 r bytes read and 4 written per token and KV head.
#include "jfa_fp4.cuh"

namespace jfa {

constexpr int kChTok = 1024;  // tokens per CTA of the score kernel (256 threads x 4)

__device__ __forceinline__ float bf16f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__global__ void __launch_bounds__(256) channel_pack_kernel(const uint16_t* __restrict__ k_src,
                                                           uint16_t* __restrict__ k_t,
                                                           float* __restrict__ k_max, int capacity,
                                                           int g_from) {
  __shared__ uint16_t tile[kKG][kD + 8];
  const int seg = blockIdx.y, t0 = (g_from + blockIdx.x) * kKG, tid = threadIdx.x;
  const uint16_t* src = k_src + ((size_t)seg * capacity + t0) * kD;
  for (int i = tid; i < kKG * kD / 8; i += 256) {
    const int row = i >> 4, ch = i & 15;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (size_t)row * kD + ch * 8);
    uint32_t* d = reinterpret_cast<uint32_t*>(&tile[row][ch * 8]);
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
  __syncthreads();
  if (tid < kD) {
    float m = 0.f;
    for (int r = 0; r < kKG; ++r) m = fmaxf(m, fabsf(bf16f(tile[r][tid])));
    // non-negative floats order like their bit patterns
    atomicMax(reinterpret_cast<int*>(k_max + (size_t)seg * kD + tid), __float_as_int(m));
  }
  // channel c = tid / 2, tokens 32 (tid mod 2) .. +31: 64 contiguous bytes
  const int c = tid >> 1, h = tid & 1;
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j)
    w[j] = (uint32_t)tile[32 * h + 2 * j][c] | ((uint32_t)tile[32 * h + 2 * j + 1][c] << 16);
  uint4* dst = reinterpret_cast<uint4*>(k_t + ((size_t)seg * kD + c) * capacity + t0 + 32 * h);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

struct ChanParams {
  const uint16_t* k_t;
  const float* k_max;
  const uint16_t* q;
  float* scores;
  uint8_t* chan;  // per-segment channel records
  int capacity, H, Hkv, G, nq, r;
  float scale;
};

// One CTA per segment: the importance of every channel, its rank
// (importance descending, index ascending) and the kept channels with the
// scaled query at them, written to the segment's channel record.
__global__ void __launch_bounds__(128) channel_select_kernel(const __grid_constant__ ChanParams p) {
  __shared__ float imp[kD];
  __shared__ int wcount[4];
  const int seg = blockIdx.x, b = seg / p.Hkv, kvh = seg % p.Hkv, tid = threadIdx.x;
  pdl_launch_dependents();  // the score kernel's set-up may overlap; it waits for this grid
  pdl_wait();
  float qv[kMaxG];
  float qm = 0.f;
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) {
    qv[h] = h < p.G ? bf16f(p.q[((size_t)b * p.H + kvh * p.G + h) * kD + tid]) : 0.f;
    qm = fmaxf(qm, fabsf(qv[h]));
  }
  const float mine = qm * p.k_max[(size_t)seg * kD + tid];
  imp[tid] = mine;
  __syncthreads();
  int rank = 0;
#pragma unroll 16
  for (int c = 0; c < kD; ++c) {
    const float o = imp[c];
    rank += (o > mine) || (o == mine && c < tid);
  }
  const bool keep = rank < p.r;
  const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
  if ((tid & 31) == 0) wcount[tid >> 5] = __popc(bal);
  __syncthreads();
  if (keep) {
    int pos = __popc(bal & ((1u << (tid & 31)) - 1u));
    for (int w = 0; w < (tid >> 5); ++w) pos += wcount[w];
    uint8_t* rec = p.chan + (size_t)seg * kChanRecBytes;
    reinterpret_cast<int*>(rec)[pos] = tid;
    float* qs = reinterpret_cast<float*>(rec + 128 * 4);
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) qs[h * kD + pos] = qv[h] * p.scale;
  }
}

// One CTA per (1024 tokens, segment), 4 tokens per thread.
__global__ void __launch_bounds__(256, 4) channel_scores_kernel(const __grid_constant__ ChanParams p) {
  __shared__ float qs[kMaxG][kD];
  __shared__ int chans[kD];
  const int seg = blockIdx.y, tid = threadIdx.x;
  pdl_wait();
  const uint8_t* rec = p.chan + (size_t)seg * kChanRecBytes;
  for (int i = tid; i < p.r; i += 256) chans[i] = reinterpret_cast<const int*>(rec)[i];
  for (int i = tid; i < kMaxG * kD; i += 256) {
    const int h = i / kD, j = i % kD;
    if (h < p.G && j < p.r) qs[h][j] = reinterpret_cast<const float*>(rec + 128 * 4)[i];
  }
  __syncthreads();

  const int t = blockIdx.x * kChTok + tid * 4;
  if (t >= p.nq) return;
  float acc[kMaxG][4];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
  const uint16_t* base = p.k_t + (size_t)seg * kD * p.capacity + t;
  // 8 channel rows per round: their loads are in flight together
  for (int j0 = 0; j0 < p.r; j0 += 8) {
    uint2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = j0 + u < p.r ? *reinterpret_cast<const uint2*>(base + (size_t)chans[j0 + u] * p.capacity)
                          : make_uint2(0, 0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (j0 + u >= p.r) break;
      const float k4[4] = {__uint_as_float(v[u].x << 16), __uint_as_float(v[u].x & 0xFFFF0000u),
                           __uint_as_float(v[u].y << 16), __uint_as_float(v[u].y & 0xFFFF0000u)};
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        if (h < p.G) {
          const float qv = qs[h][j0 + u];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][e] = fmaf(qv, k4[e], acc[h][e]);
        }
      }
    }
  }
  float s[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float m = acc[0][e];
#pragma unroll
    for (int h = 1; h < kMaxG; ++h)
      if (h < p.G) m = fmaxf(m, acc[h][e]);
    s[e] = m;
  }
  *reinterpret_cast<float4*>(p.scores + (size_t)seg * p.capacity + t) = make_float4(s[0], s[1], s[2], s[3]);
  pdl_launch_dependents();
}

int launch_channel_pack(const jfa_geom& g, int g_from, int g_to, const uint16_t* k_src, uint16_t* k_t,
                        float* k_max, cudaStream_t st) {
  if (g_to <= g_from) return JFA_OK;
  const int n_seg = g.batch * g.num_kv_heads;
  channel_pack_kernel<<<dim3(g_to - g_from, n_seg), 256, 0, st>>>(k_src, k_t, k_max, g.capacity, g_from);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

int launch_channel_scores(const jfa_geom& g, const uint16_t* k_t, const float* k_max, const uint16_t* q,
                          float scale, int r, uint8_t* ws, const jfa_workspace_layout& L,
                          cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  ChanParams p;
  p.k_t = k_t;
  p.k_max = k_max;
  p.q = q;
  p.scores = reinterpret_cast<float*>(ws + L.off_scores);
  p.chan = ws + L.off_chan;
  p.capacity = g.capacity;
  p.H = g.num_heads;
  p.Hkv = g.num_kv_heads;
  p.G = g.num_heads / g.num_kv_heads;
  p.nq = split_point(g.n_ctx);
  p.r = r;
  p.scale = scale;
  if (p.nq == 0) return JFA_OK;
  if (launch_pdl(channel_select_kernel, dim3(n_seg), dim3(kD), 0, st, p) != cudaSuccess)
    return JFA_ERR_CUDA;
  const int chunks = (p.nq + kChTok - 1) / kChTok;
  return launch_pdl(channel_scores_kernel, dim3(chunks, n_seg), dim3(256), 0, st, p) == cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

}  // namespace jfa

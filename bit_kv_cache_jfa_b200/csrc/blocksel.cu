// blocksel.cu — jfa_topk_blocks: selection of 128-token blocks instead of
// single tokens (Jet-QSparse abstract: 128-token blocks are selected for the
// sparse high-precision value aggregation, which then reads contiguous tiles
// of the exact rows).
//
// One CTA per (sequence, KV head):
//   1. block keys: the largest selection score of every 128-token block of
//      the N_q quantized tokens (the last block may hold 64), as an
//      order-preserving key, one warp per block (a float4 per lane, warp max);
//   2. the chosen blocks: up to 512 blocks by counting each block's rank
//      directly, else the n-th largest key by three radix levels (11 + 11 +
//      10 bits) over the block keys in shared memory; equal keys go to the
//      lower block;
//   3. one ordered pass lists the chosen blocks ascending, and every chosen
//      block writes its 128 token indices (t >= N_q of a partial block and
//      the unused tail of idx are -1).
#include "jfa_blocks.cuh"

namespace jfa {

constexpr int kSelBlock = JFA_BLOCK_TOKENS;
constexpr int kBlkThreads = 256;
constexpr int kBlkDirect = 512;  // direct ranking up to this many blocks

__global__ void __launch_bounds__(kBlkThreads) block_select_kernel(const float* scores,
                                                                   const uint32_t* bkeys, int capacity,
                                                                   int nq, int n_sel, int out_len,
                                                                   int32_t* idx) {
  extern __shared__ uint32_t bsm[];
  const int nb = (nq + kSelBlock - 1) / kSelBlock;
  uint32_t* keys = bsm;                           // [nb]
  uint32_t* hist = bsm + ((nb + 3) & ~3);         // [2048]
  uint32_t* chosen = hist + 2048;                 // [n_sel] block ids, ascending
  __shared__ uint32_t scratch[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  pdl_wait();
  pdl_launch_dependents();
  const int seg = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* S = scores + (size_t)seg * capacity;

  // 1. block keys: given, or the largest stored score of every block (nq is
  // a multiple of 64, so a float4 never straddles nq); a warp takes 4 blocks
  // at a time so that 4 loads per lane are in flight
  if (bkeys) {
    const uint32_t* K = bkeys + (size_t)seg * ((capacity + kSelBlock - 1) / kSelBlock);
    for (int b = tid; b < nb; b += kBlkThreads) keys[b] = K[b];
  } else {
    constexpr int kWarps = kBlkThreads / 32;
    for (int b0 = 4 * warp; b0 < nb; b0 += 4 * kWarps) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t0 = kSelBlock * (b0 + u) + 4 * lane;
        v[u] = (b0 + u < nb && t0 < nq) ? *reinterpret_cast<const float4*>(S + t0)
                                        : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float m = fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kAll, m, o));
        if (lane == 0 && b0 + u < nb) keys[b0 + u] = float_key(m);
      }
    }
  }
  __syncthreads();

  // 2. which blocks are chosen (n_eff = min(n_sel, nb) of them).  Up to
  // kBlkDirect blocks every block's rank is counted directly (flags in
  // hist[]): a radix histogram of a few hundred near-equal maxima would
  // serialize its shared-memory atomics on a handful of bins.  Beyond that,
  // the n_eff-th largest key by three radix levels.
  const int n_eff = min(n_sel, nb);
  const bool direct = n_eff < nb && nb <= kBlkDirect;
  uint32_t kstar = 0, r = (uint32_t)n_eff;
  if (direct) {
    for (int i = tid; i < nb; i += kBlkThreads) {
      const uint32_t mine = keys[i];
      uint32_t rank = 0;
      for (int c = 0; c < nb; ++c) {
        const uint32_t o = keys[c];
        rank += (o > mine) | ((o == mine) & (c < i));
      }
      hist[i] = rank < (uint32_t)n_eff ? 1u : 0u;
    }
    __syncthreads();
  } else if (n_eff < nb) {
    const int shifts[3] = {21, 10, 0};
    const int bits[3] = {11, 11, 10};
    uint32_t prefix = 0;
#pragma unroll 1
    for (int lv = 0; lv < 3; ++lv) {
      const int nbins = 1 << bits[lv];
      for (int i = tid; i < 2048; i += kBlkThreads) hist[i] = 0u;
      __syncthreads();
      const int hs = lv == 0 ? 32 : shifts[lv - 1];
      for (int i = tid; i < nb; i += kBlkThreads) {
        const uint32_t key = keys[i];
        if (lv == 0 || (key >> hs) == prefix) atomicAdd(&hist[(key >> shifts[lv]) & (nbins - 1)], 1u);
      }
      __syncthreads();
      find_from_top(hist, nbins, r, scratch, &s_bin, &s_above);
      prefix = (prefix << bits[lv]) | (uint32_t)s_bin;
      r -= s_above;
      __syncthreads();
    }
    kstar = prefix;  // take every key above it and the first r equal to it
  }

  // 3. the chosen blocks in ascending order: thread t owns blocks
  // [t*per, (t+1)*per); the equal keys before a thread decide its ties
  const int per = (nb + kBlkThreads - 1) / kBlkThreads;
  const int i0 = min(nb, tid * per), i1 = min(nb, i0 + per);
  const bool radix = n_eff < nb && !direct;
  auto take_at = [&](int i, uint32_t e) -> bool {
    if (n_eff >= nb) return true;
    if (direct) return hist[i] != 0u;
    return keys[i] > kstar || (keys[i] == kstar && e < r);
  };
  uint32_t tot;
  uint32_t n_eq = 0;
  if (radix)
    for (int i = i0; i < i1; ++i) n_eq += keys[i] == kstar;
  uint32_t er = block_prefix_excl(n_eq, scratch, &tot);
  uint32_t nc = 0;
  {
    uint32_t e2 = er;
    for (int i = i0; i < i1; ++i) {
      nc += take_at(i, e2);
      e2 += (radix && keys[i] == kstar) ? 1u : 0u;
    }
  }
  uint32_t pos = block_prefix_excl(nc, scratch, &tot);
  for (int i = i0; i < i1; ++i) {
    if (take_at(i, er)) chosen[pos++] = (uint32_t)i;
    er += (radix && keys[i] == kstar) ? 1u : 0u;
  }
  __syncthreads();

  // 4. token indices: chosen block p fills idx[128 p .. 128 p + 127]
  int32_t* out = idx + (size_t)seg * out_len;
  for (int j = tid; j < out_len; j += kBlkThreads) {
    const int p = j / kSelBlock;
    int v = -1;
    if (p < n_eff) {
      const int t = kSelBlock * (int)chosen[p] + (j % kSelBlock);
      v = t < nq ? t : -1;
    }
    out[j] = v;
  }
}

static_assert((kMaxSelBlocks + 2048 + JFA_MAX_BLOCKS) * 4 <= 48 * 1024, "block keys fit the default shared memory");

size_t block_select_smem(int nq, int n_blocks) {
  const int nb = (nq + kSelBlock - 1) / kSelBlock;
  return (size_t)(((nb + 3) & ~3) + 2048 + n_blocks) * sizeof(uint32_t);
}

int launch_topk_blocks(const jfa_geom& g, int n_blocks, uint8_t* ws, const jfa_workspace_layout& L,
                       int32_t* idx, cudaStream_t st, const uint32_t* bkeys) {
  const int n_seg = g.batch * g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  const int out_len = n_blocks * kSelBlock;
  // at most kMaxSelBlocks block keys: 40 KB, inside the default 48 KB
  const size_t smem = block_select_smem(nq, n_blocks);
  return launch_pdl(block_select_kernel, dim3(n_seg), dim3(kBlkThreads), smem, st,
                    reinterpret_cast<const float*>(ws + L.off_scores), bkeys, g.capacity, nq, n_blocks,
                    out_len, idx) == cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

}  // namespace jfa

// sparse.cu — exact softmax attention over a chosen token set and the
// exact tail, nothing else (Jet-QSparse abstract: sparse value aggregation
// over the selected 128-token blocks in high precision with FP32
// accumulation; contiguous blocks make the row loads contiguous tiles).
//
// Every (sequence, KV head) has E = k + (n_ctx - N_q) entries: idx[0..k)
// (token indices, -1 = none) then the tail tokens N_q .. n_ctx - 1.  A CTA
// takes an even share of the entries in runs of 16; each of its 4 warps
// streams its runs' K and V rows (bf16, 256 B each) into a private 2-stage
// ring (cp.async, XOR-swizzled 16-byte chunks; 3 CTAs per SM: more warps
// beat deeper rings here, measured) and runs, per run:
//   logits   S^T = q K^T on mma.sync m16n8k16 (bf16 in, fp32 accumulate),
//            rows = the KV head's query heads, so each lane holds the
//            logits of head lane/4 for 4 of the 16 tokens;
//   softmax  an online (m, l) per head in log2 units;
//   values   O += P V with P split into a bf16 high part (rows 0-7) and the
//            bf16 remainder (rows 8-15) of the same MMA: the two row halves
//            add up to P V at about 16 bits of P.
// The warps' partials merge in shared memory; the CTAs of a segment write
// theirs to the workspace and the last one to finish (a ticket counter)
// merges them and writes out.
#include "jfa_fp4.cuh"

namespace jfa {

#ifndef JFA_SP_WARPS
#define JFA_SP_WARPS 4
#endif
#ifndef JFA_SP_STAGES
#define JFA_SP_STAGES 2
#endif
#ifndef JFA_SP_CTAS_PER_SM
#define JFA_SP_CTAS_PER_SM 3
#endif
constexpr int kSpWarps = JFA_SP_WARPS;
constexpr int kSpThreads = 32 * kSpWarps;
constexpr int kSpStages = JFA_SP_STAGES;
constexpr int kSpRun = 16;                        // entries per run (one MMA k-step of P V)
constexpr int kSpStageBytes = 2 * kSpRun * kD * 2;  // K rows, then V rows
constexpr int kSpSmem = kSpWarps * kSpStages * kSpStageBytes;
constexpr int kSpPart = 132;                      // floats per (partial, head): m, l, pad, pad, acc
static_assert(kSpWarps * kMaxG * kSpPart * 4 <= kSpSmem, "warp partials fit the rings");

struct SparseParams {
  const uint16_t* q;
  const int32_t* idx;
  const uint16_t* kx;
  const uint16_t* vx;
  float* out;
  float* part;
  uint32_t* ticket;
  uint32_t* flag;
  int k, capacity, H, Hkv, G, nq, n_ctx, n_split, on_host;
  float scale_log2;  // softmax scale * log2(e)
};

__device__ __forceinline__ void mma_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// 16-byte copy, zero-filled when n == 0 (nothing read).
__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ uint32_t bf16_pair(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Byte of (row, 16-byte chunk) in a 16-row tile of 256-byte rows.
__device__ __forceinline__ uint32_t sw_off(int row, int chunk) {
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}

// Token of entry e, -1 for none; an index outside [-1, N_q) is flagged and
// skipped.
__device__ __forceinline__ int entry_token(const SparseParams& p, const int32_t* ix, int E, int e) {
  if (e >= E) return -1;
  if (e < p.k) {
    const int t = ix[e];
    if (t < -1 || t >= p.nq) {
      set_flag(p.flag, JFA_DEVERR_BAD_INDEX);
      return -1;
    }
    return t;
  }
  return p.nq + (e - p.k);
}

__global__ void __launch_bounds__(kSpThreads, JFA_SP_CTAS_PER_SM) sparse_attend_kernel(const __grid_constant__ SparseParams p) {
  extern __shared__ __align__(128) uint8_t spm[];
  __shared__ int s_last;
  const int seg = blockIdx.x / p.n_split, split = blockIdx.x % p.n_split;
  const int b = seg / p.Hkv, kvh = seg % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int E = p.k + (p.n_ctx - p.nq);
  const int nrun = (E + kSpRun - 1) / kSpRun;
  const int r_lo = (int)((long long)split * nrun / p.n_split);
  const int r_hi = (int)((long long)(split + 1) * nrun / p.n_split);
  const int n_mine = r_hi - r_lo > warp ? (r_hi - r_lo - warp + kSpWarps - 1) / kSpWarps : 0;
  const uint16_t* K = p.kx + (size_t)seg * p.capacity * kD;
  const uint16_t* V = p.vx + (size_t)seg * p.capacity * kD;
  const int32_t* ix = p.idx + (size_t)seg * p.k;
  uint8_t* ring = spm + warp * kSpStages * kSpStageBytes;
  const uint32_t ring_s = smem_u32(ring);

  pdl_wait();
  // query fragments: A rows 0-7 = heads (rows >= G and 8-15 zero)
  uint32_t qa[8][2];
  {
    const uint16_t* qh = p.q + ((size_t)b * p.H + kvh * p.G + g) * kD + 2 * t4;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = g < p.G ? *reinterpret_cast<const uint32_t*>(qh + 16 * ks) : 0u;
      qa[ks][1] = g < p.G ? *reinterpret_cast<const uint32_t*>(qh + 16 * ks + 8) : 0u;
    }
  }

  // run j of this warp: entries 16 (r_lo + warp + 4 j) ..; lane < 16 holds
  // the token of row = lane.  The tokens of the next run are loaded one run
  // ahead (their global load overlaps the current run's work) and every
  // issued run's tokens stay in shared memory until it is computed.
  __shared__ int tok_s[kSpWarps][kSpStages][kSpRun];
  auto run_token = [&](int j) -> int {
    return (lane < kSpRun && j < n_mine)
               ? entry_token(p, ix, E, kSpRun * (r_lo + warp + kSpWarps * j) + lane)
               : -1;
  };
  auto issue = [&](int j, int mytok) {
    if (lane < kSpRun) tok_s[warp][j % kSpStages][lane] = mytok;
    const uint32_t st = ring_s + (uint32_t)((j % kSpStages) * kSpStageBytes);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int lin = (i & 7) * 32 + lane, row = lin >> 4, ch = lin & 15;
      const int tok = __shfl_sync(0xFFFFFFFFu, mytok, row);
      const uint16_t* src = (i < 8 ? K : V) + (size_t)(tok < 0 ? 0 : tok) * kD + ch * 8;
      const uint32_t dst = st + (i < 8 ? 0u : (uint32_t)(kSpRun * 256)) + sw_off(row, ch);
      if (p.on_host) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (tok >= 0) v = *reinterpret_cast<const uint4*>(src);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z),
                     "r"(v.w)
                     : "memory");
      } else {
        cp16_zfill(dst, src, tok < 0 ? 0u : 16u);
      }
    }
  };

  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m = -INFINITY, l = 0.f;

  int next_tok = run_token(0);
#pragma unroll
  for (int j = 0; j < kSpStages - 1; ++j) {
    if (j < n_mine) {
      const int mytok = next_tok;
      next_tok = run_token(j + 1);
      issue(j, mytok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int j = 0; j < n_mine; ++j) {
    if (j + kSpStages - 1 < n_mine) {
      const int mytok = next_tok;
      next_tok = run_token(j + kSpStages);
      issue(j + kSpStages - 1, mytok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group %0;" ::"n"(kSpStages - 1) : "memory");
    __syncwarp();
    const unsigned valid =
        __ballot_sync(0xFFFFFFFFu, lane < kSpRun && tok_s[warp][j % kSpStages][lane] >= 0);
    const uint32_t kb = ring_s + (uint32_t)((j % kSpStages) * kSpStageBytes);
    const uint32_t vb = kb + kSpRun * 256;

    // logits of head g for tokens 2t4, 2t4+1 (s0) and 8+2t4, 9+2t4 (s1)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int mi = lane >> 3, tok = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kb + sw_off(tok, 2 * ks + (mi & 1)), r0, r1, r2, r3);
        mma_bf16(s0, qa[ks][0], 0u, qa[ks][1], 0u, r0, r1);
        mma_bf16(s1, qa[ks][0], 0u, qa[ks][1], 0u, r2, r3);
      }
    }
    const int tk = 2 * t4;
    const float x0 = (valid >> tk) & 1u ? s0[0] * p.scale_log2 : -INFINITY;
    const float x1 = (valid >> (tk + 1)) & 1u ? s0[1] * p.scale_log2 : -INFINITY;
    const float x2 = (valid >> (tk + 8)) & 1u ? s1[0] * p.scale_log2 : -INFINITY;
    const float x3 = (valid >> (tk + 9)) & 1u ? s1[1] * p.scale_log2 : -INFINITY;
    float mt = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
    mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 2));
    const float mn = fmaxf(m, mt);
    const float ref = mn == -INFINITY ? 0.f : mn;
    const float alpha = exp2f(m - ref);
    const float p0 = exp2f(x0 - ref), p1 = exp2f(x1 - ref), p2 = exp2f(x2 - ref), p3 = exp2f(x3 - ref);
    l = l * alpha + ((p0 + p1) + (p2 + p3));
    m = mn;
    if (__any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        acc[n][0] *= alpha;
        acc[n][1] *= alpha;
        acc[n][2] *= alpha;
        acc[n][3] *= alpha;
      }
    }
    // P as A: rows 0-7 the bf16 high part, rows 8-15 the bf16 remainder
    const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
    const __nv_bfloat16 h2 = __float2bfloat16_rn(p2), h3 = __float2bfloat16_rn(p3);
    const uint32_t a0 = bf16_pair(__bfloat162float(h0), __bfloat162float(h1));
    const uint32_t a1 = bf16_pair(p0 - __bfloat162float(h0), p1 - __bfloat162float(h1));
    const uint32_t a2 = bf16_pair(__bfloat162float(h2), __bfloat162float(h3));
    const uint32_t a3 = bf16_pair(p2 - __bfloat162float(h2), p3 - __bfloat162float(h3));
    {
      const int mi = lane >> 3, tok = (mi & 1) * 8 + (lane & 7);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(vb + sw_off(tok, 2 * jj + (mi >> 1)), v0, v1, v2, v3);
        mma_bf16(acc[2 * jj], a0, a1, a2, a3, v0, v1);
        mma_bf16(acc[2 * jj + 1], a0, a1, a2, a3, v2, v3);
      }
    }
    __syncwarp();
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  pdl_launch_dependents();

  // warp partial of head g: (m, l, o[128]), o = high rows + remainder rows
  l += __shfl_xor_sync(0xFFFFFFFFu, l, 1);
  l += __shfl_xor_sync(0xFFFFFFFFu, l, 2);
  __syncthreads();  // every warp is done with its ring
  float* wp = reinterpret_cast<float*>(spm);  // [warp][head][kSpPart]
  if (g < p.G) {
    float* d = wp + (warp * kMaxG + g) * kSpPart;
    if (t4 == 0) {
      d[0] = m;
      d[1] = l;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      d[4 + 8 * n + 2 * t4] = acc[n][0] + acc[n][2];
      d[5 + 8 * n + 2 * t4] = acc[n][1] + acc[n][3];
    }
  }
  __syncthreads();

  // CTA partial: thread c merges channel c of every head
  float* gp = p.part + ((size_t)seg * p.n_split + split) * kMaxG * kSpPart;
  for (int c = threadIdx.x; c < kD; c += kSpThreads) {
    for (int h = 0; h < p.G; ++h) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kSpWarps; ++w) M = fmaxf(M, wp[(w * kMaxG + h) * kSpPart]);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kSpWarps; ++w) {
          const float* d = wp + (w * kMaxG + h) * kSpPart;
          const float f = exp2f(d[0] - M);
          L += d[1] * f;
          O += d[4 + c] * f;
        }
      }
      if (c == 0) {
        gp[h * kSpPart] = M;
        gp[h * kSpPart + 1] = L;
      }
      gp[h * kSpPart + 4 + c] = O;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&p.ticket[seg], 1u) == (uint32_t)(p.n_split - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // the last CTA of the segment merges the n_split partials: every (split,
  // head) frame is read once into shared memory and turned into its factor
  // 2^(m - M); then thread c sums channel c of every head, all loads
  // independent of one another
  __shared__ float s_f[kSpMaxSplit][kMaxG];
  __shared__ float s_l[kSpMaxSplit][kMaxG];
  __shared__ float s_L[kMaxG];
  const float* sp = p.part + (size_t)seg * p.n_split * kMaxG * kSpPart;
  for (int i = threadIdx.x; i < p.n_split * p.G; i += kSpThreads) {
    const int s = i / p.G, h = i % p.G;
    s_f[s][h] = __ldcg(sp + (s * kMaxG + h) * kSpPart);
    s_l[s][h] = __ldcg(sp + (s * kMaxG + h) * kSpPart + 1);
  }
  __syncthreads();
  if (threadIdx.x < p.G) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, s_f[s][h]);
    float L = 0.f;
    for (int s = 0; s < p.n_split; ++s) {
      const float f = s_f[s][h] == -INFINITY ? 0.f : exp2f(s_f[s][h] - M);
      s_f[s][h] = f;
      L += s_l[s][h] * f;
    }
    s_L[h] = L;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < kD; c += kSpThreads)
    for (int h = 0; h < p.G; ++h) {
      float O = 0.f;
#pragma unroll 8
      for (int s = 0; s < p.n_split; ++s) O += __ldcg(sp + (s * kMaxG + h) * kSpPart + 4 + c) * s_f[s][h];
      p.out[((size_t)b * p.H + kvh * p.G + h) * kD + c] = O / s_L[h];
    }
  if (threadIdx.x == 0) p.ticket[seg] = 0u;
}

int sparse_splits(int n_seg, int entries, int num_sms) {
  const int nrun = (entries + kSpRun - 1) / kSpRun;
  int s = (JFA_SP_CTAS_PER_SM * num_sms) / (n_seg > 0 ? n_seg : 1);
  const int by_work = (nrun + kSpWarps - 1) / kSpWarps;  // at least one run per warp
  if (s > by_work) s = by_work;
  if (s > kSpMaxSplit) s = kSpMaxSplit;
  if ((long long)n_seg * s > (n_seg > kSpSlots ? n_seg : kSpSlots)) s = kSpSlots / n_seg;
  return s < 1 ? 1 : s;
}

int launch_sparse_attend(const jfa_geom& g, const uint16_t* q, float scale, const int32_t* idx, int k,
                         const uint16_t* k_exact, const uint16_t* v_exact, bool on_host, uint8_t* ws,
                         const jfa_workspace_layout& L, float* out, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(sparse_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem) !=
        cudaSuccess)
      return JFA_ERR_CUDA;
    attr_set = true;
  }
  const int n_seg = g.batch * g.num_kv_heads;
  SparseParams p;
  p.q = q;
  p.idx = idx;
  p.kx = k_exact;
  p.vx = v_exact;
  p.out = out;
  p.part = reinterpret_cast<float*>(ws + L.off_sparse);
  p.ticket = reinterpret_cast<uint32_t*>(ws + L.off_ticket);
  p.flag = reinterpret_cast<uint32_t*>(ws + L.off_flag);
  p.k = k;
  p.capacity = g.capacity;
  p.H = g.num_heads;
  p.Hkv = g.num_kv_heads;
  p.G = g.num_heads / g.num_kv_heads;
  p.nq = split_point(g.n_ctx);
  p.n_ctx = g.n_ctx;
  p.on_host = on_host ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_split = sparse_splits(n_seg, k + (g.n_ctx - p.nq), num_sms_current());
  return launch_pdl(sparse_attend_kernel, dim3(n_seg * p.n_split), dim3(kSpThreads), (size_t)kSpSmem, st,
                    p) == cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

}  // namespace jfa

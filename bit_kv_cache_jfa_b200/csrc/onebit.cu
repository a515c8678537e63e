// onebit.cu — a 1-bit KV cache and dense attention over it (TailorKV review:
// the layers whose attention is spread over many tokens keep the whole cache
// at 1 bit per number and attend over all of it, an FP16 x INT1 product;
// no tokens are fetched back).
//
// Quantization: the group rule of jfa_pack_kv at b = 1 (keys per channel over
// 64-token groups, values per token over 32-channel groups, fp16 zero = the
// rounded-down minimum, fp16 scale = the rounded-up range, code = the nearer
// end, ties to 0).  A record per (sequence, KV head, 64-token group):
//   [0, 1024)     key bit-planes: u64 per channel, bit t = token t;
//   [1024, 1536)  key scale fp16[128], then key zero fp16[128];
//   [1536, 2560)  value bits: u32[64 tokens][4], word j bit i = channel 32 j + i;
//   [2560, 3584)  value scale fp16[64][4], then value zero fp16[64][4].
//
// onebit_attend_kernel: the CTAs of a segment split its groups; each warp
// streams its groups (16-byte cp.async, 2-stage ring) and keeps an online
// softmax partial per query head: the logit of token t for head h is
//   scale * (sum_c q_hc z_c + sum_c q_hc s_c bit_tc),
// the value side acc[h][c] += sum_t p_th (z_tj + s_tj bit_tc); both bit
// products run on mma.sync with the bits as exact fp16 0/1 operands.  The
// exact tail [N_q, n_ctx) is attended by the last split's CTA from the bf16
// copy; the CTAs' partials merge as in the sparse attention (workspace
// partials, a ticket per segment).
#include "jfa_fp4.cuh"
#include "jfa_quant.cuh"

namespace jfa {

constexpr int kB1Rec = kOneBitRecBytes;
constexpr int kB1Warps = 4;
constexpr int kB1Threads = 32 * kB1Warps;
constexpr int kB1Part = 132;  // floats per (partial, head): m, l, pad, pad, acc[128]

// ---------------------------------------------------------------------------
// pack: one CTA (256 threads) per (64-token group, segment)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) onebit_pack_kernel(const uint16_t* __restrict__ k_src,
                                                          const uint16_t* __restrict__ v_src,
                                                          uint8_t* __restrict__ pool, int capacity,
                                                          int g_from, uint32_t* flag) {
  __shared__ uint16_t xk[kKG][kD + 2];
  __shared__ uint16_t xv[kKG][kD + 2];
  __shared__ __align__(16) uint8_t rec[kB1Rec];
  const int seg = blockIdx.y, gi = g_from + blockIdx.x, tid = threadIdx.x;
  const size_t row0 = ((size_t)seg * capacity + (size_t)gi * kKG) * kD;
  for (int i = tid; i < kKG * kD / 2; i += 256) {
    const int t = i / (kD / 2), c2 = (i % (kD / 2)) * 2;
    const uint32_t wk = reinterpret_cast<const uint32_t*>(k_src + row0 + (size_t)t * kD)[c2 / 2];
    const uint32_t wv = reinterpret_cast<const uint32_t*>(v_src + row0 + (size_t)t * kD)[c2 / 2];
    xk[t][c2] = (uint16_t)(wk & 0xFFFFu);
    xk[t][c2 + 1] = (uint16_t)(wk >> 16);
    xv[t][c2] = (uint16_t)(wv & 0xFFFFu);
    xv[t][c2 + 1] = (uint16_t)(wv >> 16);
  }
  __syncthreads();
  bool bad = false;
  if (tid < kD) {
    // keys: channel c over the group's 64 tokens
    const int c = tid;
    float mn = bf(xk[0][c]), mx = mn;
    for (int t = 1; t < kKG; ++t) {
      mn = fminf(mn, bf(xk[t][c]));
      mx = fmaxf(mx, bf(xk[t][c]));
    }
    uint16_t zb, sb;
    double z, s;
    quant_params((double)mn, (double)mx, 1, zb, sb, z, s);
    bad |= !finite_h(zb) || !finite_h(sb);
    unsigned long long w = 0ull;
    for (int t = 0; t < kKG; ++t)
      w |= (unsigned long long)quant_code((double)bf(xk[t][c]), z, s, 1) << t;
    reinterpret_cast<unsigned long long*>(rec)[c] = w;
    reinterpret_cast<uint16_t*>(rec + 1024)[c] = sb;
    reinterpret_cast<uint16_t*>(rec + 1280)[c] = zb;
  } else {
    // values: token t, channel groups j and j + 1
    const int u = tid - kD, t = u >> 1;
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int j = 2 * (u & 1) + jj;
      float mn = bf(xv[t][kVG * j]), mx = mn;
      for (int i = 1; i < kVG; ++i) {
        mn = fminf(mn, bf(xv[t][kVG * j + i]));
        mx = fmaxf(mx, bf(xv[t][kVG * j + i]));
      }
      uint16_t zb, sb;
      double z, s;
      quant_params((double)mn, (double)mx, 1, zb, sb, z, s);
      bad |= !finite_h(zb) || !finite_h(sb);
      uint32_t w = 0u;
      for (int i = 0; i < kVG; ++i) w |= quant_code((double)bf(xv[t][kVG * j + i]), z, s, 1) << i;
      reinterpret_cast<uint32_t*>(rec + 1536)[t * 4 + j] = w;
      reinterpret_cast<uint16_t*>(rec + 2560)[t * 4 + j] = sb;
      reinterpret_cast<uint16_t*>(rec + 3072)[t * 4 + j] = zb;
    }
  }
  if (bad) set_flag(flag, JFA_DEVERR_NONFINITE_QUANT);
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(pool + ((size_t)seg * (capacity / kKG) + gi) * kB1Rec);
  for (int i = tid; i < kB1Rec / 16; i += 256) dst[i] = reinterpret_cast<const uint4*>(rec)[i];
}

int launch_onebit_pack(const jfa_geom& g, int g_from, int g_to, const uint16_t* k_src,
                       const uint16_t* v_src, uint8_t* pool, uint32_t* flag, cudaStream_t st) {
  if (g_to <= g_from) return JFA_OK;
  const int n_seg = g.batch * g.num_kv_heads;
  onebit_pack_kernel<<<dim3(g_to - g_from, n_seg), 256, 0, st>>>(k_src, v_src, pool, g.capacity, g_from,
                                                                 flag);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// dense attention
// ---------------------------------------------------------------------------
struct OneBitParams {
  const uint8_t* pool;
  const uint16_t* q;
  const uint16_t* kx;  // exact copy: the tail rows
  const uint16_t* vx;
  float* out;
  float* part;
  uint32_t* ticket;
  int capacity, H, Hkv, G, nq, n_ctx, n_split;
  float scale_log2;
};

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

__device__ __forceinline__ void mma_f16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// fp16x2 of two code bits: 1.0 or 0.0 in each half (exact operands).
__device__ __forceinline__ uint32_t bits_h2(uint32_t lo_bit, uint32_t hi_bit) {
  return (lo_bit & 1u) * 0x3C00u | (hi_bit & 1u) * 0x3C000000u;
}
// fp16x2 (hi parts) and the fp16x2 of the remainders of two fp32 values.
__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
  __half2 a = __halves2half2(h0, h1);
  __half2 b = __floats2half2_rn(x0 - __half2float(h0), x1 - __half2float(h1));
  hi = *reinterpret_cast<uint32_t*>(&a);
  lo = *reinterpret_cast<uint32_t*>(&b);
}

// Dynamic shared memory per warp: its 2-stage record ring and w = q_hc s_c
// of the current group; after the last group the region holds the warps'
// partials (and, in the last split's CTA, the tail's, slots kB1Warps ..).
constexpr int kB1WarpBytes = 2 * kB1Rec + kMaxG * kD * 4;
constexpr int kB1Smem = kB1Warps * kB1WarpBytes;
static_assert(2 * kB1Warps * kMaxG * kB1Part * 4 <= kB1Smem, "partials fit the rings");

// Per group of 64 tokens, per warp, on mma.sync m16n8k16 (f16 in, fp32 out):
//   logits  S^T (16 x 64) = W (16 x 128) K^T (128 x 64): W rows 0-7 are the
//           fp16 high parts of w_hc = q_hc s_c per query head, rows 8-15 the
//           fp16 remainders (the two row halves add up to w at about 22
//           bits); the key bits enter as exact fp16 0/1, plus the zero-point
//           term sum_c q_hc z_c; lane (g, t4) holds head g's logits of tokens
//           8 nt + 2 t4, + 1 (nt = 0..7);
//   values  acc^T (128 x 8) += V^T (128 x 64) U (64 x 8), U = p_th s_tj in
//           fp16 high / remainder parts (two MMAs), the value bits as exact
//           fp16 0/1; the B fragments come from the lane's own softmax
//           registers; the zero-point term sum_t p_th z_tj per channel group.
__global__ void __launch_bounds__(kB1Threads) onebit_attend_kernel(const __grid_constant__ OneBitParams p) {
  extern __shared__ __align__(16) uint8_t b1sm[];
  __shared__ float zp_s[kB1Warps][kMaxG][4];
  __shared__ int s_last;
  const int seg = blockIdx.x / p.n_split, split = blockIdx.x % p.n_split;
  const int b = seg / p.Hkv, kvh = seg % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int ng = p.nq / kKG;
  const int g_lo = (int)((long long)split * ng / p.n_split);
  const int g_hi = (int)((long long)(split + 1) * ng / p.n_split);
  const int n_mine = g_hi - g_lo > warp ? (g_hi - g_lo - warp + kB1Warps - 1) / kB1Warps : 0;
  const uint8_t* recs = p.pool + (size_t)seg * (p.capacity / kKG) * kB1Rec;
  uint8_t* wbase = b1sm + warp * kB1WarpBytes;
  float (*wsm)[kD] = reinterpret_cast<float (*)[kD]>(wbase + 2 * kB1Rec);

  pdl_wait();
  // the lane's 4 channels 4 lane .. +3 of every head's query (for w and the
  // zero-point sums; the tail's exact logits use them too)
  float qv[kMaxG][4];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) {
    const uint2 w = h < p.G ? *reinterpret_cast<const uint2*>(p.q + ((size_t)b * p.H + kvh * p.G + h) * kD + 4 * lane)
                            : make_uint2(0, 0);
    qv[h][0] = __uint_as_float(w.x << 16);
    qv[h][1] = __uint_as_float(w.x & 0xFFFF0000u);
    qv[h][2] = __uint_as_float(w.y << 16);
    qv[h][3] = __uint_as_float(w.y & 0xFFFF0000u);
  }
  // running state: head g's frame and mass (lanes of quad g), acc^T columns
  // 2 t4, 2 t4 + 1 of channel rows 16 mt + g, + 8
  float m_run = -INFINITY, l_run = 0.f;
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

  auto issue = [&](int j) {
    const uint8_t* src = recs + (size_t)(g_lo + warp + kB1Warps * j) * kB1Rec;
    uint8_t* dst = wbase + (j & 1) * kB1Rec;
#pragma unroll
    for (int i = 0; i < kB1Rec / 16 / 32; ++i) {
      const int off = (i * 32 + lane) * 16;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst + off)), "l"(src + off)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (n_mine > 0) issue(0);
  for (int j = 0; j < n_mine; ++j) {
    if (j + 1 < n_mine) {
      issue(j + 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    const uint8_t* R = wbase + (j & 1) * kB1Rec;
    const unsigned long long* kb = reinterpret_cast<const unsigned long long*>(R);
    const uint16_t* ks_ = reinterpret_cast<const uint16_t*>(R + 1024);
    const uint16_t* kz = reinterpret_cast<const uint16_t*>(R + 1280);
    const uint32_t* vb = reinterpret_cast<const uint32_t*>(R + 1536);
    const uint16_t* vs = reinterpret_cast<const uint16_t*>(R + 2560);
    const uint16_t* vz = reinterpret_cast<const uint16_t*>(R + 3072);

    // w = q s of the lane's channels, and the zero-point sums per head
    float cz_g = 0.f;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = 4 * lane + i;
        wsm[h][c] = qv[h][i] * h2f(ks_[c]);
        z = fmaf(qv[h][i], h2f(kz[c]), z);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
      if (h == g) cz_g = z;
    }
    __syncwarp();

    // ---- logits of head g: 8 n-tiles of 8 tokens, 8 k-steps of 16 channels
    float d[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.f;
#pragma unroll
    for (int kst = 0; kst < 8; ++kst) {
      const int c0 = 16 * kst + 2 * t4;
      uint32_t a0, a1, a2, a3;
      split_h2(wsm[g][c0], wsm[g][c0 + 1], a0, a1);
      split_h2(wsm[g][c0 + 8], wsm[g][c0 + 9], a2, a3);
      const unsigned long long p0 = kb[c0], p1 = kb[c0 + 1], p8 = kb[c0 + 8], p9 = kb[c0 + 9];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int tk = 8 * nt + g;  // this lane's B column (token)
        const uint32_t b0 = bits_h2((uint32_t)(p0 >> tk), (uint32_t)(p1 >> tk));
        const uint32_t b1 = bits_h2((uint32_t)(p8 >> tk), (uint32_t)(p9 >> tk));
        mma_f16_16816(d[nt], a0, a1, a2, a3, b0, b1);
      }
    }
    // logits (log2 units) of head g, tokens 8 nt + 2 t4 + e
    float x[8][2];
    float mb = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        x[nt][e] = g < p.G ? (d[nt][e] + d[nt][2 + e] + cz_g) * p.scale_log2 : -INFINITY;
        mb = fmaxf(mb, x[nt][e]);
      }
    mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
    mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 2));
    const float mn = fmaxf(m_run, mb);
    const float ref = mn == -INFINITY ? 0.f : mn;
    const float alpha = exp2f(m_run - ref);
    float ps = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        x[nt][e] = exp2f(x[nt][e] - ref);  // now p
        ps += x[nt][e];
      }
    l_run = l_run * alpha + ps;
    m_run = mn;
    // acc^T columns are heads 2 t4 and 2 t4 + 1: their factors from quads 2 t4, 2 t4 + 1
    const float al0 = __shfl_sync(0xFFFFFFFFu, alpha, 8 * t4), al1 = __shfl_sync(0xFFFFFFFFu, alpha, 8 * t4 + 4);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      acc[mt][0] *= al0;
      acc[mt][1] *= al1;
      acc[mt][2] *= al0;
      acc[mt][3] *= al1;
    }

    // ---- values: per channel group jj (m-tiles 2 jj, 2 jj + 1) and k-step
    // kv of 16 tokens: B = U_jj of tokens 16 kv + 2 t4 (+1) and + 8 (+9)
    float zp[4] = {0.f, 0.f, 0.f, 0.f};  // head g: sum_t p z_tj over the lane's tokens
#pragma unroll
    for (int kv = 0; kv < 4; ++kv) {
      const int ta = 16 * kv + 2 * t4, tb = ta + 8;
      const float pa0 = x[2 * kv][0], pa1 = x[2 * kv][1], pb0 = x[2 * kv + 1][0], pb1 = x[2 * kv + 1][1];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t bh0, bl0, bh1, bl1;
        split_h2(pa0 * h2f(vs[ta * 4 + jj]), pa1 * h2f(vs[(ta + 1) * 4 + jj]), bh0, bl0);
        split_h2(pb0 * h2f(vs[tb * 4 + jj]), pb1 * h2f(vs[(tb + 1) * 4 + jj]), bh1, bl1);
        zp[jj] += pa0 * h2f(vz[ta * 4 + jj]) + pa1 * h2f(vz[(ta + 1) * 4 + jj]) +
                  pb0 * h2f(vz[tb * 4 + jj]) + pb1 * h2f(vz[(tb + 1) * 4 + jj]);
        const uint32_t wa0 = vb[ta * 4 + jj], wa1 = vb[(ta + 1) * 4 + jj];
        const uint32_t wb0 = vb[tb * 4 + jj], wb1 = vb[(tb + 1) * 4 + jj];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int mt = 2 * jj + half;
          const int sh = 16 * half + g;  // bit of channel 16 mt + g in word jj
          const uint32_t a0 = bits_h2(wa0 >> sh, wa1 >> sh);
          const uint32_t a1 = bits_h2(wa0 >> (sh + 8), wa1 >> (sh + 8));
          const uint32_t a2 = bits_h2(wb0 >> sh, wb1 >> sh);
          const uint32_t a3 = bits_h2(wb0 >> (sh + 8), wb1 >> (sh + 8));
          mma_f16_16816(acc[mt], a0, a1, a2, a3, bh0, bh1);
          mma_f16_16816(acc[mt], a0, a1, a2, a3, bl0, bl1);
        }
      }
    }
    // zero-point terms: quad sums for head g, then to the columns' lanes
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      zp[jj] += __shfl_xor_sync(0xFFFFFFFFu, zp[jj], 1);
      zp[jj] += __shfl_xor_sync(0xFFFFFFFFu, zp[jj], 2);
    }
    if (t4 == 0) {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) zp_s[warp][g][jj] = zp[jj];
    }
    __syncwarp();
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const float z0 = zp_s[warp][2 * t4][mt >> 1], z1 = zp_s[warp][2 * t4 + 1][mt >> 1];
      acc[mt][0] += z0;
      acc[mt][1] += z1;
      acc[mt][2] += z0;
      acc[mt][3] += z1;
    }
    __syncwarp();
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  pdl_launch_dependents();

  // ---- warp partials: head h's frame and mass from quad h, acc^T columns
  __syncthreads();  // every warp is done with its ring
  float (*wp)[kMaxG][kB1Part] = reinterpret_cast<float (*)[kMaxG][kB1Part]>(b1sm);
  {
    float l = l_run;
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 1);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 2);
    if (t4 == 0 && g < p.G) {
      wp[warp][g][0] = m_run;
      wp[warp][g][1] = l;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 2 * t4 + e;
        if (h < p.G) {
          wp[warp][h][4 + 16 * mt + g] = acc[mt][e];
          wp[warp][h][4 + 16 * mt + g + 8] = acc[mt][2 + e];
        }
      }
  }
  // ---- the exact tail (last split's CTA): warp w takes tail tokens
  // N_q + w + 4 i, four at a time (their rows loaded together), lane = 4
  // channels; its partial goes to slot kB1Warps + w
  const bool has_tail = split == p.n_split - 1;
  if (has_tail) {
    float tm[kMaxG], tl[kMaxG], ta[kMaxG][4];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      tm[h] = -INFINITY;
      tl[h] = 0.f;
      ta[h][0] = ta[h][1] = ta[h][2] = ta[h][3] = 0.f;
    }
    const uint16_t* K = p.kx + (size_t)seg * p.capacity * kD;
    const uint16_t* V = p.vx + (size_t)seg * p.capacity * kD;
    for (int t0 = p.nq + warp; t0 < p.n_ctx; t0 += 4 * kB1Warps) {
      uint2 kw[4], vw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + kB1Warps * u;
        kw[u] = t < p.n_ctx ? *reinterpret_cast<const uint2*>(K + (size_t)t * kD + 4 * lane) : make_uint2(0, 0);
        vw[u] = t < p.n_ctx ? *reinterpret_cast<const uint2*>(V + (size_t)t * kD + 4 * lane) : make_uint2(0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + kB1Warps * u >= p.n_ctx) break;
        const float k4[4] = {__uint_as_float(kw[u].x << 16), __uint_as_float(kw[u].x & 0xFFFF0000u),
                             __uint_as_float(kw[u].y << 16), __uint_as_float(kw[u].y & 0xFFFF0000u)};
        const float v4[4] = {__uint_as_float(vw[u].x << 16), __uint_as_float(vw[u].x & 0xFFFF0000u),
                             __uint_as_float(vw[u].y << 16), __uint_as_float(vw[u].y & 0xFFFF0000u)};
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
          if (h >= p.G) continue;
          float dd = qv[h][0] * k4[0] + qv[h][1] * k4[1] + qv[h][2] * k4[2] + qv[h][3] * k4[3];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xFFFFFFFFu, dd, o);
          const float xx = dd * p.scale_log2;
          const float mn = fmaxf(tm[h], xx);
          const float a = exp2f(tm[h] - mn), pt = exp2f(xx - mn);
          tl[h] = tl[h] * a + pt;
#pragma unroll
          for (int i = 0; i < 4; ++i) ta[h][i] = fmaf(ta[h][i], a, pt * v4[i]);
          tm[h] = mn;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h >= p.G) continue;
      if (lane == 0) {
        wp[kB1Warps + warp][h][0] = tm[h];
        wp[kB1Warps + warp][h][1] = tl[h];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) wp[kB1Warps + warp][h][4 + 4 * lane + i] = ta[h][i];
    }
  }
  __syncthreads();
  const int n_parts = has_tail ? 2 * kB1Warps : kB1Warps;
  const int c = threadIdx.x;  // 128 threads: one channel each
  float* gp = p.part + ((size_t)seg * p.n_split + split) * kMaxG * kB1Part;
  for (int h = 0; h < p.G; ++h) {
    float M = -INFINITY;
    for (int w = 0; w < n_parts; ++w) M = fmaxf(M, wp[w][h][0]);  // idle warps hold -inf
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < n_parts; ++w) {
        const float f = exp2f(wp[w][h][0] - M);
        L += wp[w][h][1] * f;
        O += wp[w][h][4 + c] * f;
      }
    }
    if (c == 0) {
      gp[h * kB1Part] = M;
      gp[h * kB1Part + 1] = L;
    }
    gp[h * kB1Part + 4 + c] = O;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&p.ticket[seg], 1u) == (uint32_t)(p.n_split - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  __shared__ float s_f[kSpMaxSplit][kMaxG];
  __shared__ float s_l[kSpMaxSplit][kMaxG];
  __shared__ float s_L[kMaxG];
  const float* sp = p.part + (size_t)seg * p.n_split * kMaxG * kB1Part;
  for (int i = threadIdx.x; i < p.n_split * p.G; i += kB1Threads) {
    const int s = i / p.G, h = i % p.G;
    s_f[s][h] = __ldcg(sp + (s * kMaxG + h) * kB1Part);
    s_l[s][h] = __ldcg(sp + (s * kMaxG + h) * kB1Part + 1);
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
  for (int h = 0; h < p.G; ++h) {
    float O = 0.f;
#pragma unroll 8
    for (int s = 0; s < p.n_split; ++s) O += __ldcg(sp + (s * kMaxG + h) * kB1Part + 4 + c) * s_f[s][h];
    p.out[((size_t)b * p.H + kvh * p.G + h) * kD + c] = O / s_L[h];
  }
  if (threadIdx.x == 0) p.ticket[seg] = 0u;
}

int sparse_splits(int n_seg, int entries, int num_sms);

int launch_onebit_attend(const jfa_geom& g, const uint8_t* pool, const uint16_t* q, float scale,
                         const uint16_t* k_exact, const uint16_t* v_exact, uint8_t* ws,
                         const jfa_workspace_layout& L, float* out, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  OneBitParams p;
  p.pool = pool;
  p.q = q;
  p.kx = k_exact;
  p.vx = v_exact;
  p.out = out;
  p.part = reinterpret_cast<float*>(ws + L.off_sparse);
  p.ticket = reinterpret_cast<uint32_t*>(ws + L.off_ticket);
  p.capacity = g.capacity;
  p.H = g.num_heads;
  p.Hkv = g.num_kv_heads;
  p.G = g.num_heads / g.num_kv_heads;
  p.nq = split_point(g.n_ctx);
  p.n_ctx = g.n_ctx;
  p.scale_log2 = scale * 1.4426950408889634f;
  // splits: up to 3 CTAs per SM over all segments, at least 4 groups per
  // CTA, within the workspace's partial slots
  const int ng = p.nq / kKG;
  int s = (3 * num_sms_current()) / (n_seg > 0 ? n_seg : 1);
  const int by_work = (ng + kB1Warps - 1) / kB1Warps;
  if (s > by_work) s = by_work;
  if (s > kSpMaxSplit) s = kSpMaxSplit;
  if ((long long)n_seg * s > (n_seg > kSpSlots ? n_seg : kSpSlots)) s = kSpSlots / n_seg;
  p.n_split = s < 1 ? 1 : s;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(onebit_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kB1Smem) !=
        cudaSuccess)
      return JFA_ERR_CUDA;
    attr_set = true;
  }
  return launch_pdl(onebit_attend_kernel, dim3(n_seg * p.n_split), dim3(kB1Threads), (size_t)kB1Smem, st, p) ==
                 cudaSuccess
             ? JFA_OK
             : JFA_ERR_CUDA;
}

}  // namespace jfa

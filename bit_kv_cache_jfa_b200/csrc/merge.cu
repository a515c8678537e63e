// merge.cu — jfa_correct_merge: exact correction of the top-k tokens and the
// log-sum-exp merge with the approximate remainder.
//
// Exact part (JetFire README, introduction: high-precision correction of the
// top-k tokens; Jet-QSparse abstract: sparse high-precision value aggregation
// with FP32 accumulation): logits scale * q.K_t from the bf16 copy for every
// top-k token and every tail token, aggregated with bf16 values in fp32.
//
// Approximate remainder: the scan accumulated every quantized token; here
// the top-k tokens' approximate terms are recomputed (codes re-derived from
// the bf16 row with the packing rule and the stored scale/zero, which gives
// the stored codes exactly) and removed:
//   (m_a, l_a, acc_a) - (m_r, l_r, acc_r)  in the m_a frame, l clamped >= 0.
// The removed mass is replaced by the exact part, so the cancellation error
// is relative to that part's weight.
//
// Two kernels: per (segment, 32-token chunk of idx + tail) exact and removal
// partials; per segment the final merge of scan slots, chunk partials and
// the normalisation.  The bf16 rows are read with plain loads, so they may
// live in HBM or in pinned host memory (zero-copy).
#include "jfa_internal.cuh"

namespace jfa {

constexpr unsigned kAll = 0xFFFFFFFFu;

struct MergeParams {
  const uint8_t* groups;
  const uint16_t* tail_k;
  const uint16_t* tail_v;
  const uint16_t* k_exact;
  const uint16_t* v_exact;
  const uint16_t* q;
  const int32_t* idx;
  const float* scan_part;
  float* chunk_part;  // [n_seg][n_chunks][2][G][132]
  float* out;
  uint32_t* flag;
  int k, tail, nq, capacity, ng_cap, hkv, G, H, n_chunks, key_bits, val_bits, rec_bytes;
  long long scan_total;
  int scan_warps, ng;
  float kappa;
};

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ float quant_dequant_bits(float x, uint16_t sb, uint16_t zb, int bits) {
  const float s = __half2float(__ushort_as_half(sb));
  const float z = __half2float(__ushort_as_half(zb));
  double c = 0.0;
  if (s != 0.f) {
    c = rint(((double)x - (double)z) / (double)s);
    const double lv = (double)((1 << bits) - 1);
    c = c < 0.0 ? 0.0 : (c > lv ? lv : c);
  }
  return fmaf(s, (float)c, z);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kAll, v, o);
  return v;
}

struct OnlineState {
  float m, l, a[4];
  __device__ void init() {
    m = -INFINITY;
    l = 0.f;
    a[0] = a[1] = a[2] = a[3] = 0.f;
  }
  __device__ void add(float u, const float* v) {
    if (u > m) {
      const float sc = exp2f(m - u);  // 0 when m = -inf
      l *= sc;
      a[0] *= sc;
      a[1] *= sc;
      a[2] *= sc;
      a[3] *= sc;
      m = u;
    }
    const float w = exp2f(u - m);
    l += w;
    a[0] = fmaf(w, v[0], a[0]);
    a[1] = fmaf(w, v[1], a[1]);
    a[2] = fmaf(w, v[2], a[2]);
    a[3] = fmaf(w, v[3], a[3]);
  }
};

// grid (n_chunks, n_seg), 4 warps; warp w handles tokens chunk*32 + w*8 + i,
// in two batches of four whose loads are all issued before any use.
template <int G>
__global__ void __launch_bounds__(128) correct_chunk_kernel(const MergeParams p) {
  __shared__ float red[4][2][G][kPartStride];
  const int seg = blockIdx.y, chunk = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = seg / p.hkv, h = seg % p.hkv;
  const int c0 = 4 * lane;
  const int jv = lane >> 3;  // channels 4*lane.. lie in value group lane/8

  float q[G][4];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const uint2 w = *reinterpret_cast<const uint2*>(p.q + ((size_t)b * p.H + h * G + j) * kD + c0);
    q[j][0] = __uint_as_float(w.x << 16);
    q[j][1] = __uint_as_float(w.x & 0xFFFF0000u);
    q[j][2] = __uint_as_float(w.y << 16);
    q[j][3] = __uint_as_float(w.y & 0xFFFF0000u);
  }
  OnlineState ex[G], rm[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    ex[j].init();
    rm[j].init();
  }
  const int ks_s0 = off_ks() + ks_scale_off(c0), ks_s1 = off_ks() + ks_scale_off(c0 + 2);
  const int ks_z0 = off_ks() + ks_zero_off(c0), ks_z1 = off_ks() + ks_zero_off(c0 + 2);

  const int e_base = chunk * kMergeChunk + warp * (kMergeChunk / 4);
  // token ids of this warp's 8 entries (lane i < 8 resolves entry i)
  int my_t = -1;
  if (lane < 8) {
    const int e = e_base + lane;
    if (e < p.k) {
      my_t = p.idx[(size_t)seg * p.k + e];
      if (my_t >= p.nq) {
        set_flag(p.flag, JFA_DEVERR_BAD_INDEX);
        my_t = -1;
      }
    } else if (e - p.k < p.tail) {
      my_t = (1 << 30) | (e - p.k);  // tail slot
    }
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    int tk[4];
    uint2 kw[4], vw[4];
    uint32_t s01[4], s23[4], z01[4], z23[4];
    uint16_t vsb[4], vzb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tk[i] = __shfl_sync(kAll, my_t, half * 4 + i);
      kw[i] = vw[i] = make_uint2(0u, 0u);
      s01[i] = s23[i] = z01[i] = z23[i] = 0u;
      vsb[i] = vzb[i] = 0;
      if (tk[i] < 0) continue;
      const uint16_t *kr, *vr;
      if (tk[i] & (1 << 30)) {
        const int tt = tk[i] & ~(1 << 30);
        kr = p.tail_k + ((size_t)seg * kTail + tt) * kD;
        vr = p.tail_v + ((size_t)seg * kTail + tt) * kD;
      } else {
        const int t = tk[i];
        kr = p.k_exact + ((size_t)seg * p.capacity + t) * kD;
        vr = p.v_exact + ((size_t)seg * p.capacity + t) * kD;
        const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + t / kKG) * p.rec_bytes;
        s01[i] = *reinterpret_cast<const uint32_t*>(rec + ks_s0);
        s23[i] = *reinterpret_cast<const uint32_t*>(rec + ks_s1);
        z01[i] = *reinterpret_cast<const uint32_t*>(rec + ks_z0);
        z23[i] = *reinterpret_cast<const uint32_t*>(rec + ks_z1);
        const int vb = off_vs(p.key_bits);
        vsb[i] = *reinterpret_cast<const uint16_t*>(rec + vb + vs_scale_off(t % kKG, jv));
        vzb[i] = *reinterpret_cast<const uint16_t*>(rec + vb + vs_zero_off(t % kKG, jv));
      }
      kw[i] = *reinterpret_cast<const uint2*>(kr + c0);
      vw[i] = *reinterpret_cast<const uint2*>(vr + c0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (tk[i] < 0) continue;  // warp-uniform
      const float kx[4] = {bf16f(kw[i].x & 0xFFFFu), bf16f(kw[i].x >> 16), bf16f(kw[i].y & 0xFFFFu),
                           bf16f(kw[i].y >> 16)};
      const float vx[4] = {bf16f(vw[i].x & 0xFFFFu), bf16f(vw[i].x >> 16), bf16f(vw[i].y & 0xFFFFu),
                           bf16f(vw[i].y >> 16)};
#pragma unroll
      for (int j = 0; j < G; ++j) {
        float d = q[j][0] * kx[0];
        d = fmaf(q[j][1], kx[1], d);
        d = fmaf(q[j][2], kx[2], d);
        d = fmaf(q[j][3], kx[3], d);
        d = warp_sum(d);
        ex[j].add(d * p.kappa, vx);
      }
      if (!(tk[i] & (1 << 30))) {
        const uint16_t ksb[4] = {(uint16_t)(s01[i] & 0xFFFFu), (uint16_t)(s01[i] >> 16),
                                 (uint16_t)(s23[i] & 0xFFFFu), (uint16_t)(s23[i] >> 16)};
        const uint16_t kzb[4] = {(uint16_t)(z01[i] & 0xFFFFu), (uint16_t)(z01[i] >> 16),
                                 (uint16_t)(z23[i] & 0xFFFFu), (uint16_t)(z23[i] >> 16)};
        float kh[4], vh[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          kh[c] = quant_dequant_bits(kx[c], ksb[c], kzb[c], p.key_bits);
          vh[c] = quant_dequant_bits(vx[c], vsb[i], vzb[i], p.val_bits);
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
          float d = q[j][0] * kh[0];
          d = fmaf(q[j][1], kh[1], d);
          d = fmaf(q[j][2], kh[2], d);
          d = fmaf(q[j][3], kh[3], d);
          d = warp_sum(d);
          rm[j].add(d * p.kappa, vh);
        }
      }
    }
  }
  // combine the 4 warps
#pragma unroll
  for (int j = 0; j < G; ++j) {
    float* re = red[warp][0][j];
    float* rr = red[warp][1][j];
    if (lane == 0) {
      re[0] = ex[j].m;
      re[1] = ex[j].l;
      rr[0] = rm[j].m;
      rr[1] = rm[j].l;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      re[4 + c0 + c] = ex[j].a[c];
      rr[4 + c0 + c] = rm[j].a[c];
    }
  }
  __syncthreads();
  const int c = threadIdx.x;  // channel
#pragma unroll
  for (int part = 0; part < 2; ++part) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float m = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (red[w][part][j][1] > 0.f) m = fmaxf(m, red[w][part][j][0]);
      float l = 0.f, a = 0.f;
      if (m > -INFINITY) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float lb = red[w][part][j][1];
          if (lb > 0.f) {
            const float sc = exp2f(red[w][part][j][0] - m);
            l = fmaf(lb, sc, l);
            a = fmaf(red[w][part][j][4 + c], sc, a);
          }
        }
      }
      float* dst = p.chunk_part +
                   ((((size_t)seg * p.n_chunks + chunk) * 2 + part) * G + j) * kPartStride;
      if (c == 0) {
        dst[0] = m;
        dst[1] = l;
      }
      dst[4 + c] = a;
    }
  }
}

// Merge all partials of (segment, head): max first, then independent sums,
// so every partial's loads are in flight together.
template <int G>
__global__ void __launch_bounds__(32 * G) merge_final_kernel(const MergeParams p) {
  const int seg = blockIdx.x;
  const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = 4 * lane;
  long long w0 = 0, w1 = -1;
  if (p.ng > 0) {
    const long long T = p.scan_total, W = p.scan_warps;
    const long long x0 = (long long)seg * p.ng, x1 = x0 + p.ng - 1;
    w0 = scan_warp_of(x0, W, T);
    w1 = scan_warp_of(x1, W, T);
  }
  const int ns = (int)(w1 - w0 + 1);
  auto srow = [&](int i) { return p.scan_part + ((size_t)(w0 + i + seg) * G + j) * kPartStride; };
  auto crow = [&](int ch, int part) {
    return p.chunk_part + ((((size_t)seg * p.n_chunks + ch) * 2 + part) * G + j) * kPartStride;
  };
  // pass 1: maxima
  float ma = -INFINITY, me = -INFINITY, mr = -INFINITY;
  for (int i = 0; i < ns; ++i) {
    const float2 ml = *reinterpret_cast<const float2*>(srow(i));
    if (ml.y > 0.f) ma = fmaxf(ma, ml.x);
  }
  for (int ch = 0; ch < p.n_chunks; ++ch) {
    const float2 e = *reinterpret_cast<const float2*>(crow(ch, 0));
    const float2 r = *reinterpret_cast<const float2*>(crow(ch, 1));
    if (e.y > 0.f) me = fmaxf(me, e.x);
    if (r.y > 0.f) mr = fmaxf(mr, r.x);
  }
  // pass 2: sums in the frames of those maxima
  float la = 0.f, le = 0.f, lr = 0.f;
  float aa[4] = {0.f, 0.f, 0.f, 0.f}, ae[4] = {0.f, 0.f, 0.f, 0.f}, ar[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int i = 0; i < ns; ++i) {
    const float* row = srow(i);
    const float2 ml = *reinterpret_cast<const float2*>(row);
    const float4 v = *reinterpret_cast<const float4*>(row + 4 + c0);
    const float sc = ml.y > 0.f ? exp2f(ml.x - ma) : 0.f;
    la = fmaf(ml.y, sc, la);
    aa[0] = fmaf(v.x, sc, aa[0]);
    aa[1] = fmaf(v.y, sc, aa[1]);
    aa[2] = fmaf(v.z, sc, aa[2]);
    aa[3] = fmaf(v.w, sc, aa[3]);
  }
#pragma unroll 4
  for (int ch = 0; ch < p.n_chunks; ++ch) {
    const float* re = crow(ch, 0);
    const float* rr = crow(ch, 1);
    const float2 e = *reinterpret_cast<const float2*>(re);
    const float2 r = *reinterpret_cast<const float2*>(rr);
    const float4 ev = *reinterpret_cast<const float4*>(re + 4 + c0);
    const float4 rv = *reinterpret_cast<const float4*>(rr + 4 + c0);
    const float se = e.y > 0.f ? exp2f(e.x - me) : 0.f;
    const float sr = r.y > 0.f ? exp2f(r.x - mr) : 0.f;
    le = fmaf(e.y, se, le);
    lr = fmaf(r.y, sr, lr);
    ae[0] = fmaf(ev.x, se, ae[0]);
    ae[1] = fmaf(ev.y, se, ae[1]);
    ae[2] = fmaf(ev.z, se, ae[2]);
    ae[3] = fmaf(ev.w, se, ae[3]);
    ar[0] = fmaf(rv.x, sr, ar[0]);
    ar[1] = fmaf(rv.y, sr, ar[1]);
    ar[2] = fmaf(rv.z, sr, ar[2]);
    ar[3] = fmaf(rv.w, sr, ar[3]);
  }
  // remainder = approximate total minus the removed top-k terms (m_a frame)
  float lrest = la, arest[4] = {aa[0], aa[1], aa[2], aa[3]};
  if (la > 0.f && lr > 0.f) {
    const float f = exp2f(mr - ma);
    lrest = la - lr * f;
#pragma unroll
    for (int i = 0; i < 4; ++i) arest[i] = aa[i] - ar[i] * f;
    if (lrest < 0.f) lrest = 0.f;
  }
  float m = me, wl = 1.f, wa = 0.f;
  if (la > 0.f) {
    m = fmaxf(me, ma);
    wl = exp2f(me - m);
    wa = exp2f(ma - m);
  }
  const float inv = 1.f / (le * wl + lrest * wa);
  float4 o;
  o.x = (ae[0] * wl + arest[0] * wa) * inv;
  o.y = (ae[1] * wl + arest[1] * wa) * inv;
  o.z = (ae[2] * wl + arest[2] * wa) * inv;
  o.w = (ae[3] * wl + arest[3] * wa) * inv;
  const int b = seg / p.hkv, h = seg % p.hkv;
  *reinterpret_cast<float4*>(p.out + ((size_t)b * p.H + h * G + j) * kD + c0) = o;
}

template <int G>
static void launch_cm_t(const MergeParams& p, int n_seg, cudaStream_t st) {
  correct_chunk_kernel<G><<<dim3(p.n_chunks, n_seg), 128, 0, st>>>(p);
  merge_final_kernel<G><<<n_seg, 32 * G, 0, st>>>(p);
}

int launch_correct_merge(const jfa_geom& g, const jfa_cache& c, const uint16_t* q, float scale,
                         const int32_t* idx, int k, const uint16_t* k_exact,
                         const uint16_t* v_exact, int exact_on_host, uint8_t* ws,
                         const jfa_workspace_layout& L, float* out, cudaStream_t st) {
  (void)exact_on_host;  // same loads either way; the rows are device-addressable
  const int n_seg = g.batch * g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  MergeParams p;
  p.groups = static_cast<const uint8_t*>(c.groups);
  p.tail_k = c.tail_k;
  p.tail_v = c.tail_v;
  p.k_exact = k_exact;
  p.v_exact = v_exact;
  p.q = q;
  p.idx = idx;
  p.scan_part = reinterpret_cast<const float*>(ws + L.off_partials);
  p.chunk_part = reinterpret_cast<float*>(ws + L.off_merge);
  p.out = out;
  p.flag = reinterpret_cast<uint32_t*>(ws + L.off_flag);
  p.k = k;
  p.tail = g.n_ctx - nq;
  p.nq = nq;
  p.capacity = g.capacity;
  p.ng_cap = g.capacity / kKG;
  p.hkv = g.num_kv_heads;
  p.G = g.num_heads / g.num_kv_heads;
  p.H = g.num_heads;
  p.n_chunks = (k + p.tail + kMergeChunk - 1) / kMergeChunk;
  p.key_bits = g.key_bits;
  p.val_bits = g.val_bits;
  p.rec_bytes = record_bytes(g.key_bits, g.val_bits);
  ScanPlan plan = scan_plan(g, num_sms_current());
  p.scan_total = plan.total_groups;
  p.scan_warps = plan.n_warps;
  p.ng = plan.ng;
  p.kappa = scale * 1.4426950408889634f;
  switch (p.G) {
    case 1: launch_cm_t<1>(p, n_seg, st); break;
    case 2: launch_cm_t<2>(p, n_seg, st); break;
    case 3: launch_cm_t<3>(p, n_seg, st); break;
    case 4: launch_cm_t<4>(p, n_seg, st); break;
    case 5: launch_cm_t<5>(p, n_seg, st); break;
    case 6: launch_cm_t<6>(p, n_seg, st); break;
    case 7: launch_cm_t<7>(p, n_seg, st); break;
    default: launch_cm_t<8>(p, n_seg, st); break;
  }
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

}  // namespace jfa

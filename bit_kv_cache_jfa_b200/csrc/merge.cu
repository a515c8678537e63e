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

__device__ __forceinline__ float quant_dequant(float x, const uint8_t* rec, int soff, int zoff,
                                               int bits) {
  const float s = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(rec + soff)));
  const float z = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(rec + zoff)));
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

// merge partial (mb, lb, ab[4]) into (m, l, a[4])
__device__ __forceinline__ void merge_into(float& m, float& l, float* a, float mb, float lb,
                                           const float* ab) {
  if (mb == -INFINITY || lb == 0.f) return;
  if (m == -INFINITY || l == 0.f) {
    m = mb;
    l = lb;
    a[0] = ab[0];
    a[1] = ab[1];
    a[2] = ab[2];
    a[3] = ab[3];
    return;
  }
  const float mn = fmaxf(m, mb);
  const float sa = exp2f(m - mn), sb = exp2f(mb - mn);
  l = l * sa + lb * sb;
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = a[i] * sa + ab[i] * sb;
  m = mn;
}

// grid (n_chunks, n_seg), 4 warps; warp w handles tokens chunk*32 + w*8 + i
__global__ void __launch_bounds__(128) correct_chunk_kernel(const MergeParams p) {
  __shared__ float red[4][2][kMaxG][kPartStride];
  const int seg = blockIdx.y, chunk = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = seg / p.hkv, h = seg % p.hkv;
  const int c0 = 4 * lane;
  const int G = p.G;

  float q[kMaxG][4];
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) {
    if (j < G) {
      const uint2 w = *reinterpret_cast<const uint2*>(p.q + ((size_t)b * p.H + h * G + j) * kD + c0);
      q[j][0] = __uint_as_float(w.x << 16);
      q[j][1] = __uint_as_float(w.x & 0xFFFF0000u);
      q[j][2] = __uint_as_float(w.y << 16);
      q[j][3] = __uint_as_float(w.y & 0xFFFF0000u);
    } else {
      q[j][0] = q[j][1] = q[j][2] = q[j][3] = 0.f;
    }
  }
  OnlineState ex[kMaxG], rm[kMaxG];
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) {
    ex[j].init();
    rm[j].init();
  }

  for (int i = 0; i < kMergeChunk / 4; ++i) {
    const int e = chunk * kMergeChunk + warp * (kMergeChunk / 4) + i;
    int t = -1;
    bool quant = false;
    const uint16_t *kr = nullptr, *vr = nullptr;
    if (e < p.k) {
      t = p.idx[(size_t)seg * p.k + e];
      if (t >= p.nq) {
        if (lane == 0) set_flag(p.flag, JFA_DEVERR_BAD_INDEX);
        t = -1;
      }
      if (t >= 0) {
        quant = true;
        kr = p.k_exact + ((size_t)seg * p.capacity + t) * kD;
        vr = p.v_exact + ((size_t)seg * p.capacity + t) * kD;
      }
    } else if (e - p.k < p.tail) {
      const int tt = e - p.k;
      t = p.nq + tt;
      kr = p.tail_k + ((size_t)seg * kTail + tt) * kD;
      vr = p.tail_v + ((size_t)seg * kTail + tt) * kD;
    }
    if (kr == nullptr) continue;  // warp-uniform
    const uint2 kw = *reinterpret_cast<const uint2*>(kr + c0);
    const uint2 vw = *reinterpret_cast<const uint2*>(vr + c0);
    float kx[4] = {bf16f(kw.x & 0xFFFFu), bf16f(kw.x >> 16), bf16f(kw.y & 0xFFFFu), bf16f(kw.y >> 16)};
    float vx[4] = {bf16f(vw.x & 0xFFFFu), bf16f(vw.x >> 16), bf16f(vw.y & 0xFFFFu), bf16f(vw.y >> 16)};
#pragma unroll
    for (int j = 0; j < kMaxG; ++j) {
      if (j < G) {
        float d = q[j][0] * kx[0];
        d = fmaf(q[j][1], kx[1], d);
        d = fmaf(q[j][2], kx[2], d);
        d = fmaf(q[j][3], kx[3], d);
        d = warp_sum(d);
        ex[j].add(d * p.kappa, vx);
      }
    }
    if (quant) {
      const int g = t / kKG, tl = t % kKG;
      const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + g) * p.rec_bytes;
      float kh[4], vh[4];
      const int jv = lane >> 3;  // channels 4*lane.. lie in value group lane/8
      const int vso = off_vs(p.key_bits) + vs_scale_off(tl, jv);
      const int vzo = off_vs(p.key_bits) + vs_zero_off(tl, jv);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        kh[c] = quant_dequant(kx[c], rec, off_ks() + ks_scale_off(c0 + c),
                              off_ks() + ks_zero_off(c0 + c), p.key_bits);
        vh[c] = quant_dequant(vx[c], rec, vso, vzo, p.val_bits);
      }
#pragma unroll
      for (int j = 0; j < kMaxG; ++j) {
        if (j < G) {
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
  for (int j = 0; j < kMaxG; ++j) {
    if (j < G) {
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
  }
  __syncthreads();
  // thread tid: channel tid; loop over (part, head)
  const int c = threadIdx.x;
  for (int part = 0; part < 2; ++part) {
    for (int j = 0; j < G; ++j) {
      float m = -INFINITY, l = 0.f, a = 0.f;
      for (int w = 0; w < 4; ++w) {
        const float mb = red[w][part][j][0], lb = red[w][part][j][1];
        if (mb == -INFINITY || lb == 0.f) continue;
        const float ab = red[w][part][j][4 + c];
        if (m == -INFINITY) {
          m = mb;
          l = lb;
          a = ab;
        } else {
          const float mn = fmaxf(m, mb);
          const float sa = exp2f(m - mn), sb = exp2f(mb - mn);
          l = l * sa + lb * sb;
          a = a * sa + ab * sb;
          m = mn;
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

// grid n_seg, one warp per query head of the segment
__global__ void __launch_bounds__(256) merge_final_kernel(const MergeParams p) {
  const int seg = blockIdx.x;
  const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (j >= p.G) return;
  const int c0 = 4 * lane;
  // approximate total over the scan slots of this segment
  float ma = -INFINITY, la = 0.f, aa[4] = {0.f, 0.f, 0.f, 0.f};
  if (p.ng > 0) {
    const long long T = p.scan_total, W = p.scan_warps;
    const long long x0 = (long long)seg * p.ng, x1 = x0 + p.ng - 1;
    const long long w0 = scan_warp_of(x0, W, T), w1 = scan_warp_of(x1, W, T);
    for (long long w = w0; w <= w1; ++w) {
      const float* row = p.scan_part + ((size_t)(w + seg) * p.G + j) * kPartStride;
      const float4 av = *reinterpret_cast<const float4*>(row + 4 + c0);
      const float ab[4] = {av.x, av.y, av.z, av.w};
      merge_into(ma, la, aa, row[0], row[1], ab);
    }
  }
  // exact and removal totals over the chunks
  float me = -INFINITY, le = 0.f, ae[4] = {0.f, 0.f, 0.f, 0.f};
  float mr = -INFINITY, lr = 0.f, ar[4] = {0.f, 0.f, 0.f, 0.f};
  for (int ch = 0; ch < p.n_chunks; ++ch) {
    const float* pe = p.chunk_part + ((((size_t)seg * p.n_chunks + ch) * 2 + 0) * p.G + j) * kPartStride;
    const float* pr = p.chunk_part + ((((size_t)seg * p.n_chunks + ch) * 2 + 1) * p.G + j) * kPartStride;
    const float4 ev = *reinterpret_cast<const float4*>(pe + 4 + c0);
    const float4 rv = *reinterpret_cast<const float4*>(pr + 4 + c0);
    const float eb[4] = {ev.x, ev.y, ev.z, ev.w};
    const float rb[4] = {rv.x, rv.y, rv.z, rv.w};
    merge_into(me, le, ae, pe[0], pe[1], eb);
    merge_into(mr, lr, ar, pr[0], pr[1], rb);
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
  const float den = le * wl + lrest * wa;
  const float inv = 1.f / den;
  float4 o;
  o.x = (ae[0] * wl + arest[0] * wa) * inv;
  o.y = (ae[1] * wl + arest[1] * wa) * inv;
  o.z = (ae[2] * wl + arest[2] * wa) * inv;
  o.w = (ae[3] * wl + arest[3] * wa) * inv;
  const int b = seg / p.hkv, h = seg % p.hkv;
  *reinterpret_cast<float4*>(p.out + ((size_t)b * p.H + h * p.G + j) * kD + c0) = o;
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
  correct_chunk_kernel<<<dim3(p.n_chunks, n_seg), 128, 0, st>>>(p);
  merge_final_kernel<<<n_seg, 32 * p.G, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

}  // namespace jfa

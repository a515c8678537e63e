// merge.cu — jfa_correct_merge: exact correction of the top-k tokens and the
// log-sum-exp merge with the approximate remainder.
//
// Exact part (JetFire README, introduction: high-precision correction of the
// top-k tokens; Jet-QSparse abstract: sparse high-precision value aggregation
// with FP32 accumulation): logits scale * q.K_t from the bf16 copy for every
// top-k token and every tail token, aggregated with bf16 values in fp32.
//
// Approximate remainder: the scan accumulated every quantized token; here
// the top-k tokens' approximate terms are recomputed from their stored codes
// and scales/zeros (exactly what the scan used) and removed:
//   (m_a, l_a, acc_a) - (m_r, l_r, acc_r)  in the m_a frame, l clamped >= 0.
// The removed mass is replaced by the exact part, so the cancellation error
// is relative to that part's weight.
//
// Two kernels: per (segment, 32-token chunk of idx + tail) exact and removal
// partials; per segment the final merge of scan slots, chunk partials and
// the normalisation.  The bf16 rows are read with plain loads, so they may
// live in HBM or in pinned host memory (zero-copy).
#include "jfa_blocks.cuh"

namespace jfa {

// grid (n_chunks, n_seg), 256 threads: chunk = 32 entries of (top-k list,
// then tail); writes one (m, l, acc) partial per (exact|removal, head).
template <int G>
__global__ void __launch_bounds__(256) correct_chunk_kernel(const MergeParams p) {
  extern __shared__ __align__(16) float sm[];
  __shared__ int s_tok[kMergeChunk];
  const CorrectSmem S = correct_smem_carve(sm, G);
  const int seg = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  if (tid < kMergeChunk) {
    const int e = chunk * kMergeChunk + tid;
    int t = -1;
    if (e < p.k) {
      t = p.idx[(size_t)seg * p.k + e];
      if (t >= p.nq) {
        set_flag(p.flag, JFA_DEVERR_BAD_INDEX);
        t = -1;
      }
    } else if (e - p.k < p.tail) {
      t = (1 << 30) | (e - p.k);  // tail slot
    }
    s_tok[tid] = t;
  }
  correct_load_q<G>(p, seg, S.qs);
  __syncthreads();
  correct_batch<G>(p, seg, s_tok, S,
                   p.chunk_part + (((size_t)seg * p.n_chunks + chunk) * 2) * G * kPartStride);
}

template <int G>
constexpr int correct_smem_bytes() {
  return correct_smem_floats<G>() * 4;
}

// grid (n_seg, G), 256 threads: one (segment, head).  All partial rows of the
// head (scan slots, exact chunks, removal chunks) are staged in shared memory
// in tiles of kTileRows with every load of a tile in flight together, then
// reduced max-first per tile into a running state.
constexpr int kTileRows = 48;
template <int G>
__global__ void __launch_bounds__(256) merge_final_kernel(const MergeParams p) {
  __shared__ __align__(16) float tile[kTileRows][kPartStride];
  const int seg = blockIdx.x, j = blockIdx.y;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  long long w0 = 0, w1 = -1;
  if (p.ng > 0) {
    const long long T = p.scan_total, W = p.scan_warps;
    const long long x0 = (long long)seg * p.ng, x1 = x0 + p.ng - 1;
    w0 = scan_warp_of(x0, W, T);
    w1 = scan_warp_of(x1, W, T);
  }
  const int ns = (int)(w1 - w0 + 1);
  const int nrows = ns + 2 * p.n_chunks;  // kind of row r: 0 scan, 1 exact, 2 removal
  auto row_ptr = [&](int r) -> const float* {
    if (r < ns) return p.scan_part + ((size_t)(w0 + r + seg) * G + j) * kPartStride;
    r -= ns;
    const int ch = r >> 1, part = r & 1;
    return p.chunk_part + ((((size_t)seg * p.n_chunks + ch) * 2 + part) * G + j) * kPartStride;
  };
  auto kind_of = [&](int r) { return r < ns ? 0 : 1 + ((r - ns) & 1); };
  const int c = tid & (kD - 1);
  const bool worker = tid < kD;
  float m[3] = {-INFINITY, -INFINITY, -INFINITY}, l[3] = {0.f, 0.f, 0.f}, a[3] = {0.f, 0.f, 0.f};
  for (int r0 = 0; r0 < nrows; r0 += kTileRows) {
    const int nr = min(kTileRows, nrows - r0);
    __syncthreads();
    constexpr int kVec = kPartStride / 4;  // float4 per row
    float4 buf[(kTileRows * kVec + 255) / 256];
#pragma unroll
    for (int u = 0; u < (kTileRows * kVec + 255) / 256; ++u) {
      const int i = tid + 256 * u;
      if (i < nr * kVec)
        buf[u] = reinterpret_cast<const float4*>(row_ptr(r0 + i / kVec))[i % kVec];
    }
#pragma unroll
    for (int u = 0; u < (kTileRows * kVec + 255) / 256; ++u) {
      const int i = tid + 256 * u;
      if (i < nr * kVec) reinterpret_cast<float4*>(tile[i / kVec])[i % kVec] = buf[u];
    }
    __syncthreads();
    if (worker) {
      // kinds: 0 scan slots (rows [0, ns)), then exact / removal alternating
      float tm0 = m[0], tm1 = m[1], tm2 = m[2];
      for (int r = 0; r < nr; ++r) {
        if (tile[r][1] > 0.f) {
          const int k = kind_of(r0 + r);
          const float x = tile[r][0];
          if (k == 0) tm0 = fmaxf(tm0, x);
          else if (k == 1) tm1 = fmaxf(tm1, x);
          else tm2 = fmaxf(tm2, x);
        }
      }
      const float tmv[3] = {tm0, tm1, tm2};
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        if (tmv[k] > m[k] && m[k] > -INFINITY) {
          const float sc = exp2f(m[k] - tmv[k]);
          l[k] *= sc;
          a[k] *= sc;
        }
        m[k] = tmv[k];
      }
      for (int r = 0; r < nr; ++r) {
        const float lb = tile[r][1];
        if (lb > 0.f) {
          const int k = kind_of(r0 + r);
          const float mk = k == 0 ? m[0] : (k == 1 ? m[1] : m[2]);
          const float sc = exp2f(tile[r][0] - mk);
          const float lv = lb * sc, av = tile[r][4 + c] * sc;
          if (k == 0) {
            l[0] += lv;
            a[0] += av;
          } else if (k == 1) {
            l[1] += lv;
            a[1] += av;
          } else {
            l[2] += lv;
            a[2] += av;
          }
        }
      }
    }
  }
  if (!worker) return;
  // remainder = approximate total minus the removed top-k terms (m_a frame)
  const float ma = m[0], la = l[0], me = m[1], le = l[1], mr = m[2], lr = l[2];
  float lrest = la, arest = a[0];
  if (la > 0.f && lr > 0.f) {
    const float f = exp2f(mr - ma);
    lrest = la - lr * f;
    arest = a[0] - a[2] * f;
    if (lrest < 0.f) lrest = 0.f;
  }
  float mm = me, wl = 1.f, wa = 0.f;
  if (la > 0.f) {
    mm = fmaxf(me, ma);
    wl = exp2f(me - mm);
    wa = exp2f(ma - mm);
  }
  const float o = (a[1] * wl + arest * wa) / (le * wl + lrest * wa);
  const int b = seg / p.hkv, h = seg % p.hkv;
  p.out[((size_t)b * p.H + h * G + j) * kD + c] = o;
}

template <int G>
static void launch_cm_t(const MergeParams& p, int n_seg, cudaStream_t st) {
  constexpr int smem = correct_smem_bytes<G>();
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaFuncSetAttribute(correct_chunk_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         smem);
    configured[dev] = true;
  }
  launch_pdl(correct_chunk_kernel<G>, dim3(p.n_chunks, n_seg), dim3(256), (size_t)smem, st, p);
  launch_pdl(merge_final_kernel<G>, dim3(n_seg, G), dim3(256), 0, st, p);
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

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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kAll, v, o);
  return v;
}

// The correction kernel reads the stored codes (exactly what the scan used)
// and the stored scales/zeros straight from the packed records.
constexpr int kRow = kD + 4;  // padded fp32 row in shared memory

// a[i] for a runtime i without spilling the array to local memory
__device__ __forceinline__ uint32_t pick8(const uint32_t (&a)[8], int i) {
  const uint32_t lo = (i & 2) ? ((i & 1) ? a[3] : a[2]) : ((i & 1) ? a[1] : a[0]);
  const uint32_t hi = (i & 2) ? ((i & 1) ? a[7] : a[6]) : ((i & 1) ? a[5] : a[4]);
  return (i & 4) ? hi : lo;
}

// grid (n_chunks, n_seg), 256 threads.  Chunk = 32 entries of (top-k list,
// then tail).  Phase A: thread (token slot, 16-channel part) stages the exact
// bf16 rows and the dequantized rows of its token in shared memory (all its
// loads issued together).  Phase B: thread (token, head) computes the exact
// and approximate logits.  Phase C: one warp per head turns them into
// weights.  Phase D: thread (channel, exact|removal) accumulates the weighted
// rows.  Writes one (m, l, acc) partial per (part, head).
template <int G>
__global__ void __launch_bounds__(256) correct_chunk_kernel(const MergeParams p) {
  extern __shared__ __align__(16) float sm[];
  float* kx = sm;                      // [32][kRow] exact keys
  float* vx = kx + kMergeChunk * kRow; // [32][kRow] exact values
  float* kh = vx + kMergeChunk * kRow; // [32][kRow] dequantized keys
  float* vh = kh + kMergeChunk * kRow; // [32][kRow] dequantized values
  float* qs = vh + kMergeChunk * kRow; // [G][kRow]
  float* ue = qs + G * kRow;           // [32][G] exact logits, then weights
  float* ur = ue + kMergeChunk * G;    // [32][G] approximate logits, then weights
  float* ml = ur + kMergeChunk * G;    // [2][G][2] (m, l)
  __shared__ int s_tok[kMergeChunk];

  const int seg = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x;
  const int b = seg / p.hkv, h = seg % p.hkv;
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
  for (int i = tid; i < G * kD; i += 256) {
    const int j = i / kD, c = i % kD;
    qs[j * kRow + c] = bf16f(p.q[((size_t)b * p.H + h * G + j) * kD + c]);
  }
  __syncthreads();

  // ---- phase A: stage the chunk's rows in shared memory.  Jobs move 16-byte
  // vectors; every load of a thread is issued before any is used.
  //   rows : 32 tokens x (K, V) x 16 pieces of 8 bf16  (4 jobs per thread)
  //   keys : 32 tokens x 4 fragment threads tig: 32 codes + their scales/zeros
  //   vals : 32 tokens x (8 or 16) fragment slots: codes of 4 or 8 m-tiles
  {
    // rows
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = tid + 256 * u;
      const int tl = j >> 5, part = j & 31, isv = part >> 4, piece = part & 15;
      const int t = s_tok[tl];
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (t >= 0) {
        const uint16_t* row;
        if (t & (1 << 30)) {
          const int tt = t & ~(1 << 30);
          row = (isv ? p.tail_v : p.tail_k) + ((size_t)seg * kTail + tt) * kD;
        } else {
          row = (isv ? p.v_exact : p.k_exact) + ((size_t)seg * p.capacity + t) * kD;
        }
        w = *reinterpret_cast<const uint4*>(row + 8 * piece);
      }
      float* dst = (isv ? vx : kx) + tl * kRow + 8 * piece;
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dst[2 * i] = __uint_as_float(ww[i] << 16);
        dst[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
      }
    }
    // keys: thread tid < 128 -> (token tid/4, fragment thread tig = tid%4)
    if (tid < 4 * kMergeChunk) {
      const int tl = tid >> 2, tg = tid & 3;
      const int t = s_tok[tl];
      float* dst = kh + tl * kRow;
      if (t >= 0 && !(t & (1 << 30))) {
        const int tt = t % kKG, nt = tt >> 3, gd = tt & 7;
        const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + t / kKG) * p.rec_bytes;
        uint4 sz[8];  // chunks 0..3: scale pairs 0..15, chunks 4..7: zero pairs
#pragma unroll
        for (int i = 0; i < 8; ++i)
          sz[i] = *reinterpret_cast<const uint4*>(rec + off_ks() + i * 64 + tg * 16);
        uint32_t cw[3];
        if (p.key_bits == 4) {
          const uint4 c4 = *reinterpret_cast<const uint4*>(rec + off_kc() + nt * 512 +
                                                           (gd * 4 + tg) * 16);
          cw[0] = c4.x;
          cw[1] = c4.y;
          cw[2] = c4.z;
          const uint32_t c3 = c4.w;
#pragma unroll
          for (int pr = 0; pr < 16; ++pr) {
            const uint32_t word = pr < 4 ? cw[0] : (pr < 8 ? cw[1] : (pr < 12 ? cw[2] : c3));
            const uint4 sq = sz[pr >> 2], zq = sz[4 + (pr >> 2)];
            const uint32_t sw = (pr & 3) == 0 ? sq.x : ((pr & 3) == 1 ? sq.y : ((pr & 3) == 2 ? sq.z : sq.w));
            const uint32_t zw = (pr & 3) == 0 ? zq.x : ((pr & 3) == 1 ? zq.y : ((pr & 3) == 2 ? zq.z : zq.w));
            const float2 s2 = unpack_h2(sw), z2 = unpack_h2(zw);
            const int c = 16 * (pr >> 1) + 2 * tg + 8 * (pr & 1);
            const int pos = 4 * (pr & 3);
            dst[c] = fmaf(s2.x, (float)((word >> pos) & 15u), z2.x);
            dst[c + 1] = fmaf(s2.y, (float)((word >> (pos + 16)) & 15u), z2.y);
          }
        } else {
          const uint8_t* cp = rec + off_kc() + (nt >> 2) * 1536 + (gd * 4 + tg) * 48 + (nt & 3) * 12;
          cw[0] = *reinterpret_cast<const uint32_t*>(cp);
          cw[1] = *reinterpret_cast<const uint32_t*>(cp + 4);
          cw[2] = *reinterpret_cast<const uint32_t*>(cp + 8);
#pragma unroll
          for (int pr = 0; pr < 16; ++pr) {
            const uint4 sq = sz[pr >> 2], zq = sz[4 + (pr >> 2)];
            const uint32_t sw = (pr & 3) == 0 ? sq.x : ((pr & 3) == 1 ? sq.y : ((pr & 3) == 2 ? sq.z : sq.w));
            const uint32_t zw = (pr & 3) == 0 ? zq.x : ((pr & 3) == 1 ? zq.y : ((pr & 3) == 2 ? zq.z : zq.w));
            const float2 s2 = unpack_h2(sw), z2 = unpack_h2(zw);
            uint32_t c0v, c1v;
            if (pr < 15) {
              const uint32_t word = cw[pr / 5];
              const int pos = 3 * (pr % 5);
              c0v = (word >> pos) & 7u;
              c1v = (word >> (pos + 16)) & 7u;
            } else {
              c0v = ((cw[0] >> 15) & 1u) | (((cw[1] >> 15) & 1u) << 1) | (((cw[2] >> 15) & 1u) << 2);
              c1v = ((cw[0] >> 31) & 1u) | (((cw[1] >> 31) & 1u) << 1) | (((cw[2] >> 31) & 1u) << 2);
            }
            const int c = 16 * (pr >> 1) + 2 * tg + 8 * (pr & 1);
            dst[c] = fmaf(s2.x, (float)c0v, z2.x);
            dst[c + 1] = fmaf(s2.y, (float)c1v, z2.y);
          }
        }
      } else {
#pragma unroll
        for (int pr = 0; pr < 16; ++pr) {
          const int c = 16 * (pr >> 1) + 2 * tg + 8 * (pr & 1);
          dst[c] = dst[c + 1] = 0.f;
        }
      }
    }
    // values: (token, slot); a slot is one fragment lane's 16 bytes of codes
    const int slots = p.val_bits == 4 ? 16 : 8;
    for (int j = tid; j < kMergeChunk * slots; j += 256) {
      const int tl = j / slots, slot = j % slots;
      const int t = s_tok[tl];
      float* dst = vh + tl * kRow;
      const int gd = slot & 7;
      if (t >= 0 && !(t & (1 << 30))) {
        const int tt = t % kKG, kk = tt >> 4, rt = tt & 15;
        const int hi8 = rt >> 3, tgt = (rt & 7) >> 1, e = rt & 1;
        const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + t / kKG) * p.rec_bytes;
        const uint8_t* vs = rec + off_vs(p.key_bits) + kk * 128 + tgt * 32;
        const uint4 sa = *reinterpret_cast<const uint4*>(vs), sb = *reinterpret_cast<const uint4*>(vs + 16);
        const uint4 za = *reinterpret_cast<const uint4*>(vs + 512);
        const uint4 zb = *reinterpret_cast<const uint4*>(vs + 528);
        const uint32_t sws[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        const uint32_t zws[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
        const int chunk = p.val_bits == 4 ? 2 * kk + (slot >> 3) : kk;
        const uint4 cv = *reinterpret_cast<const uint4*>(rec + off_vc(p.key_bits) + chunk * 512 +
                                                         (gd * 4 + tgt) * 16);
        const uint32_t cws[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
          for (int em = 0; em < 2; ++em) {
            if (p.val_bits == 4 && em == 1) continue;
            const int mt = p.val_bits == 4 ? 4 * (slot >> 3) + wd : 2 * wd + em;
            const int jg = mt >> 1;  // value group of channels 16mt..16mt+15
            const uint32_t sw = pick8(sws, 2 * jg + hi8), zw = pick8(zws, 2 * jg + hi8);
            const float sv = __half2float(__ushort_as_half((uint16_t)(e ? sw >> 16 : sw & 0xFFFFu)));
            const float zv = __half2float(__ushort_as_half((uint16_t)(e ? zw >> 16 : zw & 0xFFFFu)));
#pragma unroll
            for (int chi = 0; chi < 2; ++chi) {
              const int r = chi + 2 * hi8;
              const uint32_t code = p.val_bits == 4 ? (cws[wd] >> (4 * r + 16 * e)) & 15u
                                                    : (cws[wd] >> (2 * (4 * em + r) + 16 * e)) & 3u;
              dst[16 * mt + gd + 8 * chi] = fmaf(sv, (float)code, zv);
            }
          }
        }
      } else {
        for (int mt = 0; mt < 8; ++mt) {
          if (p.val_bits == 4 && (mt >> 2) != (slot >> 3)) continue;
          dst[16 * mt + gd] = dst[16 * mt + gd + 8] = 0.f;
        }
      }
    }
  }
  __syncthreads();

  // ---- phase B: logits (log2 units) ----
  for (int i = tid; i < kMergeChunk * G; i += 256) {
    const int tl = i / G, j = i % G;
    const int t = s_tok[tl];
    float de = -INFINITY, dr = -INFINITY;
    if (t >= 0) {
      const float4* qr = reinterpret_cast<const float4*>(qs + j * kRow);
      const float4* kr4 = reinterpret_cast<const float4*>(kx + tl * kRow);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
      for (int c = 0; c < kD / 4; ++c) {
        const float4 qv = qr[c], kv = kr4[c];
        a0 = fmaf(qv.x, kv.x, a0);
        a1 = fmaf(qv.y, kv.y, a1);
        a0 = fmaf(qv.z, kv.z, a0);
        a1 = fmaf(qv.w, kv.w, a1);
      }
      de = (a0 + a1) * p.kappa;
      if (!(t & (1 << 30))) {
        const float4* hr4 = reinterpret_cast<const float4*>(kh + tl * kRow);
        float b0 = 0.f, b1 = 0.f;
#pragma unroll 8
        for (int c = 0; c < kD / 4; ++c) {
          const float4 qv = qr[c], kv = hr4[c];
          b0 = fmaf(qv.x, kv.x, b0);
          b1 = fmaf(qv.y, kv.y, b1);
          b0 = fmaf(qv.z, kv.z, b0);
          b1 = fmaf(qv.w, kv.w, b1);
        }
        dr = (b0 + b1) * p.kappa;
      }
    }
    ue[tl * G + j] = de;
    ur[tl * G + j] = dr;
  }
  __syncthreads();

  // ---- phase C: weights, one warp per head ----
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int j = warp; j < G; j += 8) {
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float* u = part ? ur : ue;
        const float x = u[lane * G + j];
        float m = x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kAll, m, o));
        const float w = m == -INFINITY ? 0.f : exp2f(x - m);
        const float l = warp_sum(w);
        u[lane * G + j] = w;
        if (lane == 0) {
          ml[(part * G + j) * 2] = m;
          ml[(part * G + j) * 2 + 1] = l;
        }
      }
    }
  }
  __syncthreads();

  // ---- phase D: weighted rows ----
  {
    const int c = tid & (kD - 1), part = tid >> 7;
    const float* rows = part ? vh : vx;
    const float* w = part ? ur : ue;
    float acc[G];
#pragma unroll
    for (int j = 0; j < G; ++j) acc[j] = 0.f;
    for (int tl = 0; tl < kMergeChunk; ++tl) {
      const float v = rows[tl * kRow + c];
#pragma unroll
      for (int j = 0; j < G; ++j) acc[j] = fmaf(w[tl * G + j], v, acc[j]);
    }
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float* dst = p.chunk_part +
                   ((((size_t)seg * p.n_chunks + chunk) * 2 + part) * G + j) * kPartStride;
      dst[4 + c] = acc[j];
      if (c == 0) {
        dst[0] = ml[(part * G + j) * 2];
        dst[1] = ml[(part * G + j) * 2 + 1];
      }
    }
  }
}

template <int G>
constexpr int correct_smem_bytes() {
  return (4 * kMergeChunk * kRow + G * kRow + 2 * kMergeChunk * G + 4 * G) * 4;
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

// jfa_blocks.cuh — block-level building blocks shared by the selection,
// correction and finishing kernels: scans, radix find, and the correction of
// a batch of exact tokens.
#pragma once

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


// Block-wide exclusive sum over threads in DESCENDING thread order:
// returns the sum of v over threads with a larger index.
__device__ __forceinline__ uint32_t block_suffix_excl(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_down_sync(kAll, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) scratch[warp] = x;
  __syncthreads();
  uint32_t after = 0;
  for (int w = warp + 1; w < nw; ++w) after += scratch[w];
  __syncthreads();
  return after + (x - v);
}

// Block-wide exclusive prefix sum in thread order; *total gets the sum.
__device__ __forceinline__ uint32_t block_prefix_excl(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(kAll, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
  for (int w = 0; w < nw; ++w) {
    const uint32_t t = scratch[w];
    before += w < warp ? t : 0u;
    all += t;
  }
  __syncthreads();
  *total = all;
  return before + (x - v);
}

// Given per-bin counts h[0..nbins), find the bin where the count taken from
// the top reaches r (1 <= r <= total); returns the bin and the count above it.
__device__ __forceinline__ void find_from_top(const uint32_t* h, int nbins, uint32_t r, uint32_t* scratch,
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


// Correction of one batch of up to 32 entries (all 256 threads of the block
// call it).  s_tok[i]: token index (< N_q), (1 << 30) | tail slot, or -1.
// Phase A: jobs stage the exact bf16 rows and the dequantized rows (stored
// codes, stored scales/zeros) in shared memory with 16-byte loads, every load
// of a thread issued before any is used.  Phase B: thread (token, head)
// computes exact and approximate logits (log2 units).  Phase C: one warp per
// head turns them into weights.  Phase D: thread (channel, exact|removal)
// accumulates the weighted rows into dst[2][G][kPartStride] as (m, l, acc).
struct CorrectSmem {
  float *kx, *vx, *kh, *vh, *qs, *ue, *ur, *ml;
};
template <int G>
constexpr int correct_smem_floats() {
  return 4 * kMergeChunk * kRow + G * kRow + 2 * kMergeChunk * G + 4 * G;
}
__device__ __forceinline__ CorrectSmem correct_smem_carve(float* sm, int G) {
  CorrectSmem s;
  s.kx = sm;
  s.vx = s.kx + kMergeChunk * kRow;
  s.kh = s.vx + kMergeChunk * kRow;
  s.vh = s.kh + kMergeChunk * kRow;
  s.qs = s.vh + kMergeChunk * kRow;
  s.ue = s.qs + G * kRow;
  s.ur = s.ue + kMergeChunk * G;
  s.ml = s.ur + kMergeChunk * G;
  return s;
}
// q rows of the segment's G query heads into shared memory (fp32)
template <int G>
__device__ __forceinline__ void correct_load_q(const MergeParams& p, int seg, float* qs) {
  const int b = seg / p.hkv, h = seg % p.hkv;
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
    const int j = i / kD, c = i % kD;
    qs[j * kRow + c] = bf16f(p.q[((size_t)b * p.H + h * G + j) * kD + c]);
  }
}
template <int G>
__device__ __forceinline__ void correct_batch(const MergeParams& p, int seg, const int* s_tok,
                                              const CorrectSmem& S, float* dst) {
  const int tid = threadIdx.x;
  float *kx = S.kx, *vx = S.vx, *kh = S.kh, *vh = S.vh, *qs = S.qs, *ue = S.ue, *ur = S.ur,
        *ml = S.ml;
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
      float* d = dst + (part * G + j) * kPartStride;
      d[4 + c] = acc[j];
      if (c == 0) {
        d[0] = ml[(part * G + j) * 2];
        d[1] = ml[(part * G + j) * 2 + 1];
      }
    }
  }
}

}  // namespace jfa

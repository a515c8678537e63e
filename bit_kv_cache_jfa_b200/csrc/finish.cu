// finish.cu — everything after the scan in one kernel: a thread-block cluster
// of C CTAs (C <= 8) per (sequence, KV head) runs
//   P1  histogram of the top 11 selection-key bits of each CTA's score slice,
//   P1b CTA 0 sums the C histograms through distributed shared memory and
//       finds the bin b* holding the k-th key,
//   P2  each CTA writes its slice's keys with bin >= b* to an index-ordered
//       list (block-scan compaction),
//   P3  CTA 0 refines the k-th key over those lists (two more radix levels),
//       resolves ties by index and writes the chosen indices in one ordered
//       pass (to idx and to its shared memory),
//   P4  each CTA corrects its share of the exact set (chosen tokens + tail):
//       exact bf16 logits/values and the approximate terms to remove,
//   P5  the CTAs owning a query head merge the scan partials and the exact
//       and removal partials of all C CTAs (read through distributed shared
//       memory) in log-sum-exp form and write the output row.
// Cluster barriers replace the kernel boundaries of the separate
// jfa_topk / jfa_correct_merge path; the arithmetic is the same.
#include <cooperative_groups.h>

#include "jfa_blocks.cuh"

namespace cg = cooperative_groups;

namespace jfa {

constexpr int kFinThreads = 256;
constexpr int kFinStage = 4096;  // list entries CTA 0 stages in shared memory
constexpr int kFinMaxC = 8;

struct FinishParams {
  MergeParams m;          // correction / merge inputs (m.idx unused)
  const float* scores;    // [n_seg][capacity] selection scores from the scan
  int32_t* idx_out;       // [n_seg][k]
  uint2* lists;           // [n_seg * C][slice] per-CTA ordered (key, index) lists
  int slice;              // scores per CTA, multiple of 64
};

template <int G>
constexpr size_t finish_smem_bytes() {
  constexpr size_t sel = kHistBins * 4 + kFinStage * 8;
  constexpr size_t cor = (size_t)correct_smem_floats<G>() * 4;
  return JFA_MAX_TOPK * 4 + 2 * (2 * G * kPartStride * 4) + (sel > cor ? sel : cor);
}

// Selection over an index-ordered list given by get(i), i < total: the k-th
// key K* below bin b* (r = keys still to take from bin b*), ties to the lowest
// indices, chosen indices written ascending to out[] and chosen[].
template <typename Get>
__device__ void select_ordered(Get get, uint32_t total, uint32_t bstar, uint32_t r, int k,
                               int32_t* out, int32_t* chosen, uint32_t* h, uint32_t* scratch,
                               int* s_bin, uint32_t* s_above) {
  const int tid = threadIdx.x;
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
  if (tid == 0) {
    *s_bin = 0;
    *s_above = 0;
  }
  __syncthreads();
  for (uint32_t i = tid; i < total; i += blockDim.x) {
    const uint32_t key = get(i).x;
    if ((key >> 21) == bstar) atomicAdd(&h[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  find_from_top(h, 2048, r, scratch, s_bin, s_above);
  const uint32_t d2 = (uint32_t)*s_bin;
  const uint32_t r2 = r - *s_above;
  const uint32_t pre = (bstar << 11) | d2;
  __syncthreads();
  for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < total; i += blockDim.x) {
    const uint32_t key = get(i).x;
    if ((key >> 10) == pre) atomicAdd(&h[key & 1023u], 1u);
  }
  __syncthreads();
  find_from_top(h, 1024, r2, scratch, s_bin, s_above);
  const uint32_t kstar = (pre << 10) | (uint32_t)*s_bin;
  const uint32_t r3 = r2 - *s_above;
  // thread t owns entries [t*per, (t+1)*per), so block scans order the list
  const uint32_t per = (total + blockDim.x - 1) / blockDim.x;
  const uint32_t i0 = tid * per, i1 = min(total, i0 + per);
  uint32_t n_eq = 0;
  for (uint32_t i = i0; i < i1; ++i) n_eq += get(i).x == kstar;
  uint32_t tot;
  uint32_t eq_rank = block_prefix_excl(n_eq, scratch, &tot);
  uint32_t n_ch = 0;
  {
    uint32_t er = eq_rank;
    for (uint32_t i = i0; i < i1; ++i) {
      const uint32_t key = get(i).x;
      const bool eq = key == kstar;
      n_ch += (key > kstar || (eq && er < r3)) ? 1u : 0u;
      er += eq;
    }
  }
  uint32_t pos = block_prefix_excl(n_ch, scratch, &tot);
  for (uint32_t i = i0; i < i1; ++i) {
    const uint2 e = get(i);
    const bool eq = e.x == kstar;
    if (e.x > kstar || (eq && eq_rank < r3)) {
      if (pos < (uint32_t)k) {
        out[pos] = (int32_t)e.y;
        chosen[pos] = (int32_t)e.y;
      }
      ++pos;
    }
    eq_rank += eq;
  }
}

// L2 prefetch of what the correction of token t reads (t: token index, or
// (1 << 30) | tail slot): bf16 K/V rows and, for quantized tokens, the key
// scales/zeros, key codes and value scales/codes of its record.  part picks
// one of kPrefParts 128-byte pieces, so consecutive threads split the work.
constexpr int kPrefParts = 12;
__device__ __forceinline__ void prefetch_token(const MergeParams& p, int seg, int t, int part) {
  if (t < 0) return;
  if (t & (1 << 30)) {
    const int tt = t & ~(1 << 30);
    if (part < 4) {
      const uint16_t* row = ((part & 2) ? p.tail_v : p.tail_k) + ((size_t)seg * kTail + tt) * kD;
      prefetch_l2(row + 64 * (part & 1));
    }
    return;
  }
  const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + t / kKG) * p.rec_bytes;
  const int tt = t % kKG;
  if (part < 4) {
    const uint16_t* row = ((part & 2) ? p.v_exact : p.k_exact) + ((size_t)seg * p.capacity + t) * kD;
    prefetch_l2(row + 64 * (part & 1));
  } else if (part < 8) {
    prefetch_l2(rec + off_ks() + 128 * (part - 4));  // key scales/zeros (512 B)
  } else if (part == 8) {
    const int nt = tt >> 3, gd = tt & 7;
    prefetch_l2(rec + off_kc() +
                (p.key_bits == 4 ? nt * 512 + gd * 64 : (nt >> 2) * 1536 + gd * 192));
  } else if (part == 9) {
    prefetch_l2(rec + off_vs(p.key_bits) + (tt >> 4) * 128);
  } else {
    const int kk = tt >> 4;
    const int chunk = p.val_bits == 4 ? 2 * kk + (part - 10) : kk;
    prefetch_l2(rec + off_vc(p.key_bits) + chunk * 512 + 256 * (p.val_bits == 4 ? 0 : (part - 10)));
  }
}

template <int G>
__global__ void __launch_bounds__(kFinThreads, 2) finish_kernel(const FinishParams fp) {
  extern __shared__ __align__(16) uint8_t fsm[];
  const MergeParams& p = fp.m;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  const int r = (int)cl.block_rank();
  const int seg = blockIdx.x / C;
  const int tid = threadIdx.x;
  int32_t* chosen = reinterpret_cast<int32_t*>(fsm);
  float* run = reinterpret_cast<float*>(fsm + JFA_MAX_TOPK * 4);  // [2][G][kPartStride]
  float* bat = run + 2 * G * kPartStride;                          // [2][G][kPartStride]
  uint8_t* U = reinterpret_cast<uint8_t*>(bat + 2 * G * kPartStride);
  uint32_t* hist = reinterpret_cast<uint32_t*>(U);
  uint2* stage = reinterpret_cast<uint2*>(U + kHistBins * 4);
  __shared__ uint32_t scratch[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  __shared__ uint32_t s_bstar, s_babove, s_count;
  __shared__ uint32_t s_off[kFinMaxC + 1];
  __shared__ int s_tok[kMergeChunk];

  pdl_wait();
  pdl_launch_dependents();

  const int nq = p.nq, k = p.k;
  const int keff = min(k, nq);
  const bool select = k < nq;
  const int lo = r * fp.slice, hi = min(nq, lo + fp.slice);
  const float* S = fp.scores + (size_t)seg * p.capacity;
  uint2* lists = fp.lists + (size_t)seg * C * fp.slice;
  // exact-set share of this CTA (P4) and scan slots it merges (P5a)
  const int nE = keff + p.tail;
  const int e_per = (nE + C - 1) / C;
  const int e0 = r * e_per, e1 = min(nE, e0 + e_per);
  long long w0 = 0, w1 = -1;
  if (p.ng > 0) {
    const long long T = p.scan_total, W = p.scan_warps;
    const long long x0 = (long long)seg * p.ng, x1 = x0 + p.ng - 1;
    w0 = scan_warp_of(x0, W, T);
    w1 = scan_warp_of(x1, W, T);
  }
  const int ns = (int)(w1 - w0 + 1);
  const int s0 = (int)((long long)ns * r / C), s1 = (int)((long long)ns * (r + 1) / C);
  // known from the start: the tail tokens among this CTA's share, and its
  // scan-slot rows -- start pulling them into L2 now
  for (int i = tid; i < (e1 - e0) * kPrefParts; i += kFinThreads) {
    const int e = e0 + i / kPrefParts;
    if (e >= keff) prefetch_token(p, seg, (1 << 30) | (e - keff), i % kPrefParts);
  }
  for (int i = tid; i < (s1 - s0) * G * 5; i += kFinThreads) {
    const int row = s0 * G + i / 5;
    prefetch_l2(p.scan_part + ((size_t)(w0 + row / G + seg) * G + row % G) * kPartStride +
                32 * (i % 5));
  }

  // ---- P1: histogram of this CTA's slice
  if (select) {
    for (int i = tid; i < kHistBins; i += kFinThreads) hist[i] = 0u;
    __syncthreads();
    for (int t0 = lo; t0 < hi; t0 += 16 * kFinThreads) {
      const int b0 = t0 + 16 * tid;
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = b0 + 4 * u < hi ? *reinterpret_cast<const float4*>(S + b0 + 4 * u)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (b0 + 4 * u < hi) {
          atomicAdd(&hist[float_key(v[u].x) >> 21], 1u);
          atomicAdd(&hist[float_key(v[u].y) >> 21], 1u);
          atomicAdd(&hist[float_key(v[u].z) >> 21], 1u);
          atomicAdd(&hist[float_key(v[u].w) >> 21], 1u);
        }
      }
    }
  }
  cl.sync();

  // ---- P1b: CTA 0 sums the histograms (all remote loads issued first) and finds b*
  if (select && r == 0) {
    uint4 hv[kFinMaxC][2];
#pragma unroll
    for (int q = 0; q < kFinMaxC; ++q) {
      if (q < C) {
        const uint4* ph = reinterpret_cast<const uint4*>(cl.map_shared_rank(hist, q)) + 2 * tid;
        hv[q][0] = ph[0];
        hv[q][1] = ph[1];
      }
    }
    uint32_t tot[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int q = 0; q < kFinMaxC; ++q) {
      if (q < C) {
        tot[0] += hv[q][0].x;
        tot[1] += hv[q][0].y;
        tot[2] += hv[q][0].z;
        tot[3] += hv[q][0].w;
        tot[4] += hv[q][1].x;
        tot[5] += hv[q][1].y;
        tot[6] += hv[q][1].z;
        tot[7] += hv[q][1].w;
      }
    }
    __syncthreads();
    reinterpret_cast<uint4*>(hist)[2 * tid] = make_uint4(tot[0], tot[1], tot[2], tot[3]);
    reinterpret_cast<uint4*>(hist)[2 * tid + 1] = make_uint4(tot[4], tot[5], tot[6], tot[7]);
    if (tid == 0) {
      s_bin = 0;
      s_above = 0;
    }
    __syncthreads();
    find_from_top(hist, kHistBins, (uint32_t)k, scratch, &s_bin, &s_above);
    if (tid == 0) {
      s_bstar = (uint32_t)s_bin;
      s_babove = s_above;
    }
  }
  cl.sync();

  // ---- P2: index-ordered list of this slice's keys with bin >= b*
  if (select) {
    const uint32_t bstar = *cl.map_shared_rank(&s_bstar, 0);
    uint2* lst = lists + (size_t)r * fp.slice;
    uint32_t base_out = 0;
    for (int t0 = lo; t0 < hi; t0 += 16 * kFinThreads) {
      const int b0 = t0 + 16 * tid;
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = b0 + 4 * u < hi ? *reinterpret_cast<const float4*>(S + b0 + 4 * u)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      uint32_t keys[16];
      uint32_t mask = 0, n = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * u + e;
          keys[i] = float_key(vals[e]);
          const bool in = (b0 + i < hi) && (keys[i] >> 21) >= bstar;
          mask |= (in ? 1u : 0u) << i;
          n += in ? 1u : 0u;
        }
      }
      uint32_t total;
      uint32_t pos = base_out + block_prefix_excl(n, scratch, &total);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (mask & (1u << i)) lst[pos++] = make_uint2(keys[i], (uint32_t)(b0 + i));
      base_out += total;
    }
    if (tid == 0) s_count = base_out;
  }
  cl.sync();

  // ---- P3: CTA 0 selects the k tokens
  if (r == 0) {
    int32_t* out = fp.idx_out + (size_t)seg * k;
    if (!select) {
      for (int i = tid; i < k; i += kFinThreads) {
        out[i] = i < nq ? i : -1;
        if (i < keff) chosen[i] = i;
      }
    } else {
      if (tid < 32) {
        const uint32_t cnt = tid < C ? *cl.map_shared_rank(&s_count, tid) : 0u;
        uint32_t x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(kAll, x, o);
          if (tid >= o) x += y;
        }
        if (tid < C) s_off[tid] = x - cnt;
        if (tid == C - 1) s_off[C] = x;
      }
      __syncthreads();
      const uint32_t total = s_off[C];
      const uint32_t bstar = s_bstar;
      const uint32_t rr = (uint32_t)k - s_babove;  // keys still to take from bin b*
      const int slice = fp.slice;
      const int nC = C;
      auto in_place = [&](uint32_t j) -> uint2 {
        int q = 0;
        while (q + 1 < nC && s_off[q + 1] <= j) ++q;
        return lists[(size_t)q * slice + (j - s_off[q])];
      };
      if (total <= (uint32_t)kFinStage) {
        for (uint32_t j = tid; j < total; j += kFinThreads) stage[j] = in_place(j);
        __syncthreads();
        auto staged = [&](uint32_t j) -> uint2 { return stage[j]; };
        select_ordered(staged, total, bstar, rr, k, out, chosen, hist, scratch, &s_bin, &s_above);
      } else {
        select_ordered(in_place, total, bstar, rr, k, out, chosen, hist, scratch, &s_bin,
                       &s_above);
      }
    }
  }
  cl.sync();

  // ---- P4: correction of this CTA's share of the exact set
  {
    const int32_t* chosen0 = cl.map_shared_rank(chosen, 0);
    // every chosen token of the share is known now: pull its rows and record
    // pieces into L2 before the batches read them
    for (int i = tid; i < (min(e1, keff) - e0) * kPrefParts; i += kFinThreads)
      prefetch_token(p, seg, chosen0[e0 + i / kPrefParts], i % kPrefParts);
    const CorrectSmem CS = correct_smem_carve(reinterpret_cast<float*>(U), G);
    correct_load_q<G>(p, seg, CS.qs);
    for (int i = tid; i < 2 * G * kPartStride; i += kFinThreads) run[i] = 0.f;
    __syncthreads();
    if (tid < 2 * G) run[tid * kPartStride] = -INFINITY;
    for (int eb = e0; eb < e1; eb += kMergeChunk) {
      __syncthreads();
      if (tid < kMergeChunk) {
        const int e = eb + tid;
        int t = -1;
        if (e < e1) t = e < keff ? chosen0[e] : ((1 << 30) | (e - keff));
        s_tok[tid] = t;
      }
      __syncthreads();
      correct_batch<G>(p, seg, s_tok, CS, bat);
      __syncthreads();
      // fold the batch partial into the running one
      const int c = tid & (kD - 1), part = tid >> 7;
      float mv[G], lv[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float* ro = run + (part * G + j) * kPartStride;
        const float* bo = bat + (part * G + j) * kPartStride;
        const float m1 = ro[0], l1 = ro[1], m2 = bo[0], l2 = bo[1];
        const float mn = fmaxf(m1, m2);
        const float s1 = l1 > 0.f ? exp2f(m1 - mn) : 0.f;
        const float s2 = l2 > 0.f ? exp2f(m2 - mn) : 0.f;
        mv[j] = (l1 > 0.f || l2 > 0.f) ? mn : -INFINITY;
        lv[j] = l1 * s1 + l2 * s2;
        run[(part * G + j) * kPartStride + 4 + c] = ro[4 + c] * s1 + bo[4 + c] * s2;
      }
      __syncthreads();
      if (c == 0) {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          run[(part * G + j) * kPartStride] = mv[j];
          run[(part * G + j) * kPartStride + 1] = lv[j];
        }
      }
    }
  }
  cl.sync();

  // ---- P5a: each CTA merges its share of the scan slots for every head into
  // sp[G][kPartStride] (one tiled pass with all loads of a tile in flight)
  float* sp = bat;  // the batch buffer is free now: [G][kPartStride] (first half)
  {
    float* tile = reinterpret_cast<float*>(U);
    constexpr int kTile = (int)(((size_t)correct_smem_floats<G>()) / kPartStride);  // rows per tile
    const int c = tid & (kD - 1);
    float mrun[G], lrun[G], arun[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      mrun[j] = -INFINITY;
      lrun[j] = 0.f;
      arun[j] = 0.f;
    }
    for (int t0 = s0 * G; t0 < s1 * G; t0 += kTile) {
      const int nr = min(kTile, s1 * G - t0);
      __syncthreads();
      for (int i = tid; i < nr * (kPartStride / 4); i += kFinThreads) {
        const int row = i / (kPartStride / 4), v = i % (kPartStride / 4);
        const int gr = t0 + row;  // row = slot * G + head
        reinterpret_cast<float4*>(tile + row * kPartStride)[v] = reinterpret_cast<const float4*>(
            p.scan_part + ((size_t)(w0 + gr / G + seg) * G + gr % G) * kPartStride)[v];
      }
      __syncthreads();
      if (tid < kD) {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          float tm = mrun[j];
          for (int row = (j - t0 % G + G) % G; row < nr; row += G)
            if (tile[row * kPartStride + 1] > 0.f) tm = fmaxf(tm, tile[row * kPartStride]);
          const float sc0 = (lrun[j] > 0.f) ? exp2f(mrun[j] - tm) : 0.f;
          float l = lrun[j] * sc0, a = arun[j] * sc0;
          for (int row = (j - t0 % G + G) % G; row < nr; row += G) {
            const float lb = tile[row * kPartStride + 1];
            if (lb > 0.f) {
              const float sc = exp2f(tile[row * kPartStride] - tm);
              l = fmaf(lb, sc, l);
              a = fmaf(tile[row * kPartStride + 4 + c], sc, a);
            }
          }
          mrun[j] = tm;
          lrun[j] = l;
          arun[j] = a;
        }
      }
    }
    if (tid < kD) {
#pragma unroll
      for (int j = 0; j < G; ++j) {
        sp[j * kPartStride + 4 + c] = arun[j];
        if (c == 0) {
          sp[j * kPartStride] = lrun[j] > 0.f ? mrun[j] : -INFINITY;
          sp[j * kPartStride + 1] = lrun[j];
        }
      }
    }
  }
  cl.sync();

  // ---- P5b: CTA r owns heads j = r, r + C, ...: merge the C scan, exact and
  // removal partials (remote loads issued together) and write the output row
  for (int j = r; j < G; j += C) {
    const int c = tid;
    if (c < kD) {
      float2 hd[kFinMaxC][3];  // (m, l) of scan / exact / removal parts
      float av[kFinMaxC][3];   // channel c of each
#pragma unroll
      for (int q = 0; q < kFinMaxC; ++q) {
        if (q < C) {
          const float* spq = cl.map_shared_rank(sp, q) + j * kPartStride;
          const float* rq = cl.map_shared_rank(run, q);
          const float* re = rq + (0 * G + j) * kPartStride;
          const float* rm = rq + (1 * G + j) * kPartStride;
          hd[q][0] = *reinterpret_cast<const float2*>(spq);
          hd[q][1] = *reinterpret_cast<const float2*>(re);
          hd[q][2] = *reinterpret_cast<const float2*>(rm);
          av[q][0] = spq[4 + c];
          av[q][1] = re[4 + c];
          av[q][2] = rm[4 + c];
        }
      }
      float mk[3] = {-INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int q = 0; q < kFinMaxC; ++q)
        if (q < C) {
#pragma unroll
          for (int t = 0; t < 3; ++t)
            if (hd[q][t].y > 0.f) mk[t] = fmaxf(mk[t], hd[q][t].x);
        }
      float lk[3] = {0.f, 0.f, 0.f}, ak[3] = {0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < kFinMaxC; ++q)
        if (q < C) {
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            const float sc = hd[q][t].y > 0.f ? exp2f(hd[q][t].x - mk[t]) : 0.f;
            lk[t] = fmaf(hd[q][t].y, sc, lk[t]);
            ak[t] = fmaf(av[q][t], sc, ak[t]);
          }
        }
      const float ma = mk[0], la = lk[0], aa = ak[0];
      const float me = mk[1], le = lk[1], ae = ak[1];
      const float mr = mk[2], lr = lk[2], ar = ak[2];
      // remainder = approximate total minus the removed top-k terms (m_a frame)
      float lrest = la, arest = aa;
      if (la > 0.f && lr > 0.f) {
        const float f = exp2f(mr - ma);
        lrest = la - lr * f;
        arest = aa - ar * f;
        if (lrest < 0.f) lrest = 0.f;
      }
      float mm = me, wl = 1.f, wa = 0.f;
      if (la > 0.f) {
        mm = fmaxf(me, ma);
        wl = exp2f(me - mm);
        wa = exp2f(ma - mm);
      }
      const int b = seg / p.hkv, h = seg % p.hkv;
      p.out[((size_t)b * p.H + h * G + j) * kD + c] = (ae * wl + arest * wa) / (le * wl + lrest * wa);
    }
  }
  // keep this CTA's shared memory alive until every peer has read it
  cl.sync();
}

// Largest cluster size (<= 8) whose clusters all fit on the device at once
// (so the whole grid runs in one wave), using up to about two CTAs per SM.
template <int G>
static int pick_cluster(int n_seg, int num_sms) {
  constexpr size_t smem = finish_smem_bytes<G>();
  int best = 1;
  for (int c = 2; c <= kFinMaxC; c *= 2) {
    if ((long long)n_seg * c > 2LL * num_sms) break;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_seg * c);
    cfg.blockDim = dim3(kFinThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = c;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n_active = 0;
    if (cudaOccupancyMaxActiveClusters(&n_active, finish_kernel<G>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      break;
    }
    if (n_active >= n_seg) best = c;
    else break;
  }
  return best;
}

template <int G>
static int launch_finish_t(FinishParams fp, int n_seg, cudaStream_t st) {
  constexpr size_t smem = finish_smem_bytes<G>();
  static bool configured[64] = {false};
  static int memo_seg[64][8] = {{0}}, memo_c[64][8] = {{0}};  // cluster size per (device, n_seg)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(finish_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return JFA_ERR_CUDA;
    configured[dev] = true;
  }
  int C = 0;
  if (dev >= 0 && dev < 64) {
    for (int i = 0; i < 8; ++i)
      if (memo_seg[dev][i] == n_seg) C = memo_c[dev][i];
  }
  if (C == 0) {
    C = pick_cluster<G>(n_seg, num_sms_current());
    if (dev >= 0 && dev < 64) {
      for (int i = 0; i < 8; ++i)
        if (memo_seg[dev][i] == 0) {
          memo_seg[dev][i] = n_seg;
          memo_c[dev][i] = C;
          break;
        }
    }
  }
  const int nq = fp.m.nq;
  fp.slice = nq > 0 ? ((nq + C - 1) / C + 63) / 64 * 64 : 64;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_seg * C);
  cfg.blockDim = dim3(kFinThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, finish_kernel<G>, fp) == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

int launch_finish(const jfa_geom& g, const jfa_cache& c, const uint16_t* q, float scale, int k,
                  int32_t* idx, const uint16_t* k_exact, const uint16_t* v_exact, uint8_t* ws,
                  const jfa_workspace_layout& L, float* out, cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  FinishParams fp;
  MergeParams& p = fp.m;
  p.groups = static_cast<const uint8_t*>(c.groups);
  p.tail_k = c.tail_k;
  p.tail_v = c.tail_v;
  p.k_exact = k_exact;
  p.v_exact = v_exact;
  p.q = q;
  p.idx = idx;
  p.scan_part = reinterpret_cast<const float*>(ws + L.off_partials);
  p.chunk_part = nullptr;
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
  p.n_chunks = 0;
  p.key_bits = g.key_bits;
  p.val_bits = g.val_bits;
  p.rec_bytes = record_bytes(g.key_bits, g.val_bits);
  ScanPlan plan = scan_plan(g, num_sms_current());
  p.scan_total = plan.total_groups;
  p.scan_warps = plan.n_warps;
  p.ng = plan.ng;
  p.kappa = scale * 1.4426950408889634f;
  fp.scores = reinterpret_cast<const float*>(ws + L.off_scores);
  fp.idx_out = idx;
  fp.lists = reinterpret_cast<uint2*>(ws + L.off_cand);
  switch (p.G) {
    case 1: return launch_finish_t<1>(fp, n_seg, st);
    case 2: return launch_finish_t<2>(fp, n_seg, st);
    case 3: return launch_finish_t<3>(fp, n_seg, st);
    case 4: return launch_finish_t<4>(fp, n_seg, st);
    case 5: return launch_finish_t<5>(fp, n_seg, st);
    case 6: return launch_finish_t<6>(fp, n_seg, st);
    case 7: return launch_finish_t<7>(fp, n_seg, st);
    default: return launch_finish_t<8>(fp, n_seg, st);
  }
}

}  // namespace jfa

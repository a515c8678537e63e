// finish_impl.cuh — everything after the scan in one kernel.  A thread-block
// cluster of C CTAs (C <= 16) per (sequence, KV head); CTA r owns slice r of
// the quantized tokens and the tail slots r, r + C, ...
//
//   T   corrects its tail slots while the histogram's first load is in
//       flight.  A correction folds a token into the warp's running fp32
//       softmax partial per query head: its exact bf16 term in, the scan's
//       approximate term out (the fp16 weights the scan stored, against the
//       running maximum it stored, times the dequantized value);
//   S1  reads a window of the scan's 32768-bin histogram of the selection
//       keys below the segment's largest key and finds the bin b* holding
//       the k-th largest key (every CTA, redundantly);
//   S2  lists its slice's keys above b* ("sure": chosen whatever the ties
//       decide) and in b* ("ties"), in index order;
//   S3  after a cluster barrier, gathers every CTA's ties and ranks them
//       (larger key first, equal keys to the lower index);
//   C   corrects an even share of the chosen set (the CTAs' sure lists read
//       through distributed shared memory, then the chosen ties) and writes
//       its slice's chosen indices, ascending, at its offset of idx;
//   M   merges its warps' partials and its share of the scan's split
//       partials; the CTAs owning a query head combine the C CTAs' partials
//       (distributed shared memory) in log-sum-exp form and write out.
// With a given index set (jfa_correct_merge) or k >= N_q there is no
// selection: C corrects the CTA's even share of the set.  If the histogram
// does not hold the k-th key where the stored scores put it, or a list
// overflows, every CTA selects over the whole segment from the stored scores
// instead (slower, same result).
#pragma once

#include <cooperative_groups.h>
#include <mutex>

#include "finish_params.cuh"
#include "jfa_approx.cuh"
#include "jfa_blocks.cuh"

namespace cg = cooperative_groups;

namespace jfa {

constexpr int kFinThreads = 256;
constexpr int kFinWarps = kFinThreads / 32;
constexpr int kFinMaxC = kFinMaxCluster;  // 16: non-portable cluster size, few segments only
constexpr int kLCap = 1024;   // sure / tie list entries per CTA
constexpr int kTCap = 1024;   // gathered tie entries
constexpr int kRefBins = 2048;
constexpr int kTokCap = 1024;  // tokens listed per correction round (plus the tail slots)
constexpr int kChunk = 4;      // tokens a warp stages at once

// Shared memory.  The persistent part is read by the other CTAs of the
// cluster (lists, counts, partials) and lives until the last barrier.
struct FinPersist {
  uint32_t sure[kLCap];               // chosen-for-sure indices of the slice, ascending
  uint32_t tkey[kLCap], tidx[kLCap];  // ties of the slice (key, index), ascending index
  uint32_t chtie[kTCap];              // chosen ties of the whole segment, ascending
  uint32_t n_sure, n_tie, overflow, n_gl;
};
// Partials (m, l, pad, pad, acc[128]): `sp` per query head this CTA's share
// of the scan's split partials; `recv` for the heads this CTA owns (j with
// j mod C = rank) the C CTAs' partials of head j (their exact-minus-removed
// terms together with their share of the scan's partials), slot
// (j / C) C + source rank, written by the sources.
template <int G>
struct FinParts {
  float sp[G][kPartStride];
  float recv[kFinMaxC > kMaxG ? kFinMaxC : kMaxG][kPartStride];
};
// Shared-memory histograms store bin b at hpad(b) = b + b/32, so threads
// that each read a contiguous run of bins hit distinct banks.
__device__ __forceinline__ int hpad(int b) { return b + (b >> 5); }

// Pieces of one quantized token, staged by its warp (16-byte copies).
struct TokPieces {
  uint8_t vp[256];     // value-code pieces holding its column (8 or 16 x 16 B)
  uint8_t vsz[64];     // its value scales (32 B block) and zeros (32 B block)
  uint32_t w[8];       // the scan's fp16 weights: word 4n + j = head 4n + j, tokens
                       // (t mod 8) (low half) and (t mod 8) + 8 of its m-tile
  float mu[kMaxG];     // the scan's running maxima of its group, per head
};
static_assert(sizeof(TokPieces) == 384, "token pieces layout");
constexpr int kTokPieces16 = 24;  // 16-byte copies per token

struct FinWork {                 // correction working set
  TokPieces ring[kFinWarps][kChunk];
  uint32_t akey[kTCap], aidx[kTCap];      // gathered ties
  uint32_t hist[kRefBins + kRefBins / 32];
};
template <int G>
struct FinMerge {                // warps' partials, after the correction
  float w[kFinWarps][G][kPartStride];
};
template <int G>
constexpr size_t fin_union_bytes() {
  return sizeof(FinWork) > sizeof(FinMerge<G>) ? sizeof(FinWork) : sizeof(FinMerge<G>);
}
// Early copy of the CTA's share of the scan partials: 77 (slot, head) rows,
// enough for the shares of 32K-128K segments at G = 4 and G = 8 (larger
// shares are staged a tile at a time); two CTAs per SM still fit at G = 8.
constexpr size_t kEarlyBytes = 40 * 1024;
template <int G>
constexpr size_t fin_smem_bytes() {
  return sizeof(FinPersist) + sizeof(FinParts<G>) + (size_t)G * kD * sizeof(float) +
         (kTokCap + kTail) * sizeof(int32_t) + fin_union_bytes<G>() + kEarlyBytes;
}

// From bin counts h[hpad(0..nbins)) (nbins a multiple of blockDim) find the
// bin where the count taken from the top reaches r (1 <= r); *bin = -1 if
// the total < r.
static __device__ __noinline__ void find_bin_from_top(const uint32_t* h, int nbins, uint32_t r,
                                                      uint32_t* scratch, int* bin, uint32_t* above,
                                                      uint32_t* total) {
  const int per = nbins / blockDim.x;
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += h[hpad(b0 + i)];
  uint32_t tot;
  block_prefix_excl(local, scratch, &tot);
  uint32_t cum = block_suffix_excl(local, scratch);
  if (threadIdx.x == 0) *bin = -1;
  __syncthreads();
  for (int i = per - 1; i >= 0; --i) {
    const uint32_t c = h[hpad(b0 + i)];
    if (cum < r && cum + c >= r) {
      *bin = b0 + i;
      *above = cum;
    }
    cum += c;
  }
  if (threadIdx.x == 0) *total = tot;
  __syncthreads();
}

// Selection inside the histogram bin b* (keys share their top 15 bits): the
// r largest of the T ties akey/aidx (index order), larger key first and equal
// keys to the lower index, two radix levels over the other 17 bits (8 + 9)
// and one ordered pass.  Writes the chosen indices ascending to chosen[] (r
// of them).
constexpr int kRef2Shift = 32 - kScanHistBits - 8;  // level 2: the next 8 bits
constexpr int kRef3Bits = kRef2Shift;              // level 3: the rest (9 bits)
static_assert(kRef3Bits == 9, "refinement levels cover the key");
static __device__ __noinline__ void refine_ties(const uint32_t* akey, const uint32_t* aidx, uint32_t T,
                                                uint32_t r, uint32_t* h, uint32_t* chosen,
                                                uint32_t* scratch, int* s_bin, uint32_t* s_above,
                                                uint32_t* s_tot) {
  const int tid = threadIdx.x;
  constexpr uint32_t m2 = 255u, m3 = (1u << kRef3Bits) - 1u;
  // level 2: the 8 key bits below the shared ones
  for (int i = tid; i < hpad(256); i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < T; i += blockDim.x) atomicAdd(&h[hpad((akey[i] >> kRef2Shift) & m2)], 1u);
  __syncthreads();
  find_bin_from_top(h, 256, r, scratch, s_bin, s_above, s_tot);
  const uint32_t d2 = (uint32_t)*s_bin;
  const uint32_t r2 = r - *s_above;
  __syncthreads();
  // level 3: the low bits among keys whose level-2 digit is d2
  for (int i = tid; i < hpad(1 << kRef3Bits); i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < T; i += blockDim.x)
    if (((akey[i] >> kRef2Shift) & m2) == d2) atomicAdd(&h[hpad(akey[i] & m3)], 1u);
  __syncthreads();
  find_bin_from_top(h, 1 << kRef3Bits, r2, scratch, s_bin, s_above, s_tot);
  const uint32_t low = (akey[0] >> (32 - kScanHistBits)) << (32 - kScanHistBits);  // the shared top bits
  const uint32_t kstar = low | (d2 << kRef2Shift) | (uint32_t)*s_bin;
  const uint32_t r3 = r2 - *s_above;
  __syncthreads();
  // ordered pass: thread t owns entries [t*per, (t+1)*per)
  const uint32_t per = (T + blockDim.x - 1) / blockDim.x;
  const uint32_t i0 = min(T, tid * per), i1 = min(T, i0 + per);
  uint32_t n_eq = 0;
  for (uint32_t i = i0; i < i1; ++i) n_eq += akey[i] == kstar;
  uint32_t tot;
  uint32_t er = block_prefix_excl(n_eq, scratch, &tot);
  uint32_t n_ch = 0;
  {
    uint32_t e2 = er;
    for (uint32_t i = i0; i < i1; ++i) {
      const bool eq = akey[i] == kstar;
      n_ch += (akey[i] > kstar || (eq && e2 < r3)) ? 1u : 0u;
      e2 += eq;
    }
  }
  uint32_t pos = block_prefix_excl(n_ch, scratch, &tot);
  for (uint32_t i = i0; i < i1; ++i) {
    const bool eq = akey[i] == kstar;
    if (akey[i] > kstar || (eq && er < r3)) chosen[pos++] = aidx[i];
    er += eq;
  }
  __syncthreads();
}

// Fallback selection over the whole segment (stale histogram or too many
// candidates): three radix levels (11 + 11 + 10 bits) over all nq scores, then this CTA's slice
// [lo, hi) of chosen indices, ascending, into out[]; returns their count.
static __device__ __noinline__ uint32_t select_full(const float* S, int nq, int k, int lo, int hi,
                                                    uint32_t* h, uint32_t* out, uint32_t* scratch,
                                                    int* s_bin, uint32_t* s_above, uint32_t* s_tot) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, r = (uint32_t)k;
  const int shifts[3] = {21, 10, 0};
  const int bits[3] = {11, 11, 10};
#pragma unroll 1
  for (int lv = 0; lv < 3; ++lv) {
    const int nb = 1 << bits[lv];
    for (int i = tid; i < hpad(nb); i += blockDim.x) h[i] = 0u;
    __syncthreads();
    const int hs = lv == 0 ? 32 : shifts[lv - 1];
    for (int i = tid; i < nq; i += blockDim.x) {
      const uint32_t key = float_key(S[i]);
      if (lv == 0 || (key >> hs) == prefix) atomicAdd(&h[hpad((key >> shifts[lv]) & (nb - 1))], 1u);
    }
    __syncthreads();
    find_bin_from_top(h, nb, r, scratch, s_bin, s_above, s_tot);
    prefix = (prefix << bits[lv]) | (uint32_t)*s_bin;
    r -= *s_above;
    __syncthreads();
  }
  const uint32_t kstar = prefix;
  // equal keys before the slice
  uint32_t n_eq = 0;
  for (int i = tid; i < lo; i += blockDim.x) n_eq += float_key(S[i]) == kstar;
  uint32_t tot;
  block_prefix_excl(n_eq, scratch, &tot);
  const uint32_t eq_before = tot;
  const uint32_t len = (uint32_t)(hi - lo);
  const uint32_t per = (len + blockDim.x - 1) / blockDim.x;
  const uint32_t i0 = min(len, tid * per), i1 = min(len, i0 + per);
  uint32_t ne = 0;
  for (uint32_t i = i0; i < i1; ++i) ne += float_key(S[lo + i]) == kstar;
  uint32_t er = eq_before + block_prefix_excl(ne, scratch, &tot);
  uint32_t nc = 0;
  {
    uint32_t e2 = er;
    for (uint32_t i = i0; i < i1; ++i) {
      const uint32_t key = float_key(S[lo + i]);
      const bool eq = key == kstar;
      nc += (key > kstar || (eq && e2 < r)) ? 1u : 0u;
      e2 += eq;
    }
  }
  uint32_t pos = block_prefix_excl(nc, scratch, &tot);
  for (uint32_t i = i0; i < i1; ++i) {
    const uint32_t key = float_key(S[lo + i]);
    const bool eq = key == kstar;
    if (key > kstar || (eq && er < r)) out[pos++] = (uint32_t)(lo + i);
    er += eq;
  }
  __syncthreads();
  return tot;
}

// Number of entries of the ascending list a[0..n) below v.
__device__ __forceinline__ uint32_t lower_bound_u32(const uint32_t* a, uint32_t n, uint32_t v) {
  uint32_t lo = 0, hi = n;
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// Correction.  Token encoding: t in [0, nq) a quantized token,
// (1 << 30) | s the tail slot s (exact rows only); -1 none.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool tok_quant(int t) { return t >= 0 && !(t & (1 << 30)); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 16-byte piece i (0..23) of quantized token t's pieces into S: value codes,
// value scales/zeros, the scan's weights (NT n-tiles) and running maxima.
template <int KB, int VB, int NT>
__device__ __forceinline__ void stage_piece(const FinishParams& p, int seg, int t, TokPieces& S, int i) {
  const int g = t / kKG;
  const size_t rg = (size_t)seg * p.ng_cap + (size_t)g;
  const uint8_t* rec = p.groups + rg * p.rec_bytes;
  const int tt = t % kKG, kk = tt >> 4, row = tt & 7, tgt = (tt & 7) >> 1;
  if (i < 16) {
    if (VB == 4 || i < 8) {
      const int chunk = VB == 4 ? 2 * kk + (i >> 3) : kk;
      cp_async16(S.vp + 16 * i, rec + off_vc(KB) + chunk * 512 + ((i & 7) * 4 + tgt) * 16);
    }
  } else if (i < 20) {
    const int j = i - 16;
    cp_async16(S.vsz + 16 * j, rec + off_vs(KB) + kk * 128 + tgt * 32 + (j & 1) * 16 + (j >> 1) * 512);
  } else if (i < 22) {
    const int n = i - 20;
    if (n < NT) cp_async16(S.w + 4 * n, p.wts + (rg * 4 * NT + (size_t)(kk * NT + n)) * 32 + row * 4);
  } else {
    const int j = i - 22;
    cp_async16(S.mu + 4 * j, p.m_used + rg * kMaxG + 4 * j);
  }
}

// The lane's 4 channels (4 lane .. 4 lane + 3) of token t's exact K (v =
// false) or V row, as raw bf16 pairs.
__device__ __forceinline__ uint2 row4(const FinishParams& p, int seg, int t, bool v, int lane) {
  const bool tail = (t & (1 << 30)) != 0;
  const size_t off = tail ? ((size_t)seg * kTail + (t & 0xFFFF)) * kD : ((size_t)seg * p.capacity + t) * kD;
  const uint16_t* base = v ? (tail ? p.tail_v : p.v_exact) : (tail ? p.tail_k : p.k_exact);
  return *reinterpret_cast<const uint2*>(base + off + 4 * lane);
}

// L2 prefetch of one of the four 128-byte halves of token t's exact K and V rows.
__device__ __forceinline__ void prefetch_part(const FinishParams& p, int seg, int t, int part) {
  const bool tail = (t & (1 << 30)) != 0;
  const size_t off = tail ? ((size_t)seg * kTail + (t & 0xFFFF)) * kD : ((size_t)seg * p.capacity + t) * kD;
  const uint16_t* base = (part & 2) ? (tail ? p.tail_v : p.v_exact) : (tail ? p.tail_k : p.k_exact);
  prefetch_l2(base + off + 64 * (part & 1));
}

// A warp's running softmax partial per query head over the tokens it
// corrected: frame m (log2 units, uniform over the lanes) and the lane's 4
// channels of acc; exact terms enter with +, the scan's approximate terms of
// the same tokens with -.  The scalars of (head, value group) are spread over
// the lanes: lane L keeps, for its pair (h, j) = ((L mod 4GP) / 4, L mod 4),
// the mass l of head h (used from the lanes with j = 0) and the sum of the
// removed zero-point terms of head h and group j (subtracted from the
// channels of group j at the end).
template <int G>
struct WarpPart {
  float m[G], acc[G][4], lsum, zsum;
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
    }
    lsum = zsum = 0.f;
  }
};

// Warp sum of V values per lane (V a power of two <= 32) by halving
// exchanges: afterwards x[0] of lane L holds the sum of value
// (L >> (5 - log2 V)) & (V - 1); 2V - 1 shuffles instead of 5V.
template <int V>
__device__ __forceinline__ void warp_sum_scatter(float (&x)[V], int lane) {
  int n = V;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < n / 2) {
          const float keep = up ? x[i + n / 2] : x[i];
          const float send = up ? x[i] : x[i + n / 2];
          x[i] = keep + __shfl_xor_sync(kAll, send, o);
        }
      }
      n >>= 1;
    } else {
      x[0] += __shfl_xor_sync(kAll, x[0], o);
    }
  }
}
template <int V>
constexpr int log2c() { return V <= 1 ? 0 : 1 + log2c<V / 2>(); }

// Correct tokens list[warp + kFinWarps * j], j = 0, 1, ... (n entries in
// the list) into the warp's partial WP, NC tokens at a time: record pieces
// by cp.async into the warp's ring and the lane's row channels into
// registers, all issued before the first is used; then (pass 1) every
// token's exact logits, (pass 2) one frame move per head for the chunk and the
// tokens' terms.
template <int G, int KB, int VB>
__device__ __forceinline__ void warp_correct(const FinishParams& p, int seg, const int32_t* list, int n,
                                             FinWork& FW, const float* qf, WarpPart<G>& WP) {
  constexpr int GP = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8;  // heads padded to a power of two
  constexpr int NC = G > 4 ? 2 : kChunk;                        // tokens per chunk
  constexpr int V = NC * GP;                                    // logits reduced together
  constexpr int VSH = 5 - log2c<V>();
  constexpr int NT = G > 4 ? 2 : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nj = n > warp ? (n - warp + kFinWarps - 1) / kFinWarps : 0;
  // the lane's channels: c = 4 lane + i, value group j = lane / 8; value-code
  // word of channel c in the staged pieces (see vc_loc): row gid_c, high
  // half chi of the channel m-tile mt
  const int mt = lane >> 2, chi = (lane & 3) >> 1, gbase = 4 * (lane & 1), vj = lane >> 3;
#pragma unroll 1
  for (int j0 = 0; j0 < nj; j0 += NC) {
    int tk[NC];
    uint2 kr[NC], vr[NC];
#pragma unroll
    for (int u = 0; u < NC; ++u) {
      const int j = j0 + u;
      tk[u] = j < nj ? list[warp + kFinWarps * j] : -1;
      if (tok_quant(tk[u])) {
        if (lane < kTokPieces16) stage_piece<KB, VB, NT>(p, seg, tk[u], FW.ring[warp][u], lane);
      }
      if (tk[u] != -1) {
        kr[u] = row4(p, seg, tk[u], false, lane);
        vr[u] = row4(p, seg, tk[u], true, lane);
      } else {
        kr[u] = vr[u] = make_uint2(0u, 0u);
      }
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    // ---- pass 1: exact logits
    float x[V];
#pragma unroll
    for (int u = 0; u < NC; ++u) {
      const float k0 = __uint_as_float(kr[u].x << 16), k1 = __uint_as_float(kr[u].x & 0xFFFF0000u);
      const float k2 = __uint_as_float(kr[u].y << 16), k3 = __uint_as_float(kr[u].y & 0xFFFF0000u);
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        if (h < G) {
          const float4 qv = *reinterpret_cast<const float4*>(qf + h * kD + 4 * lane);
          x[u * GP + h] = fmaf(qv.w, k3, fmaf(qv.z, k2, fmaf(qv.y, k1, qv.x * k0)));
        } else {
          x[u * GP + h] = 0.f;
        }
      }
    }
    warp_sum_scatter<V>(x, lane);
    // exact logit (log2 units) of value v = u * GP + h: lanes with v(L) = v
    auto se_of = [&](int u, int h) {
      return __shfl_sync(kAll, x[0], ((u * GP + h) << VSH)) * p.kappa;
    };
    float se[NC][G];
#pragma unroll
    for (int u = 0; u < NC; ++u)
#pragma unroll
      for (int h = 0; h < G; ++h) se[u][h] = se_of(u, h);
    // ---- pass 2: frame moves (the chunk's largest term per head), then terms
    const int pair = lane & (4 * GP - 1), ph = pair >> 2, pj = pair & 3;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float top = -INFINITY;
#pragma unroll
      for (int u = 0; u < NC; ++u) {
        if (tk[u] != -1) top = fmaxf(top, se[u][h]);
        if (tok_quant(tk[u])) top = fmaxf(top, FW.ring[warp][u].mu[h]);
      }
      if (top > WP.m[h] + 8.f) {  // move the frame (0 while the partial is empty)
        const float al = exp2f(WP.m[h] - top);
        WP.acc[h][0] *= al;
        WP.acc[h][1] *= al;
        WP.acc[h][2] *= al;
        WP.acc[h][3] *= al;
        if (ph == h) {
          WP.lsum *= al;
          WP.zsum *= al;
        }
        WP.m[h] = top;
      }
    }
    // the frame and logits of the lane's pair head ph
    float mph = WP.m[0];
#pragma unroll
    for (int h = 1; h < G; ++h) mph = ph == h ? WP.m[h] : mph;
    // every token of the chunk in straight-line code (an empty slot or a
    // tail token carries zero weights), so the tokens' chains interleave
#pragma unroll
    for (int u = 0; u < NC; ++u) {
      const int t = tk[u];
      const bool valid = t != -1, quant = tok_quant(t);
      const TokPieces& S = FW.ring[warp][u];
      const int tt = quant ? t % kKG : 0, hi8 = (tt & 15) >> 3, e = tt & 1;
      // pair scalars (head ph, value group pj): exact weight pe, and for a
      // quantized token the removed value weight A = f fp16(p s_v) and
      // zero-point term f p m_v, f = 2^(m_used - m) moving the scan's frame
      float seh = se[u][0];
#pragma unroll
      for (int h = 1; h < G; ++h) seh = ph == h ? se[u][h] : seh;
      const bool live = valid && ph < G, qlive = quant && ph < G;
      const float pe = live ? exp2f(seh - mph) : 0.f;
      const uint16_t pb = reinterpret_cast<const uint16_t*>(S.w)[2 * (4 * (ph >> 2) + (ph & 3)) + hi8];
      const float f = qlive ? exp2f(S.mu[ph < G ? ph : 0] - mph) : 0.f;
      const uint16_t vsc = *reinterpret_cast<const uint16_t*>(S.vsz + pj * 8 + hi8 * 4 + 2 * e);
      const float vz = h2f(*reinterpret_cast<const uint16_t*>(S.vsz + 32 + pj * 8 + hi8 * 4 + 2 * e));
      const float pw = qlive ? h2f(pb) : 0.f;
      const float A = qlive ? f * h2f(h_mul_rn(pb, vsc)) : 0.f;
      WP.zsum = qlive ? fmaf(f * pw, vz, WP.zsum) : WP.zsum;
      WP.lsum += fmaf(-f, pw, pe);
      const float v0 = __uint_as_float(vr[u].x << 16), v1 = __uint_as_float(vr[u].x & 0xFFFF0000u);
      const float v2 = __uint_as_float(vr[u].y << 16), v3 = __uint_as_float(vr[u].y & 0xFFFF0000u);
      // the value codes of the lane's channels (meaningless, and multiplied
      // by A = 0, unless the token is quantized)
      float code[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int gc = gbase + i;
        uint32_t wd, c;
        if (VB == 4) {
          const int w8 = 2 * (mt & 3) + hi8;
          wd = *reinterpret_cast<const uint32_t*>(S.vp + ((w8 >> 2) * 8 + gc) * 16 + (w8 & 3) * 4);
          c = (wd >> (vc_pos(4, mt) + 8 * chi + 16 * e)) & 15u;
        } else {
          wd = *reinterpret_cast<const uint32_t*>(S.vp + gc * 16 + (2 * (mt & 1) + hi8) * 4);
          c = (wd >> (vc_pos(2, mt) + 8 * chi + 16 * e)) & 3u;
        }
        code[i] = (float)c;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        // head h's scalars for the lane's value group vj: lane 4h + vj
        const float peh = __shfl_sync(kAll, pe, 4 * h + vj);
        const float Ah = __shfl_sync(kAll, A, 4 * h + vj);
        WP.acc[h][0] = fmaf(-Ah, code[0], fmaf(peh, v0, WP.acc[h][0]));
        WP.acc[h][1] = fmaf(-Ah, code[1], fmaf(peh, v1, WP.acc[h][1]));
        WP.acc[h][2] = fmaf(-Ah, code[2], fmaf(peh, v2, WP.acc[h][2]));
        WP.acc[h][3] = fmaf(-Ah, code[3], fmaf(peh, v3, WP.acc[h][3]));
      }
    }
    __syncwarp();  // the ring is reused by the next chunk
  }
}

template <int G, bool SELECT, int KB, int VB>
__global__ void __launch_bounds__(kFinThreads, 2) finish_kernel(const __grid_constant__ FinishParams p) {
  extern __shared__ __align__(16) uint8_t fsm[];
  FinPersist& PS = *reinterpret_cast<FinPersist*>(fsm);
  FinParts<G>& P = *reinterpret_cast<FinParts<G>*>(fsm + sizeof(FinPersist));
  float* qf = reinterpret_cast<float*>(fsm + sizeof(FinPersist) + sizeof(FinParts<G>));
  int32_t* tok = reinterpret_cast<int32_t*>(qf + G * kD);
  uint8_t* U = reinterpret_cast<uint8_t*>(tok + kTokCap + kTail);
  FinWork& FW = *reinterpret_cast<FinWork*>(U);
  FinMerge<G>& FM = *reinterpret_cast<FinMerge<G>*>(U);
  float* early = reinterpret_cast<float*>(U + fin_union_bytes<G>());
  __shared__ uint32_t scratch[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_tot;
  __shared__ uint32_t s_cnt[kFinMaxC], s_pre[kFinMaxC + 1], s_tpre[kFinMaxC + 1];
  __shared__ uint32_t s_chq[kFinMaxC + 1];  // chosen ties before slice q
  __shared__ int s_mode;                     // 0 lists in shared memory, 1 fallback lists
  __shared__ uint32_t s_hmax[kMaxG];          // per head: largest scan-partial maximum (key)
  __shared__ uint32_t s_tie[kFinMaxC], s_ovf[kFinMaxC];
  __shared__ __align__(8) uint64_t s_early_bar;  // completion of the early copy below

  cg::cluster_group cl = cg::this_cluster();
  // every CTA of the cluster has started once the matching wait returns:
  // only then may a CTA store into another's shared memory
  cluster_arrive_relaxed();
  const int C = (int)cl.num_blocks();
  const int r = (int)cl.block_rank();
  const int seg = blockIdx.x / C;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = p.k;
  const int bb = seg / p.hkv, hh = seg % p.hkv;
  // this sequence's quantized tokens, tail and groups, and this CTA's slice
  const int n_ctx = p.seq.n_ctx[bb];
  const int nq = split_point(n_ctx), tail = n_ctx - nq, ng = nq / kKG;
  const int slice = nq > 0 ? ((nq + C - 1) / C + 63) / 64 * 64 : 64;

  // ---- set-up: nothing here is written by the scan
  {  // this CTA's tail rows into L2 while the set-up runs
    const int n_mine = tail > r ? (tail - r + C - 1) / C : 0;
    for (int i = tid; i < n_mine * 4; i += kFinThreads)
      prefetch_part(p, seg, (1 << 30) | (r + C * (i >> 2)), i & 3);
  }
  for (int i = tid; i < G * kD; i += kFinThreads) {
    const uint16_t b = p.q[((size_t)bb * p.H + (size_t)hh * G) * kD + i];
    qf[i] = __uint_as_float((uint32_t)b << 16);
  }
  if (tid == 0) {  // initialised before any thread can wait on it
    mbar_init(&s_early_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  pdl_wait();
  pdl_launch_dependents();

  // ---- early copy of this CTA's share of the scan's split partials, every
  // head, when the rows fit (else they are staged a tile at a time below)
  long long w0 = 0, w1 = -1;
  if (ng > 0) {
    const long long T = p.scan_total, W = p.scan_warps;
    const long long x0 = (long long)p.seq.gpre[bb] + (long long)hh * ng, x1 = x0 + ng - 1;
    w0 = scan_warp_of(x0, W, T);
    w1 = scan_warp_of(x1, W, T);
  }
  const int ns = (int)(w1 - w0 + 1);  // one partial slot per scan warp of the segment
  const int s0 = (int)((long long)ns * r / C), s1 = (int)((long long)ns * (r + 1) / C);
  constexpr int kV = kPartStride / 4;  // float4 per row
  const int nrows = (s1 - s0) * G;
  constexpr int kEarlyRows = (int)(kEarlyBytes / (kPartStride * sizeof(float)));
  const bool early_ok = nrows <= kEarlyRows;
  // the rows (slot, head) are consecutive in the workspace: one bulk copy,
  // completing on an mbarrier (independent of the warps' cp.async groups)
  if (early_ok && nrows > 0 && tid == 0) {
    const uint32_t bytes = (uint32_t)(nrows * kPartStride * sizeof(float));
    mbar_expect_tx(&s_early_bar, bytes);
    bulk_g2s_nohint(early, p.scan_part + ((size_t)(w0 + s0 + seg) * G) * kPartStride, bytes, &s_early_bar);
  }

  const bool select = SELECT && k < nq;
  const int lo = min(nq, r * slice), hi = min(nq, lo + slice);
  const int R = p.hist_reps;
  const uint32_t* hg = p.hist + (size_t)seg * R * kScanHistStride;
  // the segment's largest selection key (the largest over the copies)
  uint32_t top_key = 0u;
  if (select)
    for (int c = 0; c < R; ++c) top_key = max(top_key, hg[(size_t)c * kScanHistStride + kScanHistBins]);

  WarpPart<G> WP;
  WP.init();

  // ---- S1 + S2: bin b* from the scan's histogram, then this slice's lists
  bool hist_ok = false;
  uint32_t base_s_out = 0, base_t_out = 0;  // the slice's sure and tie counts
  if (select) {
    // the slice's first 16 scores of this thread, loaded together with the
    // histogram window so both round trips overlap
    const float* S = p.scores + (size_t)seg * p.capacity;
    float4 v0[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b0 = lo + 16 * tid + 4 * u;
      v0[u] = b0 < hi ? *reinterpret_cast<const float4*>(S + b0) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // the bin holding the k-th largest key: a window of 1024 bins below the
    // segment's largest key (thread t owns 4 bins), then further windows
    // down while the keys counted so far are fewer than k
    const int top = (int)(top_key >> (32 - kScanHistBits));
    int whi = min(kScanHistBins, (top | 3) + 1);
    uint32_t above = 0;  // keys in the bins above the current window
#pragma unroll 1
    for (;;) {
      const int wlo = max(0, whi - 4 * kFinThreads);
      const int b0 = wlo + 4 * tid;
      uint4 hv = make_uint4(0u, 0u, 0u, 0u);
      if (b0 < whi) {
#pragma unroll 4
        for (int c = 0; c < R; ++c) {
          const uint4 h = *reinterpret_cast<const uint4*>(hg + (size_t)c * kScanHistStride + b0);
          hv.x += h.x;
          hv.y += h.y;
          hv.z += h.z;
          hv.w += h.w;
        }
      }
      if (tid == 0) s_bin = -1;
      uint32_t cum = above + block_suffix_excl(hv.x + hv.y + hv.z + hv.w, scratch);
      const uint32_t hb[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
      for (int i = 3; i >= 0; --i) {
        if (cum < (uint32_t)k && cum + hb[i] >= (uint32_t)k) {
          s_bin = b0 + i;
          s_above = cum;
        }
        cum += hb[i];
      }
      if (tid == 0) s_tot = cum;  // every key in the bins from wlo up
      __syncthreads();
      if (s_bin >= 0 || wlo == 0) break;
      above = s_tot;
      whi = wlo;
      __syncthreads();
    }
    // the lists below are checked against the counts the histogram promised,
    // so a histogram that does not match these scores only costs the fallback
    hist_ok = s_bin >= 0;
    const uint32_t bstar = (uint32_t)s_bin;
    uint32_t base_s = 0, base_t = 0;
    if (hist_ok) {
      for (int t0 = lo; t0 < hi; t0 += 16 * kFinThreads) {
        const int b0 = t0 + 16 * tid;
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[u] = t0 == lo ? v0[u]
                          : (b0 + 4 * u < hi ? *reinterpret_cast<const float4*>(S + b0 + 4 * u)
                                             : make_float4(0.f, 0.f, 0.f, 0.f));
        uint32_t keys[16];
        uint32_t ms = 0, mtie = 0, nsu = 0, nti = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * u + e;
            keys[i] = float_key(vals[e]);
            const bool in = b0 + i < hi;
            const uint32_t bin = keys[i] >> (32 - kScanHistBits);
            const bool su = in && bin > bstar, ti = in && bin == bstar;
            ms |= (su ? 1u : 0u) << i;
            mtie |= (ti ? 1u : 0u) << i;
            nsu += su;
            nti += ti;
          }
        }
        uint32_t tot;
        const uint32_t pos = block_prefix_excl((nsu << 16) | nti, scratch, &tot);
        uint32_t ps = base_s + (pos >> 16), pt = base_t + (pos & 0xFFFFu);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (ms & (1u << i)) {
            if (ps < (uint32_t)kLCap) PS.sure[ps] = (uint32_t)(b0 + i);
            ++ps;
          }
          if (mtie & (1u << i)) {
            if (pt < (uint32_t)kLCap) {
              PS.tkey[pt] = keys[i];
              PS.tidx[pt] = (uint32_t)(b0 + i);
            }
            ++pt;
          }
        }
        base_s += tot >> 16;
        base_t += tot & 0xFFFFu;
      }
    }
    base_s_out = base_s;
    base_t_out = base_t;
    if (tid == 0) {
      PS.n_sure = base_s;
      PS.n_tie = base_t;
      PS.overflow = (base_s > (uint32_t)kLCap || base_t > (uint32_t)kLCap) ? 1u : 0u;
    }
  }
  cluster_wait();  // every CTA of the cluster has started
  if (select && tid == 0) {
    // this slice's counts into every CTA's shared memory (read after the
    // barrier below)
    const uint32_t ovf = (base_s_out > (uint32_t)kLCap || base_t_out > (uint32_t)kLCap) ? 1u : 0u;
    for (int q = 0; q < C; ++q) {
      cl.map_shared_rank(s_cnt, q)[r] = base_s_out;
      cl.map_shared_rank(s_tie, q)[r] = base_t_out;
      cl.map_shared_rank(s_ovf, q)[r] = ovf;
    }
  }

  // ---- M: this CTA's share of the scan's split partials: per head the
  // largest partial maximum M first, then every row's terms scaled by
  // 2^(m_row - M) and summed; rows from the early copy, else staged a tile
  // at a time; thread (channel, half) takes heads j = half, half + 2, ...
  {
    const int c = tid & (kD - 1), half = tid >> 7;
    constexpr int kH2 = (G + 1) / 2;
    if (tid < G) s_hmax[tid] = 0u;  // key of -inf and below
    if (early_ok && nrows > 0 && !mbar_wait_bounded(&s_early_bar, 0u)) {
      if (tid == 0) set_flag(p.flag, JFA_DEVERR_TIMEOUT);
      mbar_wait_bounded(&s_early_bar, 0u);  // the copy in flight, once more (bounded)
    }
    __syncthreads();
    for (int gr = tid; gr < nrows; gr += kFinThreads) {
      float m, l;
      if (early_ok) {
        m = early[gr * kPartStride];
        l = early[gr * kPartStride + 1];
      } else {
        const float* src = p.scan_part + ((size_t)(w0 + s0 + gr / G + seg) * G + gr % G) * kPartStride;
        m = src[0];
        l = src[1];
      }
      if (l > 0.f) atomicMax(&s_hmax[gr % G], float_key(m));
    }
    __syncthreads();
    float mh[kH2], lrun[kH2], arun[kH2];
#pragma unroll
    for (int i = 0; i < kH2; ++i) {
      const int j = half + 2 * i;
      mh[i] = j < G && s_hmax[j] != 0u ? key_float(s_hmax[j]) : -INFINITY;
      lrun[i] = 0.f;
      arun[i] = 0.f;
    }
    float* tile = reinterpret_cast<float*>(U);  // the correction's buffers are not in use yet
    constexpr int kTR = (int)(fin_union_bytes<G>() / (kPartStride * sizeof(float))) / kMaxG * kMaxG;
    __syncthreads();
    for (int r0 = 0; r0 < nrows; r0 += (early_ok ? nrows : kTR)) {
      const int nr = early_ok ? nrows : min(kTR, nrows - r0);
      if (early_ok) {
        tile = early;
      } else {
#pragma unroll 8
        for (int i = tid; i < nr * kV; i += kFinThreads) {
          const int row = i / kV, v = i % kV;
          const int gr = r0 + row;
          const float* src = p.scan_part + ((size_t)(w0 + s0 + gr / G + seg) * G + gr % G) * kPartStride;
          reinterpret_cast<float4*>(tile + row * kPartStride)[v] = *reinterpret_cast<const float4*>(src + 4 * v);
        }
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < kH2; ++i) {
        const int j = half + 2 * i;
        if (j < G) {
#pragma unroll 4
          for (int row = (j - r0 % G + G) % G; row < nr; row += G) {
            const float* tr = tile + row * kPartStride;
            const float rl = tr[1];
            const float f = rl > 0.f ? exp2f(tr[0] - mh[i]) : 0.f;
            lrun[i] = fmaf(rl, f, lrun[i]);
            arun[i] = fmaf(tr[4 + c], f, arun[i]);
          }
        }
      }
      if (!early_ok) __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kH2; ++i) {
      const int j = half + 2 * i;
      if (j < G) {
        P.sp[j][4 + c] = arun[i];
        if (c == 0) {
          P.sp[j][0] = lrun[i] > 0.f ? mh[i] : -INFINITY;
          P.sp[j][1] = lrun[i];
        }
      }
    }
  }

  if (select) cl.sync();  // every CTA's lists and counts are complete

  // ---- S3: resolve the selection; every CTA learns the whole chosen set:
  // the CTAs' sure lists (in CTA order) and the chosen ties (ascending)
  uint32_t n_ch = 0;
  const uint32_t* glist_base = p.glists + (size_t)seg * p.gl_stride;
  int mode = 0;
  if (select) {
    {  // the scan's histogram is consumed: clear it for the next scan
      uint32_t* hc = p.hist + (size_t)seg * R * kScanHistStride;
      for (int i = 4 * (r * kFinThreads + tid); i < R * kScanHistStride; i += 4 * C * kFinThreads)
        *reinterpret_cast<uint4*>(hc + i) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid == 0) {
      uint32_t ps = 0, pt = 0, ovf = 0;
      for (int q = 0; q < C; ++q) {
        s_pre[q] = ps;
        s_tpre[q] = pt;
        ps += s_cnt[q];
        pt += s_tie[q];
        ovf |= s_ovf[q];
      }
      s_pre[C] = ps;
      s_tpre[C] = pt;
      // the ties must hold the k-th key: 1 <= k - (keys above b*) <= ties
      const bool consistent = ps < (uint32_t)k && (uint32_t)k - ps <= pt;
      s_mode = (!hist_ok || ovf || pt > (uint32_t)kTCap || !consistent) ? 1 : 0;
    }
    __syncthreads();
    mode = s_mode;
    if (mode == 0) {
      // every CTA's ties in one pass (all remote loads in flight together)
      for (uint32_t i = tid; i < s_tpre[C]; i += kFinThreads) {
        int q = 0;
        while (q + 1 < C && s_tpre[q + 1] <= i) ++q;
        const FinPersist* o = cl.map_shared_rank(&PS, q);
        FW.akey[i] = o->tkey[i - s_tpre[q]];
        FW.aidx[i] = o->tidx[i - s_tpre[q]];
      }
      __syncthreads();
      n_ch = (uint32_t)k - s_pre[C];
      const uint32_t T = s_tpre[C];
      if (T <= (uint32_t)kFinThreads) {
        // direct ranking: entry i is chosen iff fewer than n_ch entries come
        // before it in (key descending, index ascending) order; tpe threads
        // (a power of two) share an entry's comparisons
        uint32_t tpe = 1;
        while (tpe < 32 && tpe * 2 * T <= (uint32_t)kFinThreads) tpe *= 2;
        const uint32_t e = tid / tpe, part = tid % tpe;
        uint32_t rank = 0, my_idx = 0;
        if (e < T) {
          const uint32_t key = FW.akey[e];
          my_idx = FW.aidx[e];
#pragma unroll 4
          for (uint32_t j = part; j < T; j += tpe) {
            const uint32_t k2 = FW.akey[j];
            rank += (k2 > key || (k2 == key && FW.aidx[j] < my_idx)) ? 1u : 0u;
          }
        }
        for (uint32_t o = 1; o < tpe; o <<= 1) rank += __shfl_xor_sync(kAll, rank, o);
        const uint32_t chosen = (e < T && part == 0 && rank < n_ch) ? 1u : 0u;
        uint32_t tot;
        const uint32_t pos = block_prefix_excl(chosen, scratch, &tot);
        if (chosen) PS.chtie[pos] = my_idx;  // entries are in index order
        __syncthreads();
      } else {
        refine_ties(FW.akey, FW.aidx, T, n_ch, FW.hist, PS.chtie, scratch, &s_bin, &s_above,
                    &s_tot);
      }
      if (tid <= C) {
        const uint32_t b0 = (uint32_t)min(nq, tid * slice);
        s_chq[tid] = lower_bound_u32(PS.chtie, n_ch, b0);
      }
      __syncthreads();
    } else {
      // fallback: select over the whole segment; each CTA lists its slice's
      // chosen indices in global memory
      uint32_t* gl = const_cast<uint32_t*>(glist_base) + (size_t)r * slice;
      const uint32_t n = select_full(p.scores + (size_t)seg * p.capacity, nq, k, lo, hi, FW.hist, gl,
                                     scratch, &s_bin, &s_above, &s_tot);
      if (tid == 0) PS.n_gl = n;
      __threadfence();
      cl.sync();  // the fallback lists and counts are complete
      if (tid < C) s_cnt[tid] = cl.map_shared_rank(&PS, tid)->n_gl;
      __syncthreads();
      if (tid == 0) {
        uint32_t ps = 0;
        for (int q = 0; q < C; ++q) {
          s_pre[q] = ps;
          ps += s_cnt[q];
        }
        s_pre[C] = ps;
      }
      __syncthreads();
    }
  }

  // ---- C: the tail slots r, r + C, ... and an even share of the chosen set
  // (positions [x0, x1) of: the CTAs' lists in CTA order, then the chosen
  // ties), or of a given index set, or of every quantized token when
  // k >= N_q
  {
    const int n_x = select ? k : (SELECT ? nq : k);
    const int per = (n_x + C - 1) / C;
    const int x0 = min(n_x, r * per), x1 = min(n_x, x0 + per);
    const int n_tail = tail > r ? (tail - r + C - 1) / C : 0;
#pragma unroll 1
    for (int xr = x0, first = 1; first || xr < x1; xr += kTokCap, first = 0) {
      const int xe = min(x1, xr + kTokCap);
      uint32_t base = 0;
      if (first) {
        for (int i = tid; i < n_tail; i += kFinThreads) {
          const int t = (1 << 30) | (r + C * i);
          tok[i] = t;
        }
        base = (uint32_t)n_tail;
      }
      if (select) {  // every position holds a chosen token: no compaction
        for (int j = xr + tid; j < xe; j += kFinThreads) {
          int t;
          if ((uint32_t)j < s_pre[C]) {
            int q = 0;
            while (q + 1 < C && s_pre[q + 1] <= (uint32_t)j) ++q;
            t = (int)(mode == 1 ? glist_base[(size_t)q * slice + (j - s_pre[q])]
                                : cl.map_shared_rank(PS.sure, q)[j - s_pre[q]]);
          } else {
            t = (int)PS.chtie[j - s_pre[C]];
          }
          tok[base + (j - xr)] = t;
        }
        base += (uint32_t)(xe - xr);
      }
#pragma unroll 1
      for (int xb = xr; !select && xb < xe; xb += kFinThreads) {
        const int j = xb + tid;
        int t = -1;
        if (j < xe) {
          if (SELECT) {
            t = j;
          } else {
            t = p.idx_in[(size_t)seg * k + j];
            if (t < -1 || t >= nq) {
              set_flag(p.flag, JFA_DEVERR_BAD_INDEX);
              t = -1;
            }
          }
        }
        uint32_t tot;
        const uint32_t pos = base + block_prefix_excl(t >= 0 ? 1u : 0u, scratch, &tot);
        if (t >= 0) tok[pos] = t;
        base += tot;
      }
      __syncthreads();
      warp_correct<G, KB, VB>(p, seg, tok, (int)base, FW, qf, WP);
      __syncthreads();
    }
  }

  // ---- idx output: this CTA's chosen indices, ascending, at its offset
  if (select) {
    const uint32_t c0 = mode == 0 ? s_chq[r] : 0u, c1 = mode == 0 ? s_chq[r + 1] : 0u;
    const uint32_t off = s_pre[r] + c0;  // earlier slices: their lists and chosen ties
    const uint32_t* Lr = mode == 1 ? glist_base + (size_t)r * slice : PS.sure;
    const uint32_t nr = s_cnt[r];
    int32_t* out = p.idx_out + (size_t)seg * k;
    for (uint32_t i = tid; i < nr; i += kFinThreads) {
      const uint32_t v = Lr[i];
      const uint32_t pos = off + i + lower_bound_u32(PS.chtie + c0, c1 - c0, v);
      if (pos < (uint32_t)k) out[pos] = (int32_t)v;
    }
    for (uint32_t j = c0 + tid; j < c1; j += kFinThreads) {
      const uint32_t v = PS.chtie[j];
      const uint32_t pos = off + (j - c0) + lower_bound_u32(Lr, nr, v);
      if (pos < (uint32_t)k) out[pos] = (int32_t)v;
    }
  } else if (SELECT && r == 0) {
    int32_t* out = p.idx_out + (size_t)seg * k;
    for (int i = tid; i < k; i += kFinThreads) out[i] = i < nq ? i : -1;
  }
  if (!select) {  // nothing reads the scan's histogram here: clear it
    uint32_t* hz = p.hist + (size_t)seg * R * kScanHistStride;
    for (int i = 4 * (r * kFinThreads + tid); i < R * kScanHistStride; i += 4 * C * kFinThreads)
      *reinterpret_cast<uint4*>(hz + i) = make_uint4(0u, 0u, 0u, 0u);
  }

  // ---- M1: this CTA's partial per head (the warps' exact-minus-removed
  // terms, largest frame first, then every warp's terms scaled to it,
  // together with the CTA's share of the scan's partials), stored straight
  // into the shared memory of the head's owner, so that the merge after the
  // barrier reads only local memory
  __syncthreads();  // the correction's shared memory is free
#pragma unroll
  for (int h = 0; h < G; ++h) {
    // head h's mass from lane 4h, its zero-point sum of group j from lane 4h + j
    const float lh = __shfl_sync(kAll, WP.lsum, 4 * h);
    const float zh = __shfl_sync(kAll, WP.zsum, 4 * h + (lane >> 3));
    float* wrow = FM.w[warp][h];
    if (lane == 0) {
      wrow[0] = WP.m[h];
      wrow[1] = lh;
    }
    *reinterpret_cast<float4*>(wrow + 4 + 4 * lane) =
        make_float4(WP.acc[h][0] - zh, WP.acc[h][1] - zh, WP.acc[h][2] - zh, WP.acc[h][3] - zh);
  }
  __syncthreads();
  {
    const int c = tid & (kD - 1), half = tid >> 7;
    for (int h = half; h < G; h += 2) {
      float m = -INFINITY;
#pragma unroll
      for (int w = 0; w < kFinWarps; ++w) m = fmaxf(m, FM.w[w][h][0]);
      float l = 0.f, a = 0.f;
#pragma unroll
      for (int w = 0; w < kFinWarps; ++w) {
        const float f = FM.w[w][h][0] == -INFINITY ? 0.f : exp2f(FM.w[w][h][0] - m);
        l = fmaf(FM.w[w][h][1], f, l);
        a = fmaf(FM.w[w][h][4 + c], f, a);
      }
      // with the scan partials' share (m_a, l_a, a_a) in one frame; an empty
      // part (no tokens, or l_a = 0) has weight 0
      const float ma = P.sp[h][0], la = P.sp[h][1];
      const float mt = la > 0.f ? fmaxf(m, ma) : m;
      const float fc = m == -INFINITY ? 0.f : exp2f(m - mt);
      const float fa = la > 0.f ? exp2f(ma - mt) : 0.f;
      float* dst = cl.map_shared_rank(&P.recv[(h / C) * C + r][0], h % C);
      dst[4 + c] = fmaf(a, fc, P.sp[h][4 + c] * fa);
      if (c == 0) {
        dst[0] = mt;
        dst[1] = fmaf(l, fc, la * fa);
      }
    }
  }

  cl.sync();  // every CTA's partials are in their owners' shared memory

  // ---- M3: CTA r owns heads j = r, r + C, ...: merge the C partials (m_q,
  // l_q, a_q) of head j and write out = sum a_q 2^(m_q-M) / sum l_q 2^(m_q-M),
  // M the largest m_q.  Only local memory is read from here on, so no CTA
  // waits for the others before it exits.
  for (int j = r; j < G; j += C) {
    const int c = tid;
    if (c < kD) {
      const float* base = &P.recv[(j / C) * C][0];
      float M = -INFINITY;
#pragma unroll 4
      for (int q = 0; q < C; ++q) M = fmaxf(M, base[q * kPartStride]);
      float l = 0.f, acc = 0.f;
#pragma unroll 4
      for (int q = 0; q < C; ++q) {
        const float mq = base[q * kPartStride];
        const float f = mq == -INFINITY ? 0.f : exp2f(mq - M);
        l = fmaf(base[q * kPartStride + 1], f, l);
        acc = fmaf(base[q * kPartStride + 4 + c], f, acc);
      }
      p.out[((size_t)bb * p.H + hh * G + j) * kD + c] = acc / l;
    }
  }
}

template <int G, bool SEL, int KB, int VB>
static int pick_cluster(int n_seg, int max_c, int num_sms) {
  constexpr size_t smem = fin_smem_bytes<G>();
  int best = 1;
  for (int c = 2; c <= max_c; c *= 2) {
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
    if (cudaOccupancyMaxActiveClusters(&n_active, finish_kernel<G, SEL, KB, VB>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      break;
    }
    if (n_active >= n_seg) best = c;
    else break;
  }
  return best;
}

template <int G, bool SEL, int KB, int VB>
static int launch_finish_t(const FinishParams& fp, int n_seg, int nq_max, cudaStream_t st) {
  constexpr size_t smem = fin_smem_bytes<G>();
  static bool configured[64] = {false};
  static int memo_seg[64][8] = {{0}}, memo_c[64][8] = {{0}};  // cluster size per (device, key)
  static std::mutex mu;  // host threads launching on one device share the tables
  std::lock_guard<std::mutex> lock(mu);
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(finish_kernel<G, SEL, KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return JFA_ERR_CUDA;
    // clusters of 16 (beyond the portable 8) for workloads with few segments;
    // if the device refuses, the occupancy query below keeps clusters <= 8
    if (cudaFuncSetAttribute(finish_kernel<G, SEL, KB, VB>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1) != cudaSuccess)
      cudaGetLastError();
    configured[dev] = true;
  }
  // clusters of 16 pay off once the slices are long (measured: 32K-token
  // segments gain, 8K ones lose); memoized per (segments, cap)
  const int max_c = nq_max >= 16384 ? kFinMaxC : 8;
  const int key = n_seg * 2 + (max_c > 8 ? 1 : 0);
  int C = 0;
  if (dev >= 0 && dev < 64) {
    for (int i = 0; i < 8; ++i)
      if (memo_seg[dev][i] == key) C = memo_c[dev][i];
  }
  if (C == 0) {
    C = pick_cluster<G, SEL, KB, VB>(n_seg, max_c, num_sms_current());
    if (dev >= 0 && dev < 64) {
      for (int i = 0; i < 8; ++i)
        if (memo_seg[dev][i] == 0) {
          memo_seg[dev][i] = key;
          memo_c[dev][i] = C;
          break;
        }
    }
  }
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
  return cudaLaunchKernelEx(&cfg, finish_kernel<G, SEL, KB, VB>, fp) == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

template <bool SEL, int KB, int VB>
static int launch_finish_g(const FinishParams& fp, int G, int n_seg, int nq_max, cudaStream_t st) {
  switch (G) {
    case 1: return launch_finish_t<1, SEL, KB, VB>(fp, n_seg, nq_max, st);
    case 2: return launch_finish_t<2, SEL, KB, VB>(fp, n_seg, nq_max, st);
    case 3: return launch_finish_t<3, SEL, KB, VB>(fp, n_seg, nq_max, st);
    case 4: return launch_finish_t<4, SEL, KB, VB>(fp, n_seg, nq_max, st);
    case 5: return launch_finish_t<5, SEL, KB, VB>(fp, n_seg, nq_max, st);
    case 6: return launch_finish_t<6, SEL, KB, VB>(fp, n_seg, nq_max, st);
    case 7: return launch_finish_t<7, SEL, KB, VB>(fp, n_seg, nq_max, st);
    default: return launch_finish_t<8, SEL, KB, VB>(fp, n_seg, nq_max, st);
  }
}

}  // namespace jfa

// finish.cu — everything after the scan in one kernel.  A thread-block
// cluster of C CTAs (C <= 8) per (sequence, KV head):
//   T   (before waiting for the scan) corrects its share of the bf16 tail;
//   P1  reads the scan's 8192-bin histogram of the selection keys and finds
//       the bin b* holding the k-th largest key (every CTA, redundantly);
//   P2  lists its slice's keys above b* ("sure") and in b* ("ties"), in
//       index order, in its shared memory;
//   P3  after a cluster barrier, gathers every CTA's ties and resolves the
//       k-th key inside b* by two more radix levels (ties to lower indices),
//       writes its own chosen indices to idx in ascending order and takes
//       an even share of the chosen set for the correction;
//   P4  corrects that share: exact bf16 logits and values, and the scan's
//       approximate terms of each chosen token recomputed bit for bit
//       (jfa_approx.cuh, with the stored running maxima) for removal;
//   P5  merges a share of the scan's split partials, then the CTAs owning a
//       query head combine scan, exact and removal partials of all C CTAs
//       (distributed shared memory) in log-sum-exp form.
// With a given index set (jfa_correct_merge) P1-P3 are skipped.  If the
// histogram is stale or the candidates overflow shared memory, every CTA
// selects over the whole segment instead (slower, same result).
#include <cooperative_groups.h>

#include "jfa_approx.cuh"
#include "jfa_blocks.cuh"

namespace cg = cooperative_groups;

namespace jfa {

constexpr int kFinThreads = 256;
constexpr int kFinMaxC = 8;
constexpr int kLCap = 1024;   // sure / tie list entries per CTA
constexpr int kTCap = 1024;   // gathered tie entries
constexpr int kRefBins = 2048;
constexpr int kWD = 3;        // cp.async stages per warp (tokens in flight)
constexpr int kFinWarps = kFinThreads / 32;

struct FinishParams {
  const uint8_t* groups;
  const uint16_t* tail_k;
  const uint16_t* tail_v;
  const uint16_t* k_exact;
  const uint16_t* v_exact;
  const uint16_t* q;
  const float* scores;     // [n_seg][capacity]
  const float* scan_part;  // per scan warp and segment: [slot][G][kPartStride]
  const float* m_used;     // [n_seg][ng_cap][16]: the scan's running maxima and biases
  uint32_t* hist;          // [n_seg][kScanHistBins], zeroed here after use
  uint32_t* glists;        // [n_seg][C][slice] chosen lists of the fallback
  const int32_t* idx_in;   // given index sets (no selection), [n_seg][k]
  int32_t* idx_out;        // [n_seg][k] (selection)
  float* out;
  uint32_t* flag;
  int k, nq, tail, capacity, ng_cap, hkv, H, key_bits, val_bits, rec_bytes, ng, slice;
  long long scan_total;
  int scan_warps;
  float kappa;
};

// Shared memory.  The persistent part is read by other CTAs of the cluster
// (lists, counts, partials) and lives until the last barrier; the union part
// is private and reused: selection buffers, then the correction's token list
// and per-warp staging rings.
struct FinPersist {
  uint32_t sure[kLCap];               // chosen-for-sure indices of the slice, ascending
  uint32_t tkey[kLCap], tidx[kLCap];  // ties of the slice (key, index), ascending index
  uint32_t chtie[kTCap];              // chosen ties of the whole segment, ascending
  uint32_t n_sure, n_tie, overflow, n_gl;
};
// A correction partial (m, l, pad, pad, acc[128]) per query head; in the
// combined form the top-k tokens' approximate terms enter with a minus sign,
// so l may be negative.
template <int G>
struct FinParts {
  float qs[G][kD];
  float run[G][kPartStride];   // this CTA's exact-minus-removed partial
  float sp[G][kPartStride];    // this CTA's share of the scan partials
  float wp[kFinWarps][G][kPartStride];  // per-warp partials
};
// Shared-memory histograms store bin b at hpad(b) = b + b/32, so threads
// that each read a contiguous run of bins hit distinct banks.
__device__ __forceinline__ int hpad(int b) { return b + (b >> 5); }
struct FinSelect {
  uint32_t hist[kRefBins + kRefBins / 32];
  uint32_t akey[kTCap], aidx[kTCap];
};
// Record pieces of one quantized token, staged by cp.async.
struct WStage {
  uint8_t ksz[512];    // key scales / zeros of its group
  uint8_t kcode[1024]; // key codes of its 16-token m-tile, in lane order
  uint8_t vp[256];     // value-code pieces holding its column (8 or 16 x 16 B)
  uint8_t vsz[64];     // its value scales (32 B block) and zeros (32 B block)
  float mu[2 * kMaxG]; // the scan's running maxima (8) and biases (8) of its group
};
constexpr int kTokCap = 1024;  // tokens listed per correction round
struct FinCorr {
  WStage st[kFinWarps][kWD];
  int32_t tok[kTokCap];
};
template <int G>
constexpr size_t fin_smem_bytes() {
  return sizeof(FinPersist) + sizeof(FinParts<G>) +
         (sizeof(FinSelect) > sizeof(FinCorr) ? sizeof(FinSelect) : sizeof(FinCorr));
}

// Block-wide maximum of a float (all threads get it).
__device__ __forceinline__ float block_max(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kAll, v, o));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float m = scratch[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, scratch[w]);
  __syncthreads();
  return m;
}

// From bin counts h[hpad(0..nbins)) (nbins a multiple of blockDim) find the
// bin where the count taken from the top reaches r (1 <= r); *bin = -1 if
// the total < r.
__device__ __noinline__ void find_bin_from_top(const uint32_t* h, int nbins, uint32_t r, uint32_t* scratch,
                                  int* bin, uint32_t* above, uint32_t* total) {
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

// Selection inside the histogram bin b* (keys share their top 13 bits):
// the r largest of the T ties akey/aidx (index order), larger key first and
// equal keys to the lower index, two radix levels (11 + 8 bits) and one
// ordered pass.  Writes the chosen indices ascending to chosen[] (r of them).
__device__ __noinline__ void refine_ties(const uint32_t* akey, const uint32_t* aidx, uint32_t T, uint32_t r,
                            uint32_t* h, uint32_t* chosen, uint32_t* scratch, int* s_bin,
                            uint32_t* s_above, uint32_t* s_tot) {
  const int tid = threadIdx.x;
  // level 2: key bits 18..8
  for (int i = tid; i < hpad(kRefBins); i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < T; i += blockDim.x) atomicAdd(&h[hpad((akey[i] >> 8) & 2047u)], 1u);
  __syncthreads();
  find_bin_from_top(h, kRefBins, r, scratch, s_bin, s_above, s_tot);
  const uint32_t d2 = (uint32_t)*s_bin;
  const uint32_t r2 = r - *s_above;
  __syncthreads();
  // level 3: key bits 7..0 among keys whose bits 18..8 are d2
  for (int i = tid; i < hpad(256); i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < T; i += blockDim.x)
    if (((akey[i] >> 8) & 2047u) == d2) atomicAdd(&h[hpad(akey[i] & 255u)], 1u);
  __syncthreads();
  find_bin_from_top(h, 256, r2, scratch, s_bin, s_above, s_tot);
  const uint32_t low = (akey[0] >> 19) << 19;  // the shared top bits
  const uint32_t kstar = low | (d2 << 8) | (uint32_t)*s_bin;
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
__device__ __noinline__ uint32_t select_full(const float* S, int nq, int k, int lo, int hi, uint32_t* h,
                                uint32_t* out, uint32_t* scratch, int* s_bin, uint32_t* s_above,
                                uint32_t* s_tot) {
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
// Correction, a warp per token.  Token encoding: t in [0, nq) a quantized
// token, (1 << 30) | s the tail slot s.  Lane l owns channels 4l..4l+3 of
// every head.  The quantized token's record pieces are staged by cp.async
// kWD tokens ahead; its exact bf16 row is loaded one token ahead.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool tok_quant(int t) { return t >= 0 && !(t & (1 << 30)); }

template <typename T4>
__device__ __forceinline__ T4 ld16(const void* p) {
  return *reinterpret_cast<const T4*>(p);
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Stage the record pieces of token t (one commit group per lane, possibly empty).
__device__ __forceinline__ void stage_issue(const FinishParams& p, int seg, int t, WStage& S,
                                            int lane) {
  if (tok_quant(t)) {
    const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + (size_t)(t / kKG)) * p.rec_bytes;
    const int tt = t % kKG, kk = tt >> 4, tgt = (tt & 7) >> 1;
    cp_async16(S.ksz + lane * 16, rec + lane * 16);
    if (p.key_bits == 4) {
      const uint8_t* src = rec + off_kc() + kk * 1024 + lane * 32;
      cp_async16(S.kcode + lane * 32, src);
      cp_async16(S.kcode + lane * 32 + 16, src + 16);
    } else {
      const uint8_t* src = rec + off_kc() + kk * 768 + lane * 24;
      cp_async8(S.kcode + lane * 24, src);
      cp_async8(S.kcode + lane * 24 + 8, src + 8);
      cp_async8(S.kcode + lane * 24 + 16, src + 16);
    }
    const int vslots = p.val_bits == 4 ? 16 : 8;
    if (lane < vslots) {
      const int chunk = p.val_bits == 4 ? 2 * kk + (lane >> 3) : kk;
      cp_async16(S.vp + lane * 16, rec + off_vc(p.key_bits) + chunk * 512 + ((lane & 7) * 4 + tgt) * 16);
    }
    if (lane < 4)
      cp_async16(S.vsz + lane * 16,
                 rec + off_vs(p.key_bits) + kk * 128 + tgt * 32 + (lane & 1) * 16 + (lane >> 1) * 512);
    if (lane < 4)
      cp_async16(reinterpret_cast<uint8_t*>(S.mu) + lane * 16,
                 p.m_used + ((size_t)seg * p.ng_cap + (size_t)(t / kKG)) * (2 * kMaxG) + lane * 4);
  }
  cp_async_commit();
}

// Exact bf16 row pieces of token t for lane l: channels 4l..4l+3 of K and V.
__device__ __forceinline__ void row_load(const FinishParams& p, int seg, int t, int lane, uint2& kr,
                                         uint2& vr) {
  const size_t off = (t & (1 << 30)) ? ((size_t)seg * kTail + (t & 0xFFFF)) * kD
                                     : ((size_t)seg * p.capacity + t) * kD;
  const uint16_t* kb = (t & (1 << 30)) ? p.tail_k : p.k_exact;
  const uint16_t* vb = (t & (1 << 30)) ? p.tail_v : p.v_exact;
  kr = *reinterpret_cast<const uint2*>(kb + off + 4 * lane);
  vr = *reinterpret_cast<const uint2*>(vb + off + 4 * lane);
}

// L2 prefetch of one of the 27 128-byte pieces token t's correction
// reads: its bf16 K and V rows, and for a quantized token its group's key
// scales/zeros, its m-tile's key codes, the value-code chunk(s) of its column,
// its value scales/zeros and the stored running maxima.
__device__ __forceinline__ void prefetch_part(const FinishParams& p, int seg, int t, int part) {
  const bool tail = (t & (1 << 30)) != 0;
  if (part < 4) {
    const size_t off = tail ? ((size_t)seg * kTail + (t & 0xFFFF)) * kD : ((size_t)seg * p.capacity + t) * kD;
    const uint16_t* base = (part & 2) ? (tail ? p.tail_v : p.v_exact) : (tail ? p.tail_k : p.k_exact);
    prefetch_l2(base + off + 64 * (part & 1));
    return;
  }
  if (tail) return;
  const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + (size_t)(t / kKG)) * p.rec_bytes;
  const int tt = t % kKG, kk = tt >> 4, tgt = (tt & 7) >> 1;
  if (part < 8) {
    prefetch_l2(rec + 128 * (part - 4));
  } else if (part < 16) {
    const int i = part - 8, mbytes = p.key_bits == 4 ? 1024 : 768;
    if (128 * i < mbytes) prefetch_l2(rec + off_kc() + kk * mbytes + 128 * i);
  } else if (part < 24) {
    const int i = part - 16;
    if (p.val_bits == 4 || i < 4)
      prefetch_l2(rec + off_vc(p.key_bits) + (p.val_bits == 4 ? 2 * kk : kk) * 512 + 128 * i);
  } else if (part < 26) {
    prefetch_l2(rec + off_vs(p.key_bits) + kk * 128 + tgt * 32 + 512 * (part - 24));
  } else {
    prefetch_l2(p.m_used + ((size_t)seg * p.ng_cap + (size_t)(t / kKG)) * (2 * kMaxG));
  }
}

// The scan's fp16 weights of quantized token t for every head, recomputed
// from its staged group pieces with the scan's own functions on the same
// operands (key_sz, scale_pos, q_tilde_col, key_afrag, qk_chain, approx_logit,
// approx_weight; the group bias as the scan stored it); ph[j] = fp16 bits of
// head j's weight, on all lanes.  q2[n]: the lane's q of head (gid >> 1) + 4n, as the scan holds it.
template <int KB, int G>
__device__ __forceinline__ void replay_weights_t(const FinishParams& p, int t, const WStage& S,
                                                 const uint32_t (&q2)[2][16], int lane,
                                                 uint32_t ph[G]) {
  constexpr int NT = G > 4 ? 2 : 1;
  const int gid = lane >> 2, tig = lane & 3;
  const int tt = t % kKG, row = tt & 7, rr = (tt >> 3) & 1;
  uint32_t sk[16], zk[16], sf[16], qb[NT][16];
  float bk[NT];
  key_sz(S.ksz, tig, sk, zk);
  // the group bias of head tig + 4n exactly as the scan computed and stored it
#pragma unroll
  for (int n = 0; n < NT; ++n) bk[n] = S.mu[kMaxG + (tig + 4 * n < G ? tig + 4 * n : 0)];
  scale_pos<KB>(sk, sf);
#pragma unroll
  for (int n = 0; n < NT; ++n) q_tilde_col(q2[n], sf, (gid & 1) != 0, qb[n]);
  uint32_t w[KeyPos<KB>::WORDS];
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(S.kcode + lane * 4 * KeyPos<KB>::WORDS);
#pragma unroll
  for (int i = 0; i < KeyPos<KB>::WORDS; ++i) w[i] = kw[i];
  uint32_t a[16][2];
  key_afrag<KB>(w, a);
  const float kappa_u = p.kappa * KeyPos<KB>::unscale;
  uint32_t mine[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float d[4];
    qk_chain(a, qb[n], d);
    const int h = tig + 4 * n;
    mine[n] = (gid == row && h < G)
                  ? f2h_rn(approx_weight(approx_logit(d, rr, kappa_u, bk[n]), S.mu[h]))
                  : 0u;
  }
#pragma unroll
  for (int j = 0; j < G; ++j) ph[j] = __shfl_sync(kAll, mine[j >> 2], row * 4 + (j & 3));
}
template <int G>
__device__ __forceinline__ void replay_weights(const FinishParams& p, int t, const WStage& S,
                                               const uint32_t (&q2)[2][16], int lane,
                                               uint32_t ph[G]) {
  if (p.key_bits == 4) replay_weights_t<4, G>(p, t, S, q2, lane, ph);
  else replay_weights_t<3, G>(p, t, S, q2, lane, ph);
}

// One token into the warp's combined partial (m, l, a): + its exact term,
// and, for a quantized token, - the approximate term the scan added for it.
template <int G>
__device__ __forceinline__ void warp_token(const FinishParams& p, int t, const WStage& S, uint2 kr,
                                           uint2 vr, const FinParts<G>& P, const uint32_t (&q2)[2][16],
                                           int lane, float (&m)[G], float (&l)[G],
                                           float (&a)[G][4]) {
  const float kf[4] = {__uint_as_float(kr.x << 16), __uint_as_float(kr.x & 0xFFFF0000u),
                       __uint_as_float(kr.y << 16), __uint_as_float(kr.y & 0xFFFF0000u)};
  const float vf[4] = {__uint_as_float(vr.x << 16), __uint_as_float(vr.x & 0xFFFF0000u),
                       __uint_as_float(vr.y << 16), __uint_as_float(vr.y & 0xFFFF0000u)};
  // exact logits: per-lane partial dots, a reduce-scatter over the lanes
  // (each level halves the values a lane carries), then every head's total
  // gathered from the lane that holds it
  constexpr int GP = G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));
  constexpr int LG = GP == 1 ? 0 : (GP == 2 ? 1 : (GP == 4 ? 2 : 3));
  float v[GP];
#pragma unroll
  for (int j = 0; j < GP; ++j) {
    if (j < G) {
      const float4 qv = *reinterpret_cast<const float4*>(&P.qs[j][4 * lane]);
      v[j] = fmaf(qv.x, kf[0], fmaf(qv.y, kf[1], fmaf(qv.z, kf[2], qv.w * kf[3])));
    } else {
      v[j] = 0.f;
    }
  }
#pragma unroll
  for (int L = 0; L < LG; ++L) {
    const int o = 16 >> L, half = GP >> (L + 1);
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = up ? v[half + i] : v[i];
      const float send = up ? v[i] : v[half + i];
      v[i] = keep + __shfl_xor_sync(kAll, send, o);
    }
  }
#pragma unroll
  for (int o = 16 >> LG; o > 0; o >>= 1) v[0] += __shfl_xor_sync(kAll, v[0], o);
  float se[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    int src = 0;
#pragma unroll
    for (int L = 0; L < LG; ++L) src += ((j >> (LG - 1 - L)) & 1) * (16 >> L);
    se[j] = __shfl_sync(kAll, v[0], src) * p.kappa;
  }
  const bool qt = tok_quant(t);
  uint32_t ph[G];
  float code[4] = {0.f, 0.f, 0.f, 0.f};
  uint16_t svb = 0;
  float zv = 0.f;
  if (qt) {
    replay_weights<G>(p, t, S, q2, lane, ph);
    const int tt = t % kKG, rt = tt & 15, hi8 = rt >> 3, e = rt & 1, jg = lane >> 3;
    svb = *reinterpret_cast<const uint16_t*>(S.vsz + jg * 8 + hi8 * 4 + 2 * e);
    zv = h2f(*reinterpret_cast<const uint16_t*>(S.vsz + 32 + jg * 8 + hi8 * 4 + 2 * e));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // the staged pieces are the token column's lanes (gd*4 + tig) of the
      // k-step's chunks; word and bit as in vc_loc
      const int c = 4 * lane + i, mt = c >> 4, rc = c & 15, gd = rc & 7, chi = rc >> 3;
      const int bit = vc_pos(p.val_bits, mt) + 8 * chi + 16 * e;
      if (p.val_bits == 4) {
        const int w8 = 2 * (mt & 3) + hi8;
        const uint32_t w = *reinterpret_cast<const uint32_t*>(S.vp + ((w8 >> 2) * 8 + gd) * 16 + (w8 & 3) * 4);
        code[i] = (float)((w >> bit) & 15u);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(S.vp + gd * 16 + (2 * (mt & 1) + hi8) * 4);
        code[i] = (float)((w >> bit) & 3u);
      }
    }
  }
  // the partial's frame m moves only when a new term would exceed it by more
  // than 2^8 (warp-uniform test), so most tokens need no rescale
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const float mu = qt ? S.mu[j] : -INFINITY;
    const float cand = fmaxf(se[j], mu);
    if (cand > m[j] + 8.f) {
      const float al = exp2f(m[j] - cand);  // 0 while the partial is empty (m = -inf)
      l[j] *= al;
#pragma unroll
      for (int i = 0; i < 4; ++i) a[j][i] *= al;
      m[j] = cand;
    }
    const float pe = exp2f(se[j] - m[j]);
    l[j] += pe;
#pragma unroll
    for (int i = 0; i < 4; ++i) a[j][i] = fmaf(pe, vf[i], a[j][i]);
    if (qt) {
      const float f = exp2f(mu - m[j]);
      const uint16_t phj = (uint16_t)ph[j];
      const float pf = h2f(phj) * f, w = h2f(h_mul_rn(phj, svb)) * f;
      const float zt = pf * zv;
      l[j] -= pf;
#pragma unroll
      for (int i = 0; i < 4; ++i) a[j][i] -= fmaf(w, code[i], zt);
    }
  }
}

// The warp's tokens tok_at(0..n) into its partial P.wp[warp] (loaded,
// updated, stored back).
template <int G, typename TokAt>
__device__ __forceinline__ void warp_correct(const FinishParams& p, int seg, TokAt tok_at, int n,
                                             WStage* ring, FinParts<G>& P, const uint32_t (&q2)[2][16],
                                             int warp, int lane) {
  float m[G], l[G], a[G][4];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    m[j] = P.wp[warp][j][0];
    l[j] = P.wp[warp][j][1];
    const float4 v = *reinterpret_cast<const float4*>(&P.wp[warp][j][4 + 4 * lane]);
    a[j][0] = v.x;
    a[j][1] = v.y;
    a[j][2] = v.z;
    a[j][3] = v.w;
  }
#pragma unroll
  for (int i = 0; i < kWD - 1; ++i) stage_issue(p, seg, i < n ? tok_at(i) : -1, ring[i], lane);
  // exact rows two tokens ahead in registers
  uint2 kr = make_uint2(0u, 0u), vr = kr, kr1 = kr, vr1 = kr;
  if (n > 0) row_load(p, seg, tok_at(0), lane, kr, vr);
  if (n > 1) row_load(p, seg, tok_at(1), lane, kr1, vr1);
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const int t = tok_at(i);
    stage_issue(p, seg, i + kWD - 1 < n ? tok_at(i + kWD - 1) : -1, ring[(i + kWD - 1) % kWD], lane);
    uint2 kr2 = kr1, vr2 = vr1;
    if (i + 2 < n) row_load(p, seg, tok_at(i + 2), lane, kr2, vr2);
    cp_async_wait<kWD - 1>();
    __syncwarp();
    warp_token<G>(p, t, ring[i % kWD], kr, vr, P, q2, lane, m, l, a);
    __syncwarp();
    kr = kr1;
    vr = vr1;
    kr1 = kr2;
    vr1 = vr2;
  }
  cp_async_wait<0>();
  __syncwarp();
#pragma unroll
  for (int j = 0; j < G; ++j) {
    if (lane == 0) {
      P.wp[warp][j][0] = m[j];
      P.wp[warp][j][1] = l[j];
    }
    *reinterpret_cast<float4*>(&P.wp[warp][j][4 + 4 * lane]) = make_float4(a[j][0], a[j][1], a[j][2], a[j][3]);
  }
  __syncwarp();
}

template <int G, bool SELECT>
__global__ void __launch_bounds__(kFinThreads, 2) finish_kernel(const FinishParams p) {
  extern __shared__ __align__(16) uint8_t fsm[];
  FinPersist& PS = *reinterpret_cast<FinPersist*>(fsm);
  FinParts<G>& P = *reinterpret_cast<FinParts<G>*>(fsm + sizeof(FinPersist));
  uint8_t* U = fsm + sizeof(FinPersist) + sizeof(FinParts<G>);
  FinSelect& SS = *reinterpret_cast<FinSelect*>(U);
  FinCorr& FC = *reinterpret_cast<FinCorr*>(U);
  __shared__ uint32_t scratch[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_tot;
  __shared__ uint32_t s_cnt[kFinMaxC], s_pre[kFinMaxC + 1], s_tpre[kFinMaxC + 1];
  __shared__ uint32_t s_chq[kFinMaxC + 1];  // chosen ties before slice q
  __shared__ int s_mode;                     // 0 lists in shared memory, 1 fallback lists

  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  const int r = (int)cl.block_rank();
  const int seg = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int nq = p.nq, k = p.k;
  const int bb = seg / p.hkv, hh = seg % p.hkv;

  // ---- set-up: nothing here is written by the scan
  {  // this CTA's tail rows into L2 while the set-up runs
    const int n_mine = p.tail > r ? (p.tail - r + C - 1) / C : 0;
    for (int i = tid; i < n_mine * 4; i += kFinThreads)
      prefetch_part(p, seg, (1 << 30) | (r + C * (i >> 2)), i & 3);
  }
  for (int i = tid; i < G * kD; i += kFinThreads)
    P.qs[i / kD][i % kD] = bf16f(p.q[((size_t)bb * p.H + hh * G + i / kD) * kD + i % kD]);
  for (int i = tid; i < kFinWarps * G * kPartStride; i += kFinThreads)
    (&P.wp[0][0][0])[i] = (i % kPartStride) == 0 ? -INFINITY : 0.f;
  // the lane's q as the scan holds it: head (gid >> 1) + 4n of n-tile n
  uint32_t q2[2][16];
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int hq = (gid >> 1) + 4 * n;
    const bool ok = hq < G && (n == 0 || G > 4);
    q_frag(p.q + ((size_t)bb * p.H + (size_t)hh * G + (ok ? hq : 0)) * kD, ok, tig, q2[n]);
  }
  __syncthreads();
  const int warp = tid >> 5;

  // ---- T: this CTA's tail slots r, r + C, ... (exact rows only), warp w
  // taking every kFinWarps-th of them
  {
    const int n_mine = p.tail > r ? (p.tail - r + C - 1) / C : 0;
    const int n_w = n_mine > warp ? (n_mine - warp + kFinWarps - 1) / kFinWarps : 0;
    auto tail_at = [&](int i) { return (1 << 30) | (r + C * (warp + kFinWarps * i)); };
    warp_correct<G>(p, seg, tail_at, n_w, FC.st[warp], P, q2, warp, lane);
  }

  pdl_wait();
  pdl_launch_dependents();

  // ---- P5a (loads): this CTA's share of the scan's split partials, every
  // head: when the rows fit beside the selection buffers they are copied now
  // (cp.async) and merged after the selection, so their latency hides
  // behind it; else they are staged tile by tile then.
    long long w0 = 0, w1 = -1;
    if (p.ng > 0) {
      const long long T = p.scan_total, W = p.scan_warps;
      const long long x0 = (long long)seg * p.ng, x1 = x0 + p.ng - 1;
      w0 = scan_warp_of(x0, W, T);
      w1 = scan_warp_of(x1, W, T);
    }
    const int ns = (int)(w1 - w0 + 1);  // one partial slot per scan warp of the segment
    const int s0 = (int)((long long)ns * r / C), s1 = (int)((long long)ns * (r + 1) / C);
    constexpr int kV = kPartStride / 4;  // float4 per row
    const int nrows = (s1 - s0) * G;
    float* early = reinterpret_cast<float*>(U + sizeof(FinSelect));
    constexpr int kEarlyRows = (int)((sizeof(FinCorr) - sizeof(FinSelect)) / (kPartStride * sizeof(float)));
    const bool early_ok = nrows <= kEarlyRows;
    if (early_ok) {
      for (int i = tid; i < nrows * kV; i += kFinThreads) {
        const int row = i / kV, v = i % kV;
        cp_async16(early + row * kPartStride + 4 * v,
                   p.scan_part + ((size_t)(w0 + s0 + row / G + seg) * G + row % G) * kPartStride + 4 * v);
      }
    }
    cp_async_commit();

  const bool select = SELECT && k < nq;
  const int lo = min(nq, r * p.slice), hi = min(nq, lo + p.slice);
  bool hist_ok = false;
  // ---- P1 + P2: bin b* from the scan's histogram, then this slice's lists
  if (select) {
    // the slice's first 16 scores of this thread, loaded together with the
    // histogram so both round trips overlap
    const float* S = p.scores + (size_t)seg * p.capacity;
    float4 v0[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b0 = lo + 16 * tid + 4 * u;
      v0[u] = b0 < hi ? ld16<float4>(S + b0) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // thread t owns bins [32t, 32t + 32): loaded straight into registers
    const uint32_t* hg = p.hist + (size_t)seg * kScanHistBins + 32 * tid;
    uint32_t hb[32];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint4 v = ld16<uint4>(hg + 4 * u);
      hb[4 * u] = v.x;
      hb[4 * u + 1] = v.y;
      hb[4 * u + 2] = v.z;
      hb[4 * u + 3] = v.w;
    }
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) local += hb[i];
    uint32_t tot_all;
    block_prefix_excl(local, scratch, &tot_all);
    uint32_t cum = block_suffix_excl(local, scratch);  // keys in bins above this thread's
    if (tid == 0) {
      s_bin = -1;
      s_tot = tot_all;
    }
    __syncthreads();
#pragma unroll
    for (int i = 31; i >= 0; --i) {
      if (cum < (uint32_t)k && cum + hb[i] >= (uint32_t)k) {
        s_bin = 32 * tid + i;
        s_above = cum;
      }
      cum += hb[i];
    }
    __syncthreads();
    hist_ok = s_tot == (uint32_t)nq && s_bin >= 0;
    const uint32_t bstar = (uint32_t)s_bin;
    uint32_t base_s = 0, base_t = 0;
    if (hist_ok) {
      for (int t0 = lo; t0 < hi; t0 += 16 * kFinThreads) {
        const int b0 = t0 + 16 * tid;
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[u] = t0 == lo ? v0[u]
                          : (b0 + 4 * u < hi ? ld16<float4>(S + b0 + 4 * u) : make_float4(0.f, 0.f, 0.f, 0.f));
        uint32_t keys[16];
        uint32_t ms = 0, mt = 0, ns = 0, nt = 0;
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
            mt |= (ti ? 1u : 0u) << i;
            ns += su;
            nt += ti;
          }
        }
        uint32_t tot;
        const uint32_t pos = block_prefix_excl((ns << 16) | nt, scratch, &tot);
        uint32_t ps = base_s + (pos >> 16), pt = base_t + (pos & 0xFFFFu);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (ms & (1u << i)) {
            if (ps < (uint32_t)kLCap) PS.sure[ps] = (uint32_t)(b0 + i);
            ++ps;
          }
          if (mt & (1u << i)) {
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
    if (tid == 0) {
      PS.n_sure = base_s;
      PS.n_tie = base_t;
      PS.overflow = (base_s > (uint32_t)kLCap || base_t > (uint32_t)kLCap) ? 1u : 0u;
    }
  }
  cl.sync();

  // ---- P3: resolve the selection; every CTA knows the whole chosen set:
  // list q (CTA q's sure list, or its fallback list) and the chosen ties.
  uint32_t n_ch = 0;  // chosen ties (ascending in PS.chtie)
  const uint32_t* glist_base = p.glists + (size_t)seg * C * p.slice;
  if (select) {
    if (r == 0) {  // the scan's histogram is consumed: clear it for the next scan
      uint32_t* hg = p.hist + (size_t)seg * kScanHistBins;
      for (int i = 4 * tid; i < kScanHistBins; i += 4 * kFinThreads)
        *reinterpret_cast<uint4*>(hg + i) = make_uint4(0u, 0u, 0u, 0u);
    }
    __shared__ uint32_t s_tie[kFinMaxC], s_ovf[kFinMaxC];
    if (tid < C) {
      const FinPersist* o = cl.map_shared_rank(&PS, tid);
      s_cnt[tid] = o->n_sure;
      s_tie[tid] = o->n_tie;
      s_ovf[tid] = o->overflow;
    }
    __syncthreads();
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
    if (s_mode == 0) {
      // every CTA's ties in one pass (all remote loads in flight together)
      for (uint32_t i = tid; i < s_tpre[C]; i += kFinThreads) {
        int q = 0;
        while (q + 1 < C && s_tpre[q + 1] <= i) ++q;
        const FinPersist* o = cl.map_shared_rank(&PS, q);
        SS.akey[i] = o->tkey[i - s_tpre[q]];
        SS.aidx[i] = o->tidx[i - s_tpre[q]];
      }
      __syncthreads();
      n_ch = (uint32_t)k - s_pre[C];
      const uint32_t T = s_tpre[C];
      if (T <= (uint32_t)kFinThreads / 2) {
        // direct ranking: entry i is chosen iff fewer than n_ch entries come
        // before it in (key descending, index ascending) order; tpe threads
        // (a power of two) share an entry's comparisons
        uint32_t tpe = 2;
        while (tpe < 32 && tpe * 2 * T <= (uint32_t)kFinThreads) tpe *= 2;
        const uint32_t e = tid / tpe, part = tid % tpe;
        uint32_t rank = 0, my_idx = 0;
        if (e < T) {
          const uint32_t key = SS.akey[e];
          my_idx = SS.aidx[e];
#pragma unroll 4
          for (uint32_t j = part; j < T; j += tpe) {
            const uint32_t k2 = SS.akey[j];
            rank += (k2 > key || (k2 == key && SS.aidx[j] < my_idx)) ? 1u : 0u;
          }
        }
        for (uint32_t o = 1; o < tpe; o <<= 1) rank += __shfl_xor_sync(kAll, rank, o);
        const uint32_t chosen = (e < T && part == 0 && rank < n_ch) ? 1u : 0u;
        uint32_t tot;
        const uint32_t pos = block_prefix_excl(chosen, scratch, &tot);
        if (chosen) PS.chtie[pos] = my_idx;  // entries are in index order
        __syncthreads();
      } else {
        refine_ties(SS.akey, SS.aidx, T, n_ch, SS.hist, PS.chtie, scratch, &s_bin, &s_above,
                    &s_tot);
      }
    } else {
      const uint32_t n =
          select_full(p.scores + (size_t)seg * p.capacity, nq, k, lo, hi, SS.hist,
                      const_cast<uint32_t*>(glist_base) + (size_t)r * p.slice, scratch, &s_bin,
                      &s_above, &s_tot);
      if (tid == 0) PS.n_gl = n;
      __threadfence();
    }
  }
  const int mode = select ? s_mode : 0;
  if (select && mode == 1) {
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
  auto list_of = [&](int q) -> const uint32_t* {
    return mode == 1 ? glist_base + (size_t)q * p.slice : cl.map_shared_rank(PS.sure, q);
  };

  // ---- idx output: this CTA's chosen indices, ascending, at its offset
  if (select) {
    if (tid <= C) {
      const uint32_t b0 = (uint32_t)min(nq, tid * p.slice);
      s_chq[tid] = lower_bound_u32(PS.chtie, n_ch, b0);
    }
    __syncthreads();
    const uint32_t c0 = s_chq[r], c1 = s_chq[r + 1];
    const uint32_t off = s_pre[r] + c0;  // earlier slices: their lists and chosen ties
    const uint32_t* Lr = list_of(r);
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
  if (!SELECT && r == 0) {  // nothing reads the scan's histogram here: clear it
    uint32_t* hg = p.hist + (size_t)seg * kScanHistBins;
    for (int i = 4 * tid; i < kScanHistBins; i += 4 * kFinThreads)
      *reinterpret_cast<uint4*>(hg + i) = make_uint4(0u, 0u, 0u, 0u);
  }

  // ---- P5a (merge)
  {
    // rows (slot, head) staged in shared memory a tile at a time, every load
    // of a tile in flight together; thread (channel, half) merges the heads
    // j = half, half + 2, ... online
    const int c = tid & (kD - 1), half = tid >> 7;
    constexpr int kH2 = (G + 1) / 2;
    float mrun[kH2], lrun[kH2], arun[kH2];
#pragma unroll
    for (int i = 0; i < kH2; ++i) {
      mrun[i] = -INFINITY;
      lrun[i] = 0.f;
      arun[i] = 0.f;
    }
    float* tile = reinterpret_cast<float*>(U);
    constexpr int kTR = (int)(sizeof(FinCorr) / (kPartStride * sizeof(float)));
    if (early_ok) {
      cp_async_wait<0>();
      __syncthreads();
    }
    for (int r0 = 0; r0 < nrows; r0 += (early_ok ? nrows : kTR)) {
      const int nr = early_ok ? nrows : min(kTR, nrows - r0);
      if (early_ok) tile = early;
#pragma unroll 8
      for (int i = tid; i < (early_ok ? 0 : nr * kV); i += kFinThreads) {
        const int row = i / kV, v = i % kV;
        const int gr = r0 + row;
        const float* src = p.scan_part + ((size_t)(w0 + s0 + gr / G + seg) * G + gr % G) * kPartStride;
        reinterpret_cast<float4*>(tile + row * kPartStride)[v] = ld16<float4>(src + 4 * v);
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kH2; ++i) {
        const int j = half + 2 * i;
        if (j < G) {
#pragma unroll 1
          for (int row = (j - r0 % G + G) % G; row < nr; row += G) {
            const float* tr = tile + row * kPartStride;
            const float rl = tr[1];
            if (rl > 0.f) {
              const float mn = fmaxf(mrun[i], tr[0]);
              const float s0f = lrun[i] > 0.f ? exp2f(mrun[i] - mn) : 0.f;
              const float s1f = exp2f(tr[0] - mn);
              lrun[i] = lrun[i] * s0f + rl * s1f;
              arun[i] = arun[i] * s0f + tr[4 + c] * s1f;
              mrun[i] = mn;
            }
          }
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kH2; ++i) {
      const int j = half + 2 * i;
      if (j < G) {
        P.sp[j][4 + c] = arun[i];
        if (c == 0) {
          P.sp[j][0] = lrun[i] > 0.f ? mrun[i] : -INFINITY;
          P.sp[j][1] = lrun[i];
        }
      }
    }
  }
  // ---- P4: correction of an even share of the chosen set: the token list
  // first (compacted, in shared memory), then a warp per token
  {
    const int n_x = select ? k : (SELECT ? nq : k);  // positions of the chosen sequence
    const int per = (n_x + C - 1) / C;
    const int x0 = min(n_x, r * per), x1 = min(n_x, x0 + per);
#pragma unroll 1
    for (int xr = x0; xr < x1; xr += kTokCap) {
    const int xe = min(x1, xr + kTokCap);
    uint32_t base = 0;
#pragma unroll 1
    for (int xb = xr; xb < xe; xb += kFinThreads) {
      const int j = xb + tid;
      int t = -1;
      if (j < xe) {
        if (select) {
          if ((uint32_t)j < s_pre[C]) {
            int q = 0;
            while (q + 1 < C && s_pre[q + 1] <= (uint32_t)j) ++q;
            t = (int)list_of(q)[j - s_pre[q]];
          } else {
            t = (int)PS.chtie[j - s_pre[C]];
          }
        } else if (SELECT) {
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
      if (t >= 0) FC.tok[pos] = t;
      base += tot;
    }
    __syncthreads();
    const int n = (int)base;
    for (int i = tid; i < n * 4; i += kFinThreads)  // the exact rows into L2
      prefetch_part(p, seg, FC.tok[i >> 2], i & 3);
    const int n_w = n > warp ? (n - warp + kFinWarps - 1) / kFinWarps : 0;
    const int32_t* tl = FC.tok;
    auto chosen_at = [&](int i) { return tl[warp + kFinWarps * i]; };
    warp_correct<G>(p, seg, chosen_at, n_w, FC.st[warp], P, q2, warp, lane);
    __syncthreads();
    }
    // combine the warps' partials into P.run: thread (channel, half) merges
    // heads half, half + 2, ...
    const int c = tid & (kD - 1), half = tid >> 7;
    for (int j = half; j < G; j += 2) {
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kFinWarps; ++w) mx = fmaxf(mx, P.wp[w][j][0]);
      float l = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < kFinWarps; ++w) {
        const float mw = P.wp[w][j][0];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - mx);  // empty partials add nothing
        l = fmaf(P.wp[w][j][1], f, l);
        acc = fmaf(P.wp[w][j][4 + c], f, acc);
      }
      P.run[j][4 + c] = acc;
      if (c == 0) {
        P.run[j][0] = mx;
        P.run[j][1] = l;
      }
    }
  }

  cl.sync();

  // ---- P5b: CTA r owns heads j = r, r + C, ...: merge the C CTAs' scan
  // partials (m_a, l_a, a_a) and exact-minus-removed partials (m_c, l_c, a_c),
  // remote loads issued together, and write
  //   out = (a_c 2^(m_c-m) + a_a 2^(m_a-m)) / (l_c 2^(m_c-m) + l_a 2^(m_a-m))
  for (int j = r; j < G; j += C) {
    const int c = tid;
    if (c < kD) {
      float2 hd[kFinMaxC][2];
      float av[kFinMaxC][2];
#pragma unroll
      for (int q = 0; q < kFinMaxC; ++q) {
        if (q < C) {
          FinParts<G>* o = cl.map_shared_rank(&P, q);
          hd[q][0] = *reinterpret_cast<const float2*>(&o->sp[j][0]);
          hd[q][1] = *reinterpret_cast<const float2*>(&o->run[j][0]);
          av[q][0] = o->sp[j][4 + c];
          av[q][1] = o->run[j][4 + c];
        }
      }
      float ma = -INFINITY, mc = -INFINITY;
#pragma unroll
      for (int q = 0; q < kFinMaxC; ++q)
        if (q < C) {
          if (hd[q][0].y > 0.f) ma = fmaxf(ma, hd[q][0].x);
          mc = fmaxf(mc, hd[q][1].x);
        }
      const float m = fmaxf(ma, mc);
      float l = 0.f, acc = 0.f;
#pragma unroll
      for (int q = 0; q < kFinMaxC; ++q)
        if (q < C) {
          const float fa = hd[q][0].y > 0.f ? exp2f(hd[q][0].x - m) : 0.f;
          const float fc = hd[q][1].x == -INFINITY ? 0.f : exp2f(hd[q][1].x - m);
          l = fmaf(hd[q][0].y, fa, fmaf(hd[q][1].y, fc, l));
          acc = fmaf(av[q][0], fa, fmaf(av[q][1], fc, acc));
        }
      p.out[((size_t)bb * p.H + hh * G + j) * kD + c] = acc / l;
    }
  }
  // keep this CTA's shared memory alive until every peer has read it
  cl.sync();
}

template <int G, bool SEL>
static int pick_cluster(int n_seg, int num_sms) {
  constexpr size_t smem = fin_smem_bytes<G>();
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
    if (cudaOccupancyMaxActiveClusters(&n_active, finish_kernel<G, SEL>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      break;
    }
    if (n_active >= n_seg) best = c;
    else break;
  }
  return best;
}

template <int G, bool SEL>
static int launch_finish_t(FinishParams fp, int n_seg, cudaStream_t st) {
  constexpr size_t smem = fin_smem_bytes<G>();
  static bool configured[64] = {false};
  static int memo_seg[64][8] = {{0}}, memo_c[64][8] = {{0}};  // cluster size per (device, n_seg)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(finish_kernel<G, SEL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    C = pick_cluster<G, SEL>(n_seg, num_sms_current());
    if (dev >= 0 && dev < 64) {
      for (int i = 0; i < 8; ++i)
        if (memo_seg[dev][i] == 0) {
          memo_seg[dev][i] = n_seg;
          memo_c[dev][i] = C;
          break;
        }
    }
  }
  const int nq = fp.nq;
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
  return cudaLaunchKernelEx(&cfg, finish_kernel<G, SEL>, fp) == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

template <bool SEL>
static int launch_finish_g(const FinishParams& fp, int G, int n_seg, cudaStream_t st) {
  switch (G) {
    case 1: return launch_finish_t<1, SEL>(fp, n_seg, st);
    case 2: return launch_finish_t<2, SEL>(fp, n_seg, st);
    case 3: return launch_finish_t<3, SEL>(fp, n_seg, st);
    case 4: return launch_finish_t<4, SEL>(fp, n_seg, st);
    case 5: return launch_finish_t<5, SEL>(fp, n_seg, st);
    case 6: return launch_finish_t<6, SEL>(fp, n_seg, st);
    case 7: return launch_finish_t<7, SEL>(fp, n_seg, st);
    default: return launch_finish_t<8, SEL>(fp, n_seg, st);
  }
}

int launch_finish(const jfa_geom& g, const jfa_cache& c, const uint16_t* q, float scale, int k,
                  int32_t* idx_out, const int32_t* idx_in, const uint16_t* k_exact,
                  const uint16_t* v_exact, uint8_t* ws, const jfa_workspace_layout& L, float* out,
                  cudaStream_t st) {
  const int n_seg = g.batch * g.num_kv_heads;
  const int nq = split_point(g.n_ctx);
  FinishParams fp;
  fp.groups = static_cast<const uint8_t*>(c.groups);
  fp.tail_k = c.tail_k;
  fp.tail_v = c.tail_v;
  fp.k_exact = k_exact;
  fp.v_exact = v_exact;
  fp.q = q;
  fp.scores = reinterpret_cast<const float*>(ws + L.off_scores);
  fp.scan_part = reinterpret_cast<const float*>(ws + L.off_partials);
  fp.m_used = reinterpret_cast<const float*>(ws + L.off_mused);
  fp.hist = reinterpret_cast<uint32_t*>(ws + L.off_scan_hist);
  fp.glists = reinterpret_cast<uint32_t*>(ws + L.off_cand);
  fp.idx_in = idx_in;
  fp.idx_out = idx_out;
  fp.out = out;
  fp.flag = reinterpret_cast<uint32_t*>(ws + L.off_flag);
  fp.k = k;
  fp.nq = nq;
  fp.tail = g.n_ctx - nq;
  fp.capacity = g.capacity;
  fp.ng_cap = g.capacity / kKG;
  fp.hkv = g.num_kv_heads;
  fp.H = g.num_heads;
  fp.key_bits = g.key_bits;
  fp.val_bits = g.val_bits;
  fp.rec_bytes = record_bytes(g.key_bits, g.val_bits);
  const ScanPlan plan = scan_plan(g, num_sms_current());
  fp.scan_total = plan.total_groups;
  fp.scan_warps = plan.n_warps;
  fp.ng = plan.ng;
  fp.kappa = scale * 1.4426950408889634f;
  fp.slice = 64;
  const int G = g.num_heads / g.num_kv_heads;
  return idx_in ? launch_finish_g<false>(fp, G, n_seg, st) : launch_finish_g<true>(fp, G, n_seg, st);
}

}  // namespace jfa

// finish_impl.cuh — everything after the scan in one kernel.  A thread-block
// cluster of C CTAs (C <= 16) per (sequence, KV head):
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
#pragma once

#include <cooperative_groups.h>

#include "finish_params.cuh"
#include "jfa_approx.cuh"
#include "jfa_blocks.cuh"

namespace cg = cooperative_groups;

namespace jfa {

constexpr int kFinThreads = 256;
constexpr int kFinMaxC = kFinMaxCluster;  // 16: non-portable cluster size, few segments only
constexpr int kLCap = 1024;   // sure / tie list entries per CTA
constexpr int kTCap = 1024;   // gathered tie entries
constexpr int kRefBins = 2048;


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
  float run[G][kPartStride];   // this CTA's exact-minus-removed partial (frame, mass, acc)
  float sp[G][kPartStride];    // this CTA's share of the scan partials
};
// Shared-memory histograms store bin b at hpad(b) = b + b/32, so threads
// that each read a contiguous run of bins hit distinct banks.
__device__ __forceinline__ int hpad(int b) { return b + (b >> 5); }
struct FinSelect {
  uint32_t hist[kRefBins + kRefBins / 32];
  uint32_t akey[kTCap], aidx[kTCap];
};
// One token of a correction batch: its record pieces (cp.async) and its
// exact bf16 K and V rows.  The 16-byte pad puts the rows of consecutive
// tokens 4 banks apart, so the tensor-core operand loads are conflict-free.
struct TokStage {
  uint8_t ksz[512];      // key scales / zeros of its group
  uint8_t kcode[128];    // key-code words of the 4 lanes holding its m-tile row
  uint8_t vp[256];       // value-code pieces holding its column (8 or 16 x 16 B)
  uint8_t vsz[64];       // its value scales (32 B block) and zeros (32 B block)
  float mu[2 * kMaxG];   // the scan's running maxima (8) and biases (8) of its group
  uint16_t krow[kD];     // bf16 K row
  uint16_t vrow[kD];     // bf16 V row
  uint8_t pad[16];
};
static_assert(sizeof(TokStage) == 1552, "token stage layout");
constexpr int kTokCap = 1024;  // tokens listed per correction round
constexpr int kBT = 16;        // tokens per correction batch (one mma k-step)
// Correction batches, double-buffered: batch b + 1 is staged while batch b
// is computed.  The weights are bf16 triples (hi, mid, lo: 24 significant
// bits), head-major (the B operands of the value MMAs).
struct FinBatchT {
  TokStage st[2][kBT];
  int tok[2][kBT];
  uint16_t bex[3][kMaxG][kBT];      // exact weights
  uint16_t brem[3][4][kMaxG][kBT];  // minus the removed weights per 32-channel group
  uint16_t bpf[2][kMaxG][kBT];      // removed masses 2^(m_used - m) p as fp16 (hi, lo)
  float se[kBT][kMaxG];             // exact logits (log2 units)
  uint16_t ph[kBT][kMaxG];          // replayed fp16 weights of the scan
  float alpha[kMaxG];               // frame move of this batch per head
  float zsum[kMaxG][4];             // removed zero-point terms per head and channel group (final)
};
struct FinCorr {
  FinBatchT b;
  int32_t tok[kTokCap + kTail];
};
template <int G>
constexpr size_t fin_smem_bytes() {
  return sizeof(FinPersist) + sizeof(FinParts<G>) +
         (sizeof(FinSelect) > sizeof(FinCorr) ? sizeof(FinSelect) : sizeof(FinCorr));
}

// From bin counts h[hpad(0..nbins)) (nbins a multiple of blockDim) find the
// bin where the count taken from the top reaches r (1 <= r); *bin = -1 if
// the total < r.
static __device__ __noinline__ void find_bin_from_top(const uint32_t* h, int nbins, uint32_t r, uint32_t* scratch,
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
static __device__ __noinline__ void refine_ties(const uint32_t* akey, const uint32_t* aidx, uint32_t T, uint32_t r,
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
static __device__ __noinline__ uint32_t select_full(const float* S, int nq, int k, int lo, int hi, uint32_t* h,
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
// Correction helpers.  Token encoding: t in [0, nq) a quantized token,
// (1 << 30) | s the tail slot s (exact rows only); -1 an empty batch slot.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool tok_quant(int t) { return t >= 0 && !(t & (1 << 30)); }

template <typename T4>
__device__ __forceinline__ T4 ld16(const void* p) {
  return *reinterpret_cast<const T4*>(p);
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Record pieces of quantized token t into S: piece i (0..63) of the token
// is one 16-byte cp.async; the caller commits.
template <int KB, int VB>
__device__ __forceinline__ void stage_piece(const FinishParams& p, int seg, int t, TokStage& S, int i) {
  const uint8_t* rec = p.groups + ((size_t)seg * p.ng_cap + (size_t)(t / kKG)) * p.rec_bytes;
  const int tt = t % kKG, kk = tt >> 4, row = tt & 7, tgt = (tt & 7) >> 1;
  if (i < 32) {
    cp_async16(S.ksz + 16 * i, rec + 16 * i);
  } else if (i < 40) {
    const int j = i - 32;
    if (KB == 4) cp_async16(S.kcode + 16 * j, rec + off_kc() + kk * 1024 + row * 128 + 16 * j);
    else if (j < 6) cp_async16(S.kcode + 16 * j, rec + off_kc() + kk * 768 + row * 96 + 16 * j);
  } else if (i < 56) {
    const int j = i - 40;
    if (VB == 4 || j < 8) {
      const int chunk = VB == 4 ? 2 * kk + (j >> 3) : kk;
      cp_async16(S.vp + 16 * j, rec + off_vc(KB) + chunk * 512 + ((j & 7) * 4 + tgt) * 16);
    }
  } else if (i < 60) {
    const int j = i - 56;
    cp_async16(S.vsz + 16 * j, rec + off_vs(KB) + kk * 128 + tgt * 32 + (j & 1) * 16 + (j >> 1) * 512);
  } else {
    const int j = i - 60;
    cp_async16(reinterpret_cast<uint8_t*>(S.mu) + 16 * j,
               p.m_used + ((size_t)seg * p.ng_cap + (size_t)(t / kKG)) * (2 * kMaxG) + 4 * j);
  }
}

// 16-byte piece `piece` (0..15) of token t's exact K (v = false) or V row.
__device__ __forceinline__ uint4 row_piece(const FinishParams& p, int seg, int t, bool v, int piece) {
  const bool tail = (t & (1 << 30)) != 0;
  const size_t off = tail ? ((size_t)seg * kTail + (t & 0xFFFF)) * kD : ((size_t)seg * p.capacity + t) * kD;
  const uint16_t* base = v ? (tail ? p.tail_v : p.v_exact) : (tail ? p.tail_k : p.k_exact);
  return ld16<uint4>(base + off + 8 * piece);
}

// L2 prefetch of one of the four 128-byte halves of token t's exact K and V
// rows.
__device__ __forceinline__ void prefetch_part(const FinishParams& p, int seg, int t, int part) {
  const bool tail = (t & (1 << 30)) != 0;
  const size_t off = tail ? ((size_t)seg * kTail + (t & 0xFFFF)) * kD : ((size_t)seg * p.capacity + t) * kD;
  const uint16_t* base = (part & 2) ? (tail ? p.tail_v : p.v_exact) : (tail ? p.tail_k : p.k_exact);
  prefetch_l2(base + off + 64 * (part & 1));
}

// The scan's fp16 weights of quantized token t for every head, recomputed
// from its staged group pieces with the scan's own functions on the same
// operands (key_sz, scale_pos, q_tilde_col, key_afrag, qk_chain, approx_logit,
// approx_weight; the group bias as the scan stored it); ph[j] = fp16 bits of
// head j's weight, written by the lane whose MMA row and column hold it.
// q2[n]: the lane's q of head (gid >> 1) + 4n, as the scan holds it.
template <int KB, int G>
__device__ __forceinline__ void replay_weights_t(const FinishParams& p, int t, const TokStage& S,
                                                 const uint32_t (&q2)[2][16], int lane,
                                                 uint16_t* ph) {
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
  // only row `row` of the m-tile is staged; the other rows' codes are zero
  // (an MMA output row depends on its own A row alone)
  uint32_t w[KeyPos<KB>::WORDS];
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(S.kcode + tig * 4 * KeyPos<KB>::WORDS);
#pragma unroll
  for (int i = 0; i < KeyPos<KB>::WORDS; ++i) w[i] = gid == row ? kw[i] : 0u;
  uint32_t a[16][2];
  key_afrag<KB>(w, a);
  const float kappa_u = p.kappa * KeyPos<KB>::unscale;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float d[4];
    qk_chain(a, qb[n], d);
    const int h = tig + 4 * n;
    if (gid == row && h < G) ph[h] = f2h_rn(approx_weight(approx_logit(d, rr, kappa_u, bk[n]), S.mu[h]));
  }
}
__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// fp32 x as a bf16 triple hi + mid + lo (each the bf16 rounding of what the
// previous limbs leave; the remainder is below 2^-24 |x|).
__device__ __forceinline__ uint16_t bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ void split3(float x, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
  hi = bf16_bits(x);
  const float r1 = x - bf16_val(hi);
  mid = bf16_bits(r1);
  lo = bf16_bits(r1 - bf16_val(mid));
}
// Correction of the tokens tok_at(0..n), 16 at a time, into this CTA's
// combined partial P.run (frame m, mass l, acc; all 256 threads).  Batch
// b + 1 is staged (record pieces by cp.async, exact rows through registers)
// while batch b is computed:
//   replay the scan's fp16 weights of each quantized token (warp w: tokens
//          2w, 2w + 1); warp 0 also computes the 16 x 8 exact logits (bf16
//          MMA) and moves the frame of a head when one of the batch's terms
//          exceeds it by more than 2^8;
//   weights thread (head, token): exact weight 2^(s - m), removed mass
//          2^(m_used - m) p and removed value weights 2^(m_used - m) fp16(p s_v),
//          split into bf16 triples / fp16 pairs (B operands);
//   values warp w = channels 16w..16w+15: acc += V^T exact + codes^T removed;
//          the last warp also sums the masses (ones x exact, ones x removed)
//          and the zero-point terms (zeros x removed) on tensor cores; fp32
//          accumulators stay in registers across batches.
template <int G, int KB, int VB, typename TokAt>
__device__ __forceinline__ void batch_correct(const FinishParams& p, int seg, TokAt tok_at, int n,
                                              FinBatchT& B, FinParts<G>& P,
                                              const uint32_t (&q2)[2][16],
                                              const uint32_t (&qb)[8][2]) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  constexpr int kSumWarp = kFinThreads / 32 - 1;
  const int c0 = 16 * warp + gid;
  const bool h0ok = 2 * tig < G, h1ok = 2 * tig + 1 < G;
  float acc[4];
  acc[0] = h0ok ? P.run[2 * tig][4 + c0] : 0.f;
  acc[1] = h1ok ? P.run[2 * tig + 1][4 + c0] : 0.f;
  acc[2] = h0ok ? P.run[2 * tig][4 + c0 + 8] : 0.f;
  acc[3] = h1ok ? P.run[2 * tig + 1][4 + c0 + 8] : 0.f;
  // sums (last warp): dE = exact mass (every row), dF row 0 = removed mass,
  // rows 1..4 = removed zero-point terms of channel groups 0..3
  float dE[4], dF[4] = {0.f, 0.f, 0.f, 0.f};
  dE[0] = dE[2] = h0ok ? P.run[2 * tig][1] : 0.f;
  dE[1] = dE[3] = h1ok ? P.run[2 * tig + 1][1] : 0.f;
  const int nbatch = (n + kBT - 1) / kBT;
  // staging of batch bi into buffer buf: this warp's tokens 2w, 2w + 1;
  // the lane's row pieces: token 2w + (lane >> 4), piece lane & 15
  int rt = -1;
  uint4 kx = make_uint4(0u, 0u, 0u, 0u), vx = kx;
  auto issue = [&](int bi, int buf) {
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
      const int j = bi * kBT + 2 * warp + k2;
      const int t = j < n ? tok_at(j) : -1;
      if (tok_quant(t)) {
        TokStage& S = B.st[buf][2 * warp + k2];
#pragma unroll
        for (int i = lane; i < 64; i += 32) stage_piece<KB, VB>(p, seg, t, S, i);
      }
      if ((lane >> 4) == k2) rt = t;
    }
    cp_async_commit();
    kx = make_uint4(0u, 0u, 0u, 0u);
    vx = kx;
    if (rt != -1) {
      kx = row_piece(p, seg, rt, false, lane & 15);
      vx = row_piece(p, seg, rt, true, lane & 15);
    }
  };
  auto store_rows = [&](int buf) {
    TokStage& S = B.st[buf][2 * warp + (lane >> 4)];
    *reinterpret_cast<uint4*>(&S.krow[8 * (lane & 15)]) = kx;
    *reinterpret_cast<uint4*>(&S.vrow[8 * (lane & 15)]) = vx;
    if ((lane & 15) == 0) B.tok[buf][2 * warp + (lane >> 4)] = rt;
  };
  if (nbatch > 0) {
    issue(0, 0);
    store_rows(0);
  }
#pragma unroll 1
  for (int bi = 0; bi < nbatch; ++bi) {
    const int buf = bi & 1;
    cp_async_wait<0>();
    __syncthreads();
    if (bi + 1 < nbatch) issue(bi + 1, buf ^ 1);
    // ---- exact logits and frames (warp 0), replay (warp w: tokens 2w, 2w + 1)
    if (warp == 0) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint16_t* r0 = B.st[buf][gid].krow + 16 * ks + 2 * tig;
        const uint16_t* r1 = B.st[buf][gid + 8].krow + 16 * ks + 2 * tig;
        mma_bf16_16816(d, *reinterpret_cast<const uint32_t*>(r0), *reinterpret_cast<const uint32_t*>(r1),
                       *reinterpret_cast<const uint32_t*>(r0 + 8), *reinterpret_cast<const uint32_t*>(r1 + 8),
                       qb[ks][0], qb[ks][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] *= p.kappa;
      B.se[gid][2 * tig] = d[0];
      B.se[gid][2 * tig + 1] = d[1];
      B.se[gid + 8][2 * tig] = d[2];
      B.se[gid + 8][2 * tig + 1] = d[3];
      // the batch's largest term per head (exact logits, the scan maxima of
      // the removed tokens' groups), over the 16 token rows
      const int ta = B.tok[buf][gid], tb = B.tok[buf][gid + 8];
      const float* mua = B.st[buf][gid].mu;
      const float* mub = B.st[buf][gid + 8].mu;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int h = 2 * tig + c;
        float v = -INFINITY;
        if (ta != -1) v = fmaxf(v, d[c]);
        if (tb != -1) v = fmaxf(v, d[2 + c]);
        if (tok_quant(ta)) v = fmaxf(v, mua[h]);
        if (tok_quant(tb)) v = fmaxf(v, mub[h]);
        v = fmaxf(v, __shfl_xor_sync(kAll, v, 4));
        v = fmaxf(v, __shfl_xor_sync(kAll, v, 8));
        v = fmaxf(v, __shfl_xor_sync(kAll, v, 16));
        if (gid == 0 && h < G) {
          const float m = P.run[h][0];
          float al = 1.f;
          if (v > m + 8.f) {
            al = exp2f(m - v);  // 0 while the partial is empty (m = -inf)
            P.run[h][0] = v;
          }
          B.alpha[h] = al;
        }
      }
    }
#pragma unroll 1
    for (int k2 = 0; k2 < 2; ++k2) {
      const int tl = 2 * warp + k2, t = B.tok[buf][tl];
      if (tok_quant(t)) replay_weights_t<KB, G>(p, t, B.st[buf][tl], q2, lane, B.ph[tl]);
    }
    __syncthreads();
    // ---- weights: thread (head h, token slot tl)
    if (tid < kBT * G) {
      const int h = tid >> 4, tl = tid & 15;
      const int t = B.tok[buf][tl];
      const bool valid = t != -1, qt = tok_quant(t);
      const TokStage& S = B.st[buf][tl];
      const float m = P.run[h][0];
      const float pe = valid ? exp2f(B.se[tl][h] - m) : 0.f;
      split3(pe, B.bex[0][h][tl], B.bex[1][h][tl], B.bex[2][h][tl]);
      const float f = qt ? exp2f(S.mu[h] - m) : 0.f;
      const uint16_t phb = qt ? B.ph[tl][h] : (uint16_t)0;
      const float pf = h2f(phb) * f;
      const uint16_t pfh = f2h_rn(pf);
      B.bpf[0][h][tl] = pfh;
      B.bpf[1][h][tl] = f2h_rn(pf - h2f(pfh));
      const int tt = qt ? t % kKG : 0, hi8 = (tt & 15) >> 3, e = tt & 1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint16_t vsc = *reinterpret_cast<const uint16_t*>(S.vsz + j * 8 + hi8 * 4 + 2 * e);
        const float wv = qt ? h2f(h_mul_rn(phb, vsc)) * f : 0.f;
        split3(-wv, B.brem[0][j][h][tl], B.brem[1][j][h][tl], B.brem[2][j][h][tl]);
      }
    }
    __syncthreads();
    // ---- values: warp w = channels 16w .. 16w + 15
    {
      const float a0s = h0ok ? B.alpha[2 * tig] : 1.f;
      const float a1s = h1ok ? B.alpha[2 * tig + 1] : 1.f;
      acc[0] *= a0s;
      acc[1] *= a1s;
      acc[2] *= a0s;
      acc[3] *= a1s;
      // A operands: rows = channels c0, c0 + 8; columns = token slots
      // 2tig, 2tig + 1 (a0, a1) and 2tig + 8, 2tig + 9 (a2, a3)
      uint32_t va[4], ca[4];
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int s0 = 2 * tig + 8 * hs;
        const TokStage& S0 = B.st[buf][s0];
        const TokStage& S1 = B.st[buf][s0 + 1];
        va[2 * hs] = (uint32_t)S0.vrow[c0] | ((uint32_t)S1.vrow[c0] << 16);
        va[2 * hs + 1] = (uint32_t)S0.vrow[c0 + 8] | ((uint32_t)S1.vrow[c0 + 8] << 16);
        uint32_t cb[2][2];  // [token][row half]: bf16 bits of the code
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int t = B.tok[buf][s0 + u];
          const TokStage& S = u ? S1 : S0;
          uint32_t c_lo = 0u, c_hi = 0u;
          if (tok_quant(t)) {
            const int tt = t % kKG, hi8 = (tt & 15) >> 3, e = tt & 1;
            const int bit = vc_pos(VB, warp) + 16 * e;
            if (VB == 4) {
              const int w8 = 2 * (warp & 3) + hi8;
              const uint32_t wd = *reinterpret_cast<const uint32_t*>(S.vp + ((w8 >> 2) * 8 + gid) * 16 + (w8 & 3) * 4);
              c_lo = (wd >> bit) & 15u;
              c_hi = (wd >> (bit + 8)) & 15u;
            } else {
              const uint32_t wd = *reinterpret_cast<const uint32_t*>(S.vp + gid * 16 + (2 * (warp & 1) + hi8) * 4);
              c_lo = (wd >> bit) & 3u;
              c_hi = (wd >> (bit + 8)) & 3u;
            }
          }
          cb[u][0] = __float_as_uint((float)c_lo) >> 16;
          cb[u][1] = __float_as_uint((float)c_hi) >> 16;
        }
        ca[2 * hs] = cb[0][0] | (cb[1][0] << 16);
        ca[2 * hs + 1] = cb[0][1] | (cb[1][1] << 16);
      }
      const int j = warp >> 1;
#pragma unroll
      for (int l = 0; l < 3; ++l)
        mma_bf16_16816(acc, va[0], va[1], va[2], va[3], *reinterpret_cast<const uint32_t*>(&B.bex[l][gid][2 * tig]),
                       *reinterpret_cast<const uint32_t*>(&B.bex[l][gid][2 * tig + 8]));
#pragma unroll
      for (int l = 0; l < 3; ++l)
        mma_bf16_16816(acc, ca[0], ca[1], ca[2], ca[3], *reinterpret_cast<const uint32_t*>(&B.brem[l][j][gid][2 * tig]),
                       *reinterpret_cast<const uint32_t*>(&B.brem[l][j][gid][2 * tig + 8]));
      if (warp == kSumWarp) {
        dE[0] *= a0s;
        dE[1] *= a1s;
        dE[2] *= a0s;
        dE[3] *= a1s;
        dF[0] *= a0s;
        dF[1] *= a1s;
        dF[2] *= a0s;
        dF[3] *= a1s;
        constexpr uint32_t kOnesBf = 0x3F803F80u;
#pragma unroll
        for (int l = 0; l < 3; ++l)
          mma_bf16_16816(dE, kOnesBf, kOnesBf, kOnesBf, kOnesBf,
                         *reinterpret_cast<const uint32_t*>(&B.bex[l][gid][2 * tig]),
                         *reinterpret_cast<const uint32_t*>(&B.bex[l][gid][2 * tig + 8]));
        // A rows: 0 = ones, 1..4 = the value zero points of channel group
        // gid - 1 (fp16), others 0; columns = token slots
        uint32_t za[2];
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          uint32_t zz = 0u;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int sl = 2 * tig + 8 * hs + u, t = B.tok[buf][sl];
            uint32_t zh = 0u;
            if (gid == 0) {
              zh = 0x3C00u;
            } else if (gid <= 4 && tok_quant(t)) {
              const int tt = t % kKG, hi8 = (tt & 15) >> 3, e = tt & 1;
              zh = *reinterpret_cast<const uint16_t*>(B.st[buf][sl].vsz + 32 + (gid - 1) * 8 + hi8 * 4 + 2 * e);
            }
            zz |= zh << (16 * u);
          }
          za[hs] = zz;
        }
#pragma unroll
        for (int l = 0; l < 2; ++l)
          mma16816(dF, za[0], 0u, za[1], 0u, *reinterpret_cast<const uint32_t*>(&B.bpf[l][gid][2 * tig]),
                   *reinterpret_cast<const uint32_t*>(&B.bpf[l][gid][2 * tig + 8]));
      }
    }
    if (bi + 1 < nbatch) store_rows(buf ^ 1);
  }
  if (warp == kSumWarp) {
    if (gid == 0) {  // mass: exact minus removed
      if (h0ok) P.run[2 * tig][1] = dE[0] - dF[0];
      if (h1ok) P.run[2 * tig + 1][1] = dE[1] - dF[1];
    } else if (gid <= 4) {
      if (h0ok) B.zsum[2 * tig][gid - 1] = -dF[0];
      if (h1ok) B.zsum[2 * tig + 1][gid - 1] = -dF[1];
    }
  }
  __syncthreads();
  {
    const int j = warp >> 1;
    if (h0ok) {
      P.run[2 * tig][4 + c0] = acc[0] + B.zsum[2 * tig][j];
      P.run[2 * tig][4 + c0 + 8] = acc[2] + B.zsum[2 * tig][j];
    }
    if (h1ok) {
      P.run[2 * tig + 1][4 + c0] = acc[1] + B.zsum[2 * tig + 1][j];
      P.run[2 * tig + 1][4 + c0 + 8] = acc[3] + B.zsum[2 * tig + 1][j];
    }
  }
  __syncthreads();
}

template <int G, bool SELECT, int KB, int VB>
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
  __shared__ uint32_t s_hmax[kMaxG];          // per head: largest scan-partial maximum (key)

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
  for (int i = tid; i < G * kPartStride; i += kFinThreads)
    (&P.run[0][0])[i] = (i % kPartStride) == 0 ? -INFINITY : 0.f;
  // the lane's q as the scan holds it (head (gid >> 1) + 4n of n-tile n), and
  // as bf16 B fragments of the exact-logit MMA (head gid)
  uint32_t q2[2][16];
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int hq = (gid >> 1) + 4 * n;
    const bool ok = hq < G && (n == 0 || G > 4);
    q_frag(p.q + ((size_t)bb * p.H + (size_t)hh * G + (ok ? hq : 0)) * kD, ok, tig, q2[n]);
  }
  uint32_t qb[8][2];
  {
    const uint16_t* qrow = p.q + ((size_t)bb * p.H + (size_t)hh * G + (gid < G ? gid : 0)) * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qb[ks][0] = gid < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tig) : 0u;
      qb[ks][1] = gid < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tig + 8) : 0u;
    }
  }
  __syncthreads();

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

  // ---- P5a (merge): per head the largest partial maximum M first, then
  // every row's terms scaled by 2^(m_row - M) and summed (no exponential on
  // the accumulation chain); rows from the early copy, else staged a tile
  // at a time; thread (channel, half) takes heads j = half, half + 2, ...
  {
    const int c = tid & (kD - 1), half = tid >> 7;
    constexpr int kH2 = (G + 1) / 2;
    if (tid < G) s_hmax[tid] = 0u;  // key of -inf and below
    if (early_ok) cp_async_wait<0>();
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
    float* tile = reinterpret_cast<float*>(U);
    constexpr int kTR = (int)(sizeof(FinCorr) / (kPartStride * sizeof(float))) / kMaxG * kMaxG;
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
          reinterpret_cast<float4*>(tile + row * kPartStride)[v] = ld16<float4>(src + 4 * v);
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
  // ---- P4: correction of this CTA's tail slots r, r + C, ... and an even
  // share of the chosen set: the token list first (compacted, in shared
  // memory), then batches of 16 tokens
  {
    const int n_x = select ? k : (SELECT ? nq : k);  // positions of the chosen sequence
    const int per = (n_x + C - 1) / C;
    const int x0 = min(n_x, r * per), x1 = min(n_x, x0 + per);
    const int n_tail = p.tail > r ? (p.tail - r + C - 1) / C : 0;
#pragma unroll 1
    for (int xr = x0, first = 1; first || xr < x1; xr += kTokCap, first = 0) {
    const int xe = min(x1, xr + kTokCap);
    uint32_t base = 0;
    if (first) {
      for (int i = tid; i < n_tail; i += kFinThreads) FC.tok[i] = (1 << 30) | (r + C * i);
      base = (uint32_t)n_tail;
    }
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
    const int32_t* tl = FC.tok;
    auto chosen_at = [&](int i) { return tl[i]; };
    batch_correct<G, KB, VB>(p, seg, chosen_at, n, FC.b, P, q2, qb);
    }
  }
  cl.sync();

  // ---- P5b: CTA r owns heads j = r, r + C, ...: merge the C CTAs' scan
  // partials (m_a, l_a, a_a) and exact-minus-removed partials (m_c, l_c, a_c),
  // remote loads issued together, and write
  //   out = (a_c 2^(m_c-m) + a_a 2^(m_a-m)) / (l_c 2^(m_c-m) + l_a 2^(m_a-m))
  for (int j = r; j < G; j += C) {
    const int c = tid;
    if (c < kD && C > 8) {  // large clusters: frame first, then the sums (re-reading the frames)
      float ma = -INFINITY, mc = -INFINITY;
#pragma unroll 4
      for (int q = 0; q < C; ++q) {
        const FinParts<G>* o = cl.map_shared_rank(&P, q);
        const float2 ha = *reinterpret_cast<const float2*>(&o->sp[j][0]);
        const float2 hc = *reinterpret_cast<const float2*>(&o->run[j][0]);
        if (ha.y > 0.f) ma = fmaxf(ma, ha.x);
        mc = fmaxf(mc, hc.x);
      }
      const float m = fmaxf(ma, mc);
      float l = 0.f, acc = 0.f;
#pragma unroll 4
      for (int q = 0; q < C; ++q) {
        const FinParts<G>* o = cl.map_shared_rank(&P, q);
        const float2 ha = *reinterpret_cast<const float2*>(&o->sp[j][0]);
        const float2 hc = *reinterpret_cast<const float2*>(&o->run[j][0]);
        const float fa = ha.y > 0.f ? exp2f(ha.x - m) : 0.f;
        const float fc = hc.x == -INFINITY ? 0.f : exp2f(hc.x - m);
        l = fmaf(ha.y, fa, fmaf(hc.y, fc, l));
        acc = fmaf(o->sp[j][4 + c], fa, fmaf(o->run[j][4 + c], fc, acc));
      }
      p.out[((size_t)bb * p.H + hh * G + j) * kD + c] = acc / l;
    } else if (c < kD) {
      float2 hd[8][2];
      float av[8][2];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
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
      for (int q = 0; q < 8; ++q)
        if (q < C) {
          if (hd[q][0].y > 0.f) ma = fmaxf(ma, hd[q][0].x);
          mc = fmaxf(mc, hd[q][1].x);
        }
      const float m = fmaxf(ma, mc);
      float l = 0.f, acc = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q)
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
static int launch_finish_t(FinishParams fp, int n_seg, cudaStream_t st) {
  constexpr size_t smem = fin_smem_bytes<G>();
  static bool configured[64] = {false};
  static int memo_seg[64][8] = {{0}}, memo_c[64][8] = {{0}};  // cluster size per (device, key)
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
  const int max_c = fp.nq >= 16384 ? kFinMaxC : 8;
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
  return cudaLaunchKernelEx(&cfg, finish_kernel<G, SEL, KB, VB>, fp) == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

template <bool SEL, int KB, int VB>
static int launch_finish_g(const FinishParams& fp, int G, int n_seg, cudaStream_t st) {
  switch (G) {
    case 1: return launch_finish_t<1, SEL, KB, VB>(fp, n_seg, st);
    case 2: return launch_finish_t<2, SEL, KB, VB>(fp, n_seg, st);
    case 3: return launch_finish_t<3, SEL, KB, VB>(fp, n_seg, st);
    case 4: return launch_finish_t<4, SEL, KB, VB>(fp, n_seg, st);
    case 5: return launch_finish_t<5, SEL, KB, VB>(fp, n_seg, st);
    case 6: return launch_finish_t<6, SEL, KB, VB>(fp, n_seg, st);
    case 7: return launch_finish_t<7, SEL, KB, VB>(fp, n_seg, st);
    default: return launch_finish_t<8, SEL, KB, VB>(fp, n_seg, st);
  }
}

}  // namespace jfa

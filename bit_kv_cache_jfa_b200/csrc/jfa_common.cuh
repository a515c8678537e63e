// jfa_common.cuh — shared definitions of the sm_100a decode-attention kernels:
// the packed group-record layout, fp16 directed rounding, code unpacking and
// thin PTX wrappers (mma.sync, mbarrier, bulk copy).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "jfa.h"

#define JFA_HD __host__ __device__ __forceinline__

namespace jfa {

constexpr int kD = JFA_HEAD_DIM;         // 128 channels
constexpr int kKG = JFA_KEY_GROUP;       // 64 tokens per key group
constexpr int kVG = JFA_VAL_GROUP;       // 32 channels per value group
constexpr int kTail = JFA_TAIL_MAX;      // 64
constexpr int kMaxG = JFA_MAX_GQA;       // 8
constexpr int kPartStride = 132;         // floats per (slot, head): m, l, pad2, acc[128]
constexpr int kMaxScanWarps = 4096;      // cap on scan warps (partial slots)
constexpr int kFinMaxCluster = 16;       // CTAs per (sequence, KV head) in the finishing kernel
constexpr int kScanMinRecords = 2;       // records per scan warp at least (when the
                                         // work allows): fewer partials to merge
constexpr int kScanHistBits = 15;        // selection-score histogram of the scan: top 15 key bits
constexpr int kScanHistBins = 1 << kScanHistBits;
constexpr int kScanHistStride = kScanHistBins + 32;  // per segment: the bins, then the largest key
// Copies of each segment's scan histogram.  With few segments every scan warp
// adds into the same few hot bins, and atomics on one address serialise in
// L2; scan warp w adds into copy w mod R, and the readers sum the copies.
__host__ __device__ __forceinline__ int scan_hist_reps(long long n_seg) {
  return n_seg >= 32 ? 1 : (n_seg <= 2 ? 16 : (int)(32 / n_seg));
}
constexpr int kHistBins = 2048;          // top-k first-level histogram (11 key bits)
constexpr int kCtrStride = 8;            // top-k counters per segment: [0] scan warps done, [2] b*, [3] keys above b*

// ---------------------------------------------------------------------------
// Packed group record: 64 tokens of one (sequence, KV head).
//   [KS: key scales+zeros 512 B][KC: key codes 64*128*kb/8 B]
//   [VS: value scales+zeros 1024 B][VC: value codes 64*128*vb/8 B]
// The code order follows the register fragments of mma.sync.m16n8k16 so the
// scan kernel turns 128-bit shared-memory loads into ready A operands (keys
// and values); see kc_bits / vc_loc for the exact bit positions.
// ---------------------------------------------------------------------------
JFA_HD int kc_bytes(int kb) { return kKG * kD * kb / 8; }
JFA_HD int vc_bytes(int vb) { return kKG * kD * vb / 8; }
JFA_HD int off_ks() { return 0; }
JFA_HD int off_kc() { return 512; }
JFA_HD int off_vs(int kb) { return 512 + kc_bytes(kb); }
JFA_HD int off_vc(int kb) { return 512 + kc_bytes(kb) + 1024; }
JFA_HD int record_bytes(int kb, int vb) { return off_vc(kb) + vc_bytes(vb); }

// Warps per scan CTA: each warp owns a two-record shared-memory ring and the
// CTA takes a whole SM (227 KB of shared memory); at most 16 warps (12 when
// the query heads of a KV head fill two n-tiles and need more registers).
constexpr int scan_cta_warps(int kb, int vb, int nt) {
  return ((227 * 1024 - 1024) / (2 * (512 + 1024 * kb + 1024 + 1024 * vb))) > (nt == 2 ? 12 : 16)
             ? (nt == 2 ? 12 : 16)
             : ((227 * 1024 - 1024) / (2 * (512 + 1024 * kb + 1024 + 1024 * vb)));
}

struct BitLoc {
  int byte;  // byte offset of the 32-bit word inside its section
  int bit;   // bit of the code's least significant bit inside that word
};

// Fragment coordinates of key channel c as a q-pair index of the lane:
// k-step ks = c/16; inside it the thread tig = (c%8)/2 holds channels
// {2tig, 2tig+1} (half hf=0) and {2tig+8, 2tig+9} (hf=1); e picks the fp16
// half of the register.  Pair index p = 2*ks + hf runs over 16 pairs.
JFA_HD void key_channel_frag(int c, int& tig, int& pair, int& e) {
  int ks = c >> 4, r = c & 15;
  int hf = r >> 3;
  tig = (r & 7) >> 1;
  e = r & 1;
  pair = 2 * ks + hf;
}

// Key code of (token t, channel c) for the QK product with tokens as the
// A-operand rows of mma.sync.m16n8k16: m-tile mt = t/16 holds 32 lanes x W
// 32-bit words (W = 6 for 3-bit, 8 for 4-bit codes); lane = (t%8)*4 + tig,
// pair slot s = key_channel_frag's pair, row r = (t%16)/8 (token gid or
// gid + 8), half e (+16 bits).  Inside a 16-bit half a code sits at bit
// position 0, 3 or 6 (3-bit) or 0 or 4 (4-bit), so the half read as fp16 is
// the subnormal code * 2^(pos-24) after one AND; rows gid + 8 sit 9 (3-bit)
// or 8 (4-bit) bits higher, or in the next word.  3-bit slot 15 spreads its
// three code bits over bit 15 of three words.  Returns the number of pieces:
// 1 (code bits contiguous from L[0]) or 3 (code bit b at L[b]).
JFA_HD int kc_bits(int kb, int t, int c, BitLoc L[3]) {
  int tig, s, e;
  key_channel_frag(c, tig, s, e);
  const int mt = t >> 4, row = t & 15, gid = row & 7, r = row >> 3;
  const int W = kb == 4 ? 8 : 6;
  const int base = mt * 32 * 4 * W + (gid * 4 + tig) * 4 * W;
  if (kb == 4) {
    L[0].byte = base + 4 * (s & 7);
    L[0].bit = 4 * (s >> 3) + 8 * r + 16 * e;
    return 1;
  }
  if (s < 6) {
    L[0].byte = base + 4 * s;
    L[0].bit = 9 * r + 16 * e;
    return 1;
  }
  if (s < 12) {
    L[0].byte = base + 4 * (s - 6);
    L[0].bit = 3 + 9 * r + 16 * e;
    return 1;
  }
  if (s < 15) {
    L[0].byte = base + 4 * (2 * (s - 12) + r);
    L[0].bit = 6 + 16 * e;
    return 1;
  }
  for (int b = 0; b < 3; ++b) {
    L[b].byte = base + 4 * (3 * r + b);
    L[b].bit = 15 + 16 * e;
  }
  return 3;
}

// Key scale/zero of channel c: chunk i (16 B per tig) holds 4 pairs; chunks
// 0..3 hold scales of pairs 4i..4i+3, chunks 4..7 the zeros.
JFA_HD int ks_scale_off(int c) {
  int tig, p, e;
  key_channel_frag(c, tig, p, e);
  return (p >> 2) * 64 + tig * 16 + (p & 3) * 4 + 2 * e;
}
JFA_HD int ks_zero_off(int c) {
  int tig, p, e;
  key_channel_frag(c, tig, p, e);
  return (4 + (p >> 2)) * 64 + tig * 16 + (p & 3) * 4 + 2 * e;
}

// Value code of (token t, channel c) for the PV product (A operand: rows =
// channels, columns = tokens).  k-step kk = t/16; thread tig holds tokens
// {2tig, 2tig+1} (hi8 = 0) and {2tig+8, 2tig+9} (hi8 = 1); m-tile mt = c/16,
// row gid = c%8, chi = 1 for channels 8..15 of the tile.  Every code of
// m-tile mt sits at bit position p(mt) inside its 16-bit half (2-bit codes:
// 2*(mt/2), 4-bit: 4*(mt/4)), rows chi = 1 eight bits higher, so one AND
// (after a shift by 8) gives the fp16 subnormal code * 2^(p - 24) and the
// tile's accumulator is scaled back once.  Per lane and k-step: 4 words
// (2-bit, one 512-byte chunk) or 8 words (4-bit, chunks 2kk and 2kk+1); word
// 2*(mt%2) + hi8 (2-bit) or 2*(mt%4) + hi8 (4-bit).
JFA_HD int vc_pos(int vb, int mt) { return vb == 4 ? 4 * (mt >> 2) : 2 * (mt >> 1); }
JFA_HD BitLoc vc_loc(int vb, int t, int c) {
  int kk = t >> 4, rt = t & 15;
  int hi8 = rt >> 3, tig = (rt & 7) >> 1, e = rt & 1;
  int mt = c >> 4, rc = c & 15;
  int gid = rc & 7, chi = rc >> 3;
  int lane = gid * 4 + tig;
  BitLoc L;
  L.bit = vc_pos(vb, mt) + 8 * chi + 16 * e;
  if (vb == 4) {
    int w8 = 2 * (mt & 3) + hi8;  // word among the k-step's 8
    L.byte = (2 * kk + (w8 >> 2)) * 512 + lane * 16 + (w8 & 3) * 4;
  } else {  // 2-bit
    L.byte = kk * 512 + lane * 16 + (2 * (mt & 1) + hi8) * 4;
  }
  return L;
}

// Value scale/zero of (token t, channel group j).
JFA_HD int vs_scale_off(int t, int j) {
  int kk = t >> 4, rt = t & 15;
  int hi8 = rt >> 3, tig = (rt & 7) >> 1, e = rt & 1;
  return kk * 128 + tig * 32 + j * 8 + hi8 * 4 + 2 * e;
}
JFA_HD int vs_zero_off(int t, int j) { return 512 + vs_scale_off(t, j); }

// Quantized-token count for n tokens: the tail keeps N - N_q in [1, 64].
JFA_HD int split_point(int n) { return n <= 0 ? 0 : kKG * ((n - 1) / kKG); }

// ---------------------------------------------------------------------------
// fp16 directed rounding of an fp64 value (largest fp16 <= x / smallest >= x)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint16_t fp16_bits_rd(double x) {
  __half h = __double2half(x);  // round to nearest even
  uint16_t b = __half_as_ushort(h);
  double back = (double)__half2float(h);
  if (back > x) {               // step one fp16 ulp toward -inf
    if (b == 0x0000u) b = 0x8001u;
    else if (b & 0x8000u) b = (uint16_t)(b + 1);
    else b = (uint16_t)(b - 1);
  }
  return b;
}
__device__ __forceinline__ uint16_t fp16_bits_ru(double x) {
  __half h = __double2half(x);
  uint16_t b = __half_as_ushort(h);
  double back = (double)__half2float(h);
  if (back < x) {               // step one fp16 ulp toward +inf
    if (b == 0x8000u) b = 0x0001u;
    else if (b & 0x8000u) b = (uint16_t)(b - 1);
    else b = (uint16_t)(b + 1);
  }
  return b;
}

// ---------------------------------------------------------------------------
// Code unpacking: (x & mask) | 0x6400 in each fp16 half gives 1024 + code *
// 2^pos exactly; one fp16x2 FMA by (2^-pos, -1024*2^-pos) leaves the code.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

constexpr uint32_t kOneH2 = 0x3C003C00u;  // fp16x2 (1.0, 1.0)

// ---------------------------------------------------------------------------
// mma.sync m16n8k16, fp16 inputs, fp32 accumulate (D += A * B)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// mbarrier + bulk copy (global -> shared), bounded waits
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_g2s_nohint(void* dst, const void* src, uint32_t bytes,
                                                uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase with the given parity; gives up after ~1 s and returns
// false (the caller records JFA_DEVERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; it < (1u << 26); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && globaltimer_ns() - t0 > 1000000000ull) break;
  }
  return false;
}

// Programmatic dependent launch: wait for the preceding kernel of the stream
// (its writes visible) / let the next kernel of the stream start launching.
// Both are no-ops for a kernel launched without the PDL attribute.
// Split cluster barrier: a relaxed arrive (orders no memory access) and the
// wait for every thread of the cluster's arrive; between the two a thread
// runs no other cluster barrier.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void set_flag(uint32_t* flag, uint32_t bits) {
  if (flag) atomicOr(flag, bits);
}

// Orderable 32-bit key of an fp32 score: larger float -> larger key.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Inverse of float_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

}  // namespace jfa

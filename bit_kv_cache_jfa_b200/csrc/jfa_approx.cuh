// jfa_approx.cuh — the approximate-logit and weight arithmetic of one key
// group, shared by the scan (which adds every quantized token's softmax terms
// to its partials) and the correction (which takes the top-k tokens' terms
// back out).  Both call these functions on the same operands, so a removed
// weight equals the added one bit for bit and the subtraction leaves only the
// fp32 rounding of the two sums.
//
// Arithmetic (HACK review, Eq. (4): the product with affinely quantized keys
// is an integer product plus correction terms), per 64-token group g:
//   u[h][t] = kappa * ( sum_c (q[h][c] s[g][c]) k'[t][c] + sum_c q[h][c] m[g][c] )
// in log2 units (kappa = softmax scale * log2 e), on mma.sync.m16n8k16:
//   A = key codes, rows = 16 tokens of an m-tile, columns = channels.  A code
//       sits in the low mantissa bits of an fp16 half at bit position pos, so
//       the half is the subnormal code * 2^(pos - 24) and one AND extracts it.
//   B = q*s as an exact fp16 pair: column 2*h' + 0 holds hi = fp16(q s F),
//       column 2*h' + 1 holds lo = q s F - hi, for the 4 heads h' of an
//       n-tile; F = 2^(P - pos) per channel pair undoes the bit position, so
//       every product is code * q*s * 2^(P - 24).
//   The bias sum_c q_c m_c is an MMA chain with A = the zero points (every
//   row) and B = q.
#pragma once

#include "jfa_common.cuh"

namespace jfa {

// Key-code bit positions: largest position P and the position of slot s
// (slot = channel pair of the B fragment, s = 2*k_step + (channels 8..15)).
template <int KB>
struct KeyPos {
  static constexpr int P = KB == 4 ? 4 : 6;
  static constexpr int WORDS = KB == 4 ? 8 : 6;  // 32-bit words per lane per m-tile
  __host__ __device__ static constexpr int pos(int s) {
    return KB == 4 ? (s < 8 ? 0 : 4) : (s < 6 ? 0 : (s < 12 ? 3 : (s < 15 ? 6 : 0)));
  }
  // fp16x2 of F = 2^(P - pos(s))
  __host__ __device__ static constexpr uint32_t factor(int s) {
    return KB == 4 ? (s < 8 ? 0x4C004C00u : 0x3C003C00u)
                   : (s < 6 ? 0x54005400u : (s < 12 ? 0x48004800u : (s < 15 ? 0x3C003C00u : 0x54005400u)));
  }
  // kappa multiplier undoing the common 2^(P - 24)
  static constexpr float unscale = KB == 4 ? 1048576.0f : 262144.0f;
};

// q of query head h as mma.sync B-fragment channel pairs of the lane:
// pair pp = 0..15 holds channels c = 16*(pp>>1) + 2*tig + 8*(pp&1), c + 1.
__device__ __forceinline__ void q_frag(const uint16_t* qrow, bool ok, int tig, uint32_t q2[16]) {
#pragma unroll
  for (int pp = 0; pp < 16; ++pp) {
    const int c = 16 * (pp >> 1) + 2 * tig + 8 * (pp & 1);
    const uint32_t w = ok ? *reinterpret_cast<const uint32_t*>(qrow + c) : 0u;
    q2[pp] = pack_h2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
}

// The lane's key scale and zero pairs of a group (same pair order as q_frag)
// from the record's 512-byte scale/zero section (shared or global memory).
__device__ __forceinline__ void key_sz(const uint8_t* ks, int tig, uint32_t s[16], uint32_t z[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 sv = *reinterpret_cast<const uint4*>(ks + i * 64 + tig * 16);
    const uint4 zv = *reinterpret_cast<const uint4*>(ks + (4 + i) * 64 + tig * 16);
    s[4 * i + 0] = sv.x;
    s[4 * i + 1] = sv.y;
    s[4 * i + 2] = sv.z;
    s[4 * i + 3] = sv.w;
    z[4 * i + 0] = zv.x;
    z[4 * i + 1] = zv.y;
    z[4 * i + 2] = zv.z;
    z[4 * i + 3] = zv.w;
  }
}

// Key scales times the position factors F (exact powers of two).
template <int KB>
__device__ __forceinline__ void scale_pos(const uint32_t s[16], uint32_t sf[16]) {
#pragma unroll
  for (int pp = 0; pp < 16; ++pp) sf[pp] = h2_mul(s[pp], KeyPos<KB>::factor(pp));
}

// The lane's B column of q~ = q * s * F: limb 0 (hi) or 1 (lo), hi + lo exact.
__device__ __forceinline__ void q_tilde_col(const uint32_t q2[16], const uint32_t sf[16], bool lo,
                                            uint32_t b[16]) {
#pragma unroll
  for (int pp = 0; pp < 16; ++pp) {
    const uint32_t hi = h2_mul(q2[pp], sf[pp]);
    b[pp] = h2_fma(q2[pp], sf[pp], lo ? (hi ^ 0x80008000u) : 0u);
  }
}

// kappa * sum_c q_c m_c for the head of the lane's n-tile column pair
// (lane (gid, tig): head tig of the n-tile); rows all equal.
__device__ __forceinline__ float bias_mma(const uint32_t q2[16], const uint32_t z[16], float kappa) {
  float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    mma16816(d, z[2 * ks], z[2 * ks], z[2 * ks + 1], z[2 * ks + 1], q2[2 * ks], q2[2 * ks + 1]);
  return __fmul_rn(d[0], kappa);
}

// Key codes of one m-tile as A fragments: a[s][0] = slot s for token row gid,
// a[s][1] = for row gid + 8, from the lane's WORDS words.
template <int KB>
__device__ __forceinline__ void key_afrag(const uint32_t* w, uint32_t a[16][2]) {
  if constexpr (KB == 4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t ws = w[i] >> 8;
      a[i][0] = w[i] & 0x000F000Fu;
      a[i][1] = ws & 0x000F000Fu;
      a[8 + i][0] = w[i] & 0x00F000F0u;
      a[8 + i][1] = ws & 0x00F000F0u;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      const uint32_t ws = w[i] >> 9;
      a[i][0] = w[i] & 0x00070007u;
      a[i][1] = ws & 0x00070007u;
      a[6 + i][0] = w[i] & 0x00380038u;
      a[6 + i][1] = ws & 0x00380038u;
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      a[12 + i][0] = w[2 * i] & 0x01C001C0u;
      a[12 + i][1] = w[2 * i + 1] & 0x01C001C0u;
    }
    // slot 15: bit b of the code in bit 15 (31) of word b (rows gid) or 3 + b
    uint32_t t0 = (w[0] >> 15) & 0x00010001u, t1 = (w[3] >> 15) & 0x00010001u;
    t0 = lop_and_or(w[1] >> 14, 0x00020002u, t0);
    t1 = lop_and_or(w[4] >> 14, 0x00020002u, t1);
    a[15][0] = lop_and_or(w[2] >> 13, 0x00040004u, t0);
    a[15][1] = lop_and_or(w[5] >> 13, 0x00040004u, t1);
  }
}

// One m-tile x one n-tile, 8 k-steps: d[0] (hi) + d[1] (lo) for token row
// gid, d[2] + d[3] for row gid + 8, head tig of the n-tile.
__device__ __forceinline__ void qk_chain(const uint32_t a[16][2], const uint32_t b[16], float d[4]) {
  d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    mma16816(d, a[2 * ks][0], a[2 * ks][1], a[2 * ks + 1][0], a[2 * ks + 1][1], b[2 * ks], b[2 * ks + 1]);
}

// Approximate logit (log2 units) of token row gid (r = 0) or gid + 8 (r = 1).
__device__ __forceinline__ float approx_logit(const float d[4], int r, float kappa_u, float bk) {
  return __fmaf_rn(__fadd_rn(d[2 * r], d[2 * r + 1]), kappa_u, bk);
}

// Softmax weight of a logit u against the running maximum m, as the scan
// feeds it to the value MMAs (rounded to fp16 there): 2^(u - m) from the
// hardware base-2 exponential; results below 2^-126 flush to zero, far under
// the fp16 range the weight is stored in.
__device__ __forceinline__ float approx_weight(float u, float m) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(__fsub_rn(u, m)));
  return r;
}

// fp16 multiply with round-to-nearest (the value weight p * s_v of one token).
__device__ __forceinline__ uint16_t h_mul_rn(uint16_t a, uint16_t b) {
  uint16_t r;
  asm("mul.rn.f16 %0, %1, %2;" : "=h"(r) : "h"(a), "h"(b));
  return r;
}
__device__ __forceinline__ uint16_t f2h_rn(float x) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

}  // namespace jfa

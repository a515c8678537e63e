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
// in log2 units (kappa = softmax scale * log2 e).  q*s enters mma.sync as an
// exact fp16 pair (hi, lo): rows 0-7 of the A operand hold hi for the G <= 8
// heads, rows 8-15 lo; the codes k' are exact small integers in fp16.
#pragma once

#include "jfa_common.cuh"

namespace jfa {

// q of query head `gid` as mma.sync A fragments: pair pp = 0..15 holds
// channels c = 16*(pp>>1) + 2*tig + 8*(pp&1) and c+1 (bf16 -> fp16).
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

// q~ = q*s as (hi, lo) fp16 pairs with hi + lo = q*s exactly, and the group
// bias kappa * sum_c q_c m_c (an fp32 MMA chain: A = q rows, B = the zero
// points broadcast over the 8 columns).
__device__ __forceinline__ float q_tilde(const uint32_t q2[16], const uint32_t s[16],
                                         const uint32_t z[16], float kappa, uint32_t hi[16],
                                         uint32_t lo[16]) {
#pragma unroll
  for (int pp = 0; pp < 16; ++pp) {
    hi[pp] = h2_mul(q2[pp], s[pp]);
    lo[pp] = h2_fma(q2[pp], s[pp], hi[pp] ^ 0x80008000u);
  }
  float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) mma16816(d, q2[2 * ks], 0u, q2[2 * ks + 1], 0u, z[2 * ks], z[2 * ks + 1]);
  return __fmul_rn(d[0], kappa);
}

// One n-tile (8 tokens): d[e] (hi rows) and d[2+e] (lo rows) for head gid,
// token 8*nt + 2*tig + e.  b[] = the n-tile's codes as B fragments.
__device__ __forceinline__ void qk_chain(const uint32_t hi[16], const uint32_t lo[16],
                                         const uint32_t b[16], float d[4]) {
  d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    mma16816(d, hi[2 * ks], lo[2 * ks], hi[2 * ks + 1], lo[2 * ks + 1], b[2 * ks], b[2 * ks + 1]);
}

// Approximate logit (log2 units) of head gid, token 8*nt + 2*tig + e.
__device__ __forceinline__ float approx_logit(const float d[4], int e, float kappa, float bk) {
  return __fmaf_rn(__fadd_rn(d[e], d[2 + e]), kappa, bk);
}

// Softmax weight of a logit u against the running maximum m, as the scan
// feeds it to the value MMAs: fp16(2^(u - m)).
__device__ __forceinline__ float approx_weight(float u, float m) { return exp2f(__fsub_rn(u, m)); }

// fp16 multiply with round-to-nearest (the value weight p * s_v of one token).
__device__ __forceinline__ uint16_t h_mul_rn(uint16_t a, uint16_t b) {
  uint16_t r;
  asm("mul.rn.f16 %0, %1, %2;" : "=h"(r) : "h"(a), "h"(b));
  return r;
}
__device__ __forceinline__ uint16_t f2h_rn(float x) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Key codes of n-tile nt as B fragments of the lane, from the record's key
// code section (shared or global memory).
template <int KB>
__device__ __forceinline__ void key_codes(const uint8_t* kc, int nt, int lane, uint32_t b[16]) {
  if constexpr (KB == 4) {
    const uint4 c = *reinterpret_cast<const uint4*>(kc + nt * 512 + lane * 16);
    unpack4(c.x, b);
    unpack4(c.y, b + 4);
    unpack4(c.z, b + 8);
    unpack4(c.w, b + 12);
  } else {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(kc + (nt >> 2) * 1536 + lane * 48 + (nt & 3) * 12);
    unpack3(w[0], w[1], w[2], b);
  }
}

}  // namespace jfa

// jfa_fp4.cuh — the NVFP4 key pool and the block-sparse exact attention
// (Jet-QSparse abstract: NVFP4 cache storage, FP4 query-key products on
// Blackwell tensor cores, 128-token blocks aggregated in high precision).
//
// A pool record holds the keys of one (sequence, KV head, 128-token block):
//   [0, 8192)     E2M1 codes, 128 rows x 128 channels, two per byte (even
//                 channel in the low nibble), in the tensor core's K-major
//                 no-swizzle layout: 8-row x 16-byte core matrices, the four
//                 16-byte column chunks of a row group at 128-byte steps, row
//                 groups at 512-byte steps;
//   [8192, 9216)  UE4M3 block scales (one per 16 channels of a row), as two
//                 512-byte scale-factor atoms (channels 0-63, 64-127): the
//                 4 scales of row r at byte 16 (r mod 32) + 4 (r / 32);
//   [9216, 9224)  fp32 group scale of rows 0-63 and 64-127;
//   [9224, 9232)  padding.
// The query record of a (sequence, KV head) holds its G <= 8 query heads in
// the same code and scale layout (rows = heads, the rest zero) and the fp32
// scale of every head.
#pragma once
#include "jfa_internal.cuh"

namespace jfa {

constexpr int kF4Tok = 128;           // tokens per record (the MMA's M)
constexpr int kF4SfOff = 8192;
constexpr int kF4GsOff = 9216;
constexpr int kF4RecBytes = 9232;
constexpr int kF4QBytes = 1568;       // query record
constexpr int kF4QSfOff = 512;
constexpr int kF4QScaleOff = 1536;
constexpr double kE2M1Max = 6.0;
constexpr double kE4M3Max = 448.0;

// Byte of (row r, channel c) in a code block (the low nibble for even c).
__host__ __device__ __forceinline__ int f4_code_off(int r, int c) {
  return ((((r >> 3) << 2) + (c >> 5)) << 7) + ((r & 7) << 4) + ((c & 31) >> 1);
}
// Byte of the scale of (row r, 16-channel block j = 0..7) in a scale block.
__host__ __device__ __forceinline__ int f4_sf_off(int r, int j) {
  return ((j >> 2) << 9) + ((r & 31) << 4) + ((r >> 5) << 2) + (j & 3);
}

// --- the two minifloat formats, from their definitions ----------------------
// Nearest UE4M3 value to v >= 0 (3 mantissa bits, exponent bias 7, smallest
// normal 2^-6, subnormal step 2^-9), ties to the even mantissa, saturating
// at 448.  Exact: frexp/ldexp only move the exponent and rint rounds to
// nearest even.
__device__ __forceinline__ double e4m3_rn_pos(double v) {
  if (!(v > 0.0)) return 0.0;
  if (v >= kE4M3Max) return kE4M3Max;
  int e;
  frexp(v, &e);                       // v = f 2^e, f in [0.5, 1)
  const int ex = max(e - 1, -6);
  return ldexp(rint(ldexp(v, 3 - ex)), ex - 3);
}
// Encoding of a representable UE4M3 value.
__device__ __forceinline__ uint32_t e4m3_bits(double v) {
  if (v < 0.015625) return (uint32_t)(v * 512.0);
  int e;
  frexp(v, &e);
  const int ex = e - 1;
  return ((uint32_t)(ex + 7) << 3) | ((uint32_t)ldexp(v, 3 - ex) - 8u);
}
// E2M1 code (bit 3 = sign) of the value nearest to q, ties to the even code,
// |q| > 6 saturating: the grid 0, .5, 1, 1.5, 2, 3, 4, 6 and its midpoints.
__device__ __forceinline__ uint32_t e2m1_code(double q) {
  const double a = fabs(q);
  const uint32_t c = (a > 0.25) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5) +
                     (a >= 3.5) + (a > 5.0);
  return (q < 0.0 && c) ? (c | 8u) : c;
}
// fp32 tensor scale amax / (6 * 448), 1 when amax is 0 (the quotient of
// two doubles rounded once to fp32).
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
  return amax > 0.f ? __double2float_rn((double)amax / (kE2M1Max * kE4M3Max)) : 1.f;
}

// --- launchers ----------------------------------------------------------------
// Quantize key groups [g_from, g_to) (64 tokens each) of every segment from
// the exact bf16 keys k_src [B][H_kv][capacity][128] into the pool.
int launch_fp4_pack(const jfa_geom& g, int g_from, int g_to, const uint16_t* k_src, uint8_t* pool,
                    uint32_t* flag, cudaStream_t st);
// Quantize the queries (one record per segment into the workspace) and scan
// every block of the N_q quantized tokens: selection scores into the
// workspace's score array.
int launch_fp4_scores(const jfa_geom& g, const uint8_t* pool, const uint16_t* q, float scale,
                      uint8_t* ws, const jfa_workspace_layout& L, cudaStream_t st);
// Exact softmax attention over idx [B][H_kv][k] (ascending or not, -1 =
// none) and the tail [N_q, n_ctx) of every segment, rows from the exact copy.
int launch_sparse_attend(const jfa_geom& g, const uint16_t* q, float scale, const int32_t* idx,
                         int k, const uint16_t* k_exact, const uint16_t* v_exact, bool on_host,
                         uint8_t* ws, const jfa_workspace_layout& L, float* out, cudaStream_t st);
// Per-segment record of the critical channels: int32 channel[128] (the kept
// ones first, ascending), then fp32 q[8][128] (scale * q_h at the kept
// channels, in the same order).
constexpr int kChanRecBytes = 128 * 4 + 8 * 128 * 4;
// Channel-major key copy and per-channel max|K| for tokens in groups
// [g_from, g_to); critical-channel selection scores into the workspace.
int launch_channel_pack(const jfa_geom& g, int g_from, int g_to, const uint16_t* k_src, uint16_t* k_t,
                        float* k_max, cudaStream_t st);
int launch_channel_scores(const jfa_geom& g, const uint16_t* k_t, const float* k_max, const uint16_t* q,
                          float scale, int r, uint8_t* ws, const jfa_workspace_layout& L,
                          cudaStream_t st);
// 1-bit KV pool: records of 64-token groups quantized at 1 bit from the exact
// bf16 rows; dense attention over every quantized token and the exact tail.
constexpr int kOneBitRecBytes = 3584;
int launch_onebit_pack(const jfa_geom& g, int g_from, int g_to, const uint16_t* k_src,
                       const uint16_t* v_src, uint8_t* pool, uint32_t* flag, cudaStream_t st);
int launch_onebit_attend(const jfa_geom& g, const uint8_t* pool, const uint16_t* q, float scale,
                         const uint16_t* k_exact, const uint16_t* v_exact, uint8_t* ws,
                         const jfa_workspace_layout& L, float* out, cudaStream_t st);
// Splits per segment of the sparse attention (host rule shared with the
// workspace sizing): at most kSpMaxSplit, and n_seg * splits <= max(n_seg, 512).
constexpr int kSpMaxSplit = 32;
constexpr int kSpSlots = 512;

}  // namespace jfa

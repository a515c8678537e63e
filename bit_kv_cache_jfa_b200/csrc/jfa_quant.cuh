// jfa_quant.cuh — the group quantization rule shared by the packing kernels
// (HACK review, Eq. (4) context: x ~ s * x' + m with m the partition
// minimum; TailorKV review: FP16 zero point and scale per group):
//   zero  = largest fp16 <= min,  scale = smallest fp16 >= (max - zero)/(2^b - 1)
//   code  = round-half-even((x - zero) / scale), clipped; both quotients fp64.
#pragma once
#include "jfa_internal.cuh"

namespace jfa {

__device__ __forceinline__ void quant_params(double mn, double mx, int bits, uint16_t& zbits,
                                             uint16_t& sbits, double& z, double& s) {
  zbits = fp16_bits_rd(mn);
  z = (double)__half2float(__ushort_as_half(zbits));
  sbits = fp16_bits_ru((mx - z) / (double)((1 << bits) - 1));
  s = (double)__half2float(__ushort_as_half(sbits));
}

__device__ __forceinline__ uint32_t quant_code(double x, double z, double s, int bits) {
  if (s == 0.0) return 0u;
  double c = rint((x - z) / s);
  double lv = (double)((1 << bits) - 1);
  c = c < 0.0 ? 0.0 : (c > lv ? lv : c);
  return (uint32_t)c;
}

__device__ __forceinline__ bool finite_h(uint16_t b) { return (b & 0x7C00u) != 0x7C00u; }
__device__ __forceinline__ float bf(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

}  // namespace jfa

// RoPE rotation of bf16 operands, in two rounding schemes.
//
// RoPE ("Embeddings & the Residual Stream", section "Positional information:
// RoPE, not a learned table") rotates feature i with feature i + d/2:
//   out[i]       = x[i]       * cos - x[i + d/2] * sin
//   out[i + d/2] = x[i + d/2] * cos + x[i]       * sin
//
// 1. rope_bf16x2: the rotation as that page's apply_rope evaluates it on bf16
//    tensors (cos and sin cast to x.dtype, then x*cos + rotate_half(x)*sin in
//    that dtype): cos and sin rounded to bf16, each product rounded to bf16,
//    the sum rounded to bf16, all to nearest even. A product of two bf16
//    values is exact in fp32, so mul.rn.bf16x2 (one rounding of the exact
//    product) gives what an fp32 product cast to bf16 gives. The sum of two
//    bf16 values is exact in fp32 unless their exponents differ by 16 or
//    more, and then it lies closer to the larger addend than a quarter of
//    that addend's bf16 spacing, so add.rn.bf16x2 (one rounding) and an fp32
//    sum cast to bf16 both give the larger addend. Used for Q and K in the
//    attention kernels.
//
// 2. rope_round_bf16: x*c + y*s' rotated exactly and rounded once to bf16,
//    for an fp32 value x (the projection's accumulator, whose fused epilogue
//    rounds once). Both products are exact in fp64 for a bf16 x; one fp64
//    fused multiply-add gives the exact value rounded once to fp64, rounded
//    to bf16 through a round-to-odd fp32 intermediate, which makes the two
//    roundings equal to a single rounding of the fp64 value.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace gqa {

// Two fp32 values -> one bf16x2 word (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two lanes of the bf16 rotation: lo, hi hold features (i, i+1) and
// (i + d/2, i + 1 + d/2); c, s the bf16 cos and sin of frequencies i, i+1.
//   lo' = RN(RN(lo*c) - RN(hi*s)),  hi' = RN(RN(hi*c) + RN(lo*s))
__device__ __forceinline__ void rope_bf16x2(uint32_t lo, uint32_t hi, uint32_t c, uint32_t s, uint32_t& olo,
                                            uint32_t& ohi) {
  asm("{\n\t.reg .b32 lc, hs, hc, ls;\n\t"
      "mul.rn.bf16x2 lc, %2, %4;\n\t"
      "mul.rn.bf16x2 hs, %3, %5;\n\t"
      "mul.rn.bf16x2 hc, %3, %4;\n\t"
      "mul.rn.bf16x2 ls, %2, %5;\n\t"
      "sub.rn.bf16x2 %0, lc, hs;\n\t"
      "add.rn.bf16x2 %1, hc, ls;\n\t}"
      : "=r"(olo), "=r"(ohi)
      : "r"(lo), "r"(hi), "r"(c), "r"(s));
}

// fp64 -> bf16, round to nearest even, in one rounding (round-to-odd to fp32
// first keeps the second rounding exact).
__device__ __forceinline__ uint16_t f64_to_bf16_bits_rn(double v) {
  float f = __double2float_rz(v);
  if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// bf16 bits of RN(x*c + y*sp), exact single rounding.
__device__ __forceinline__ uint16_t rope_round_bf16(float x, float c, float y, float sp) {
  return f64_to_bf16_bits_rn(fma((double)x, (double)c, (double)y * (double)sp));
}

}  // namespace gqa

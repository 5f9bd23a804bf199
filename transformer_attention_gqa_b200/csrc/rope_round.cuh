// Exactly rounded RoPE rotation of bf16 operands.
//
// RoPE ("Embeddings & the Residual Stream", section "Positional information:
// RoPE, not a learned table") rotates feature i with feature i + d/2:
//   out[i]       = x[i]       * cos - x[i + d/2] * sin
//   out[i + d/2] = x[i + d/2] * cos + x[i]       * sin
// Both have the form x*c + y*s' (s' = -sin or +sin) with x, y bf16 and c, s'
// fp32. Both products are exact in fp64, so one fp64 fused multiply-add gives
// the exact value rounded once to fp64; that is rounded once more, to nearest
// even, to bf16 through a round-to-odd fp32 intermediate, which makes the two
// roundings equal to a single rounding of the exact value. (A branch-free
// fp32 evaluation with an fp64 fallback near bf16 rounding midpoints was
// measured slower: the rare fallbacks diverge whole warps.)
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace gqa {

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

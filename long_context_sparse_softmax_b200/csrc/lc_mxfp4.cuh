// MXFP4 quantisation of a 128-element chunk held 4 per lane by a warp (OCP Microscaling
// Formats v1.0): per block of 32 elements (an aligned group of 8 lanes) the scale is
// X = 2^(floor(log2 amax) - 2) (2 = the largest exponent of E2M1; a zero block takes X = 2^0)
// and each element v / X is converted to E2M1 with round-to-nearest-even and saturation at
// +-6.  Zero is always code 0.  Element 2i goes to the low nibble of byte i.  Shared by the
// standalone quantiser and the indexer that quantises its queries itself, so that both
// produce the same bytes.
#pragma once

#include <cstdint>

namespace lc {

// Two bytes of E2M1 codes: byte 0 = (v0 low nibble, v1 high), byte 1 = (v2, v3).
__device__ __forceinline__ uint32_t e2m1x4(float v0, float v1, float v2, float v3) {
  uint32_t r;
  asm("{\n.reg .b8 b0, b1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
      "mov.b32 %0, {b0, b1, b0, b1};\n}\n"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
  r &= 0xffffu;
  // negative zero (sign bit over a zero magnitude) -> code 0
  const uint32_t mag = r & 0x7777u;
  const uint32_t zero = ~(mag | (mag >> 1) | (mag >> 2)) & 0x1111u;
  return r & ~(zero << 3);
}

// The 4 values of this lane (elements 4 lane .. 4 lane + 3 of the chunk): their 2 code bytes
// (low 16 bits of the result) and, in *scale, the E8M0 byte of this lane's block.  Every
// lane of the warp takes part (the block maximum is a shuffle).
__device__ __forceinline__ uint32_t mxfp4_quant4(const float (&v)[4], uint32_t* scale) {
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int e = amax > 0.f ? ilogbf(amax) - 2 : 0;
  e = min(max(e, -127), 127);
  *scale = static_cast<uint32_t>(e + 127);
  return e2m1x4(ldexpf(v[0], -e), ldexpf(v[1], -e), ldexpf(v[2], -e), ldexpf(v[3], -e));
}

}  // namespace lc

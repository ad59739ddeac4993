// 8-bit (E4M3) cache codes: conversions through the hardware's cvt forms.
// E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits, finite values only
// (largest 448, S.1111.111 is NaN).  Every E4M3 value is exact in fp16.
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

namespace pa {

// Two floats -> two codes, `lo` in the low byte: round to nearest even,
// magnitudes past 448 (infinities too) saturate to 448, NaN stays NaN.
__device__ __forceinline__ uint16_t e4m3x2_from_floats(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Eight numbers -> their eight codes (low byte first) of x / scale: the
// quotient in IEEE fp32 (round to nearest), then rounded as above.  The
// cache write and the one-launch step's new row both use this, so the same
// inputs give the same codes.
__device__ __forceinline__ uint2 e4m3x8_quantize(const float (&x)[8], float scale) {
  uint2 o;
  o.x = e4m3x2_from_floats(__fdiv_rn(x[0], scale), __fdiv_rn(x[1], scale)) |
        (static_cast<uint32_t>(e4m3x2_from_floats(__fdiv_rn(x[2], scale),
                                                  __fdiv_rn(x[3], scale))) << 16);
  o.y = e4m3x2_from_floats(__fdiv_rn(x[4], scale), __fdiv_rn(x[5], scale)) |
        (static_cast<uint32_t>(e4m3x2_from_floats(__fdiv_rn(x[6], scale),
                                                  __fdiv_rn(x[7], scale))) << 16);
  return o;
}

// Two codes (low byte first) -> their values as a half2 (exact).
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint16_t x) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(x));
  return *reinterpret_cast<__half2*>(&r);
}

// Four codes (one 32-bit word, low byte first) -> two half2 words: codes 0, 1
// in `lo`, codes 2, 3 in `hi` (exact).
__device__ __forceinline__ void e4m3x4_to_half2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// c + a.x * b.x + a.y * b.y for two fp16 pairs (a, b packed as half2 words),
// summed in fp32: each fp16 x fp16 product is exact in fp32.
__device__ __forceinline__ float dot2_f16_f32(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t.reg .f32 t;\n\t"
      "mov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 t, a0, b0, %3;\n\tfma.rn.f32.f16 %0, a1, b1, t;\n\t}"
      : "=f"(d)
      : "r"(a), "r"(b), "f"(c));
  return d;
}

// Sixteen codes (one 16-byte vector) -> sixteen floats.
__device__ __forceinline__ void unpack16_e4m3(const uint4& v, float (&f)[16]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 a = __half22float2(e4m3x2_to_half2(static_cast<uint16_t>(w[i] & 0xffffu)));
    const float2 b = __half22float2(e4m3x2_to_half2(static_cast<uint16_t>(w[i] >> 16)));
    f[4 * i + 0] = a.x;
    f[4 * i + 1] = a.y;
    f[4 * i + 2] = b.x;
    f[4 * i + 3] = b.y;
  }
}

}  // namespace pa

// Device-side FP4/FP8 helpers for sm_100a: E2M1 / E4M3 conversion instructions, decoders
// written from the format definitions, and the exact float32 helpers the quantisation
// recipe needs (IEEE round-to-nearest, no contraction).
//
// Formats: E2M1 = 1 sign, 2 exponent (bias 1), 1 mantissa bit, magnitudes
// {0, .5, 1, 1.5, 2, 3, 4, 6}; E4M3 ("fn") = bias 7, 3 mantissa bits, max 448;
// E8M0 = 2^(c-127). These are the encodings of the OCP Microscaling specification cited
// by the SharQ page (pith.science 2606.26587, reference list) and of NVFP4.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace sharq {

// 8 floats -> 8 E2M1 codes in one word, v[0] in bits 0..3 (round to nearest even,
// saturating at +-6, sign kept).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float v0, float v1, float v2, float v3,
                                               float v4, float v5, float v6, float v7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// Non-negative float -> E4M3 code (round to nearest even, saturating at 448).
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFFu;
}

// E2M1 code (low 4 bits) -> float, from the bit fields.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  // e == 0: 0 or 0.5; e > 0: (1 + m/2) * 2^(e-1)
  uint32_t bits = e ? (((e - 1u + 127u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
  bits |= (c & 8u) << 28;
  return __uint_as_float(bits);
}

// E4M3 code (unsigned) -> float, from the bit fields.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return __fmul_rn(__uint2float_rn(m), 0.001953125f);  // m * 2^-9, exact
  return __uint_as_float(((e - 7u + 127u) << 23) | (m << 20));
}

// 2^e as a float for e in [-127, 127] (2^-127 is the one subnormal case).
__device__ __forceinline__ float pow2f(int e) {
  return e >= -126 ? __uint_as_float(uint32_t(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// 8 E2M1 codes (code i in bits 4i..4i+3) -> 4 f16x2 words; code 2j goes to the low half
// of word j, code 2j+1 to the high half. Exact (every E2M1 value is an f16 value).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(codes));
}

// Packed float32 pairs (sm_100a f32x2 arithmetic, round to nearest even per lane).
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// float from a 16-bit input element
template <bool BF16>
__device__ __forceinline__ float in_to_float(uint32_t h) {
  if (BF16) return __uint_as_float(h << 16);
  float f;
  asm("{ .reg .f16 t; mov.b16 t, %1; cvt.f32.f16 %0, t; }" : "=f"(f) : "h"(uint16_t(h)));
  return f;
}

}  // namespace sharq

// Block quantisation recipes shared by the activation and weight kernels (device code).
//
// NVFP4: sf = E4M3_rne(a * k) with a the block's max |v| and k = 448 / amax per tensor;
// d = E4M3(sf) * s_g with s_g = amax / 2688; inv = 1 / d (one correctly rounded
// reciprocal per block); q = E2M1_rne(v * inv).
// MXFP4 (OCP MX): e = clamp(floor(log2 a) - 2, -127, 127); q = E2M1_rne(v * 2^-e).
// Every float operation is an explicit round-to-nearest intrinsic so that the compiler
// cannot contract or reassociate them.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "fp4_device.cuh"
#include "sharq_internal.h"

namespace sharq {

// NVFP4 quantisation of N values with one E4M3 block scale, given the tensor constants
// s_g = amax / 2688 and k = 448 / amax:
//   sf = E4M3(a * k), d = E4M3(sf) * s_g, inv = 1 / d, q = E2M1(v * inv).
// Returns the scale code; codes (4 bits each, v[0] lowest) go to `packed`; deq[i] =
// (E2M1(q_i) * E4M3(sf)) * s_g when WANT_DEQ.
template <int N, bool WANT_DEQ>
__device__ __forceinline__ uint32_t quant_nv(const float* v, float s_g, float k,
                                             uint32_t* packed, float* deq) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) a = fmaxf(a, fabsf(v[i]));
  uint32_t sf = 0;
  float sf_val = 0.f, inv = 0.f;
  bool live = false;
  if (s_g > 0.f) {
    sf = cvt_e4m3(__fmul_rn(a, k));
    sf_val = e4m3_value(sf);
    const float d = __fmul_rn(sf_val, s_g);
    live = d > 0.f;
    inv = live ? __frcp_rn(d) : 0.f;
  }
  const float2 inv2 = make_float2(inv, inv);
#pragma unroll
  for (int w = 0; w < N / 8; ++w) {
    const float* s = v + 8 * w;
    const float2 p0 = mul2_rn(make_float2(s[0], s[1]), inv2);
    const float2 p1 = mul2_rn(make_float2(s[2], s[3]), inv2);
    const float2 p2 = mul2_rn(make_float2(s[4], s[5]), inv2);
    const float2 p3 = mul2_rn(make_float2(s[6], s[7]), inv2);
    packed[w] = live ? cvt_e2m1x8(p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y) : 0u;
  }
  if (WANT_DEQ) {
    // E2M1(q) * E4M3(sf) is exact in f16 (at most 6 significant bits, magnitude in
    // [2^-10, 2688]); one float32 rounding for the tensor scale.
    // scalar __fmul_rn: never merged into a multiply-add with the caller's x - deq
    const __half2 sf2 = __float2half2_rn(sf_val);
#pragma unroll
    for (int w = 0; w < N / 8; ++w) {
      uint32_t h[4];
      e2m1x8_to_f16x2(packed[w], h);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(__hmul2(*reinterpret_cast<const __half2*>(&h[j]), sf2));
        deq[8 * w + 2 * j] = __fmul_rn(f.x, s_g);
        deq[8 * w + 2 * j + 1] = __fmul_rn(f.y, s_g);
      }
    }
  }
  return sf;
}

// MXFP4 (OCP MX) quantisation of N values with one E8M0 block scale:
//   e = clamp(floor(log2 a) - 2, -127, 127), q = E2M1(v * 2^-e); a == 0 -> all zero.
template <int N, bool WANT_DEQ>
__device__ __forceinline__ uint32_t quant_mx(const float* v, uint32_t* packed, float* deq) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) a = fmaxf(a, fabsf(v[i]));
  // for normal a the biased exponent field is floor(log2 a) + 127; subnormal a gives 0,
  // which clamps to e = -127 like floor(log2 a) - 2 would
  int e = int((__float_as_uint(a) >> 23) & 0xFFu) - 127 - 2;
  e = max(e, -127);
  const bool live = a > 0.f;
  if (!live) e = -127;
  const float scale = __uint_as_float(uint32_t(127 - e) << 23);  // 2^-e, -e in [-125, 127]
  const float2 sc2 = make_float2(scale, scale);
#pragma unroll
  for (int w = 0; w < N / 8; ++w) {
    const float* s = v + 8 * w;
    const float2 p0 = mul2_rn(make_float2(s[0], s[1]), sc2);
    const float2 p1 = mul2_rn(make_float2(s[2], s[3]), sc2);
    const float2 p2 = mul2_rn(make_float2(s[4], s[5]), sc2);
    const float2 p3 = mul2_rn(make_float2(s[6], s[7]), sc2);
    packed[w] = live ? cvt_e2m1x8(p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y) : 0u;
  }
  if (WANT_DEQ) {
    const float p2 = pow2f(e);
#pragma unroll
    for (int w = 0; w < N / 8; ++w) {
      uint32_t h[4];
      e2m1x8_to_f16x2(packed[w], h);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[j]));
        deq[8 * w + 2 * j] = __fmul_rn(f.x, p2);
        deq[8 * w + 2 * j + 1] = __fmul_rn(f.y, p2);
      }
    }
  }
  return uint32_t(e + 127);
}

// Per-tensor constants of the NVFP4 recipe from amax (one float32 division each).
struct TensorConsts {
  float s_g;  // amax / 2688: the FP32 tensor scale
  float k;    // 448 / amax: block-scale factor
};
__device__ __forceinline__ TensorConsts tensor_consts(float amax) {
  TensorConsts c;
  c.s_g = __fdiv_rn(amax, 2688.0f);
  c.k = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  return c;
}

template <int FMT, int N, bool WANT_DEQ>
__device__ __forceinline__ uint32_t quant_block(const float* v, TensorConsts c, uint32_t* packed,
                                                float* deq) {
  if (FMT == SHARQ_NVFP4) return quant_nv<N, WANT_DEQ>(v, c.s_g, c.k, packed, deq);
  return quant_mx<N, WANT_DEQ>(v, packed, deq);
}

// One block's scale, split from the per-element work so that a kernel can encode values
// of one block in any order: `code` is the scale byte (E4M3 or E8M0), `mul` maps a value
// onto the E2M1 grid (1/d for NVFP4, 2^-e for MXFP4), `sf` is what dequantisation
// multiplies the E2M1 value by (E4M3(sf) for NVFP4, 2^e for MXFP4), and a block that is
// not `live` encodes every value as code 0. Same arithmetic as quant_nv / quant_mx.
struct BlockScale {
  uint32_t code;
  float mul;
  float sf;
  bool live;
};

template <int FMT>
__device__ __forceinline__ BlockScale block_scale(float a, TensorConsts c) {
  BlockScale b;
  if (FMT == SHARQ_NVFP4) {
    b.code = 0;
    b.sf = 0.f;
    b.mul = 0.f;
    b.live = false;
    if (c.s_g > 0.f) {
      b.code = cvt_e4m3(__fmul_rn(a, c.k));
      b.sf = e4m3_value(b.code);
      const float d = __fmul_rn(b.sf, c.s_g);
      b.live = d > 0.f;
      b.mul = b.live ? __frcp_rn(d) : 0.f;
    }
  } else {
    int e = int((__float_as_uint(a) >> 23) & 0xFFu) - 127 - 2;
    e = max(e, -127);
    b.live = a > 0.f;
    if (!b.live) e = -127;
    b.mul = __uint_as_float(uint32_t(127 - e) << 23);
    b.sf = pow2f(e);
    b.code = uint32_t(e + 127);
  }
  return b;
}

// NVFP4 block scale from per-tensor tables: for every E4M3 code c (0..127) of one tensor,
// inv[c] = 1 / (E4M3(c) * s_g) (0 when that product is 0) and sfh[c] = E4M3(c) as an f16
// pair. Built once per CTA after s_g is known; gives exactly block_scale<SHARQ_NVFP4>.
struct NvScaleTable {
  float inv[128];
  uint32_t sfh[128];
};

__device__ __forceinline__ void nv_table_fill(NvScaleTable* t, float s_g, int tid) {
  if (tid < 128) {
    const float sf = e4m3_value(uint32_t(tid));
    const float d = __fmul_rn(sf, s_g);
    t->inv[tid] = d > 0.f ? __frcp_rn(d) : 0.f;
    const __half2 h = __float2half2_rn(sf);
    t->sfh[tid] = *reinterpret_cast<const uint32_t*>(&h);
  }
}

__device__ __forceinline__ BlockScale nv_block_scale(float a, TensorConsts c,
                                                     const NvScaleTable* t) {
  BlockScale b;
  b.code = cvt_e4m3(__fmul_rn(a, c.k));  // k = 0 for an all-zero tensor: code 0
  b.mul = t->inv[b.code];
  b.live = b.mul > 0.f;
  b.sf = __uint_as_float(t->sfh[b.code]);  // f16 pair bits, read by decode8_nv
  return b;
}

// decode8 for a block from nv_block_scale (sf holds the E4M3 value as an f16 pair):
// (E2M1 * E4M3) * s_g per value with one float32 rounding. E2M1 * E4M3 comes from sm_100's
// mixed-precision FMA (f16 sources; the product has at most 6 significant bits, so it is
// exact in float32, and the -0 addend leaves it and the sign of a zero unchanged). The s_g
// product is a packed FMA with a -0 addend: the same single rounding as a multiply. The
// addend is formed at run time (-0 * s_g, s_g finite and >= 0) so that the compiler cannot
// turn the FMA back into a multiply and fuse that with the caller's x - deq.
__device__ __forceinline__ void decode8_nv(uint32_t codes, const BlockScale& b, float s_g,
                                           float* out) {
  uint32_t h[4];
  e2m1x8_to_f16x2(codes, h);
  const uint32_t sfh = __float_as_uint(b.sf);
  const float nz = __fmul_rn(-0.f, s_g);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float lo, hi;
    asm("{\n\t.reg .f16 a0, a1, s0, s1;\n\t"
        "mov.b32 {a0, a1}, %2;\n\tmov.b32 {s0, s1}, %3;\n\t"
        "fma.rn.f32.f16 %0, a0, s0, 0f80000000;\n\t"
        "fma.rn.f32.f16 %1, a1, s0, 0f80000000;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h[j]), "r"(sfh));
    const float2 d = fma2_rn(make_float2(lo, hi), make_float2(s_g, s_g), make_float2(nz, nz));
    out[2 * j] = d.x;
    out[2 * j + 1] = d.y;
  }
}

// 8 values -> 8 E2M1 codes (v[0] in bits 0..3) with a block's multiplier.
__device__ __forceinline__ uint32_t encode8(const float* v, const BlockScale& b) {
  const float2 m2 = make_float2(b.mul, b.mul);
  const float2 p0 = mul2_rn(make_float2(v[0], v[1]), m2);
  const float2 p1 = mul2_rn(make_float2(v[2], v[3]), m2);
  const float2 p2 = mul2_rn(make_float2(v[4], v[5]), m2);
  const float2 p3 = mul2_rn(make_float2(v[6], v[7]), m2);
  const uint32_t c = cvt_e2m1x8(p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y);
  return b.live ? c : 0u;
}

// 8 E2M1 codes -> their dequantised values: NVFP4 (E2M1 * E4M3(sf)) * s_g, the first
// product exact in f16; MXFP4 E2M1 * 2^e.
template <int FMT>
__device__ __forceinline__ void decode8(uint32_t codes, const BlockScale& b, float s_g,
                                        float* out) {
  uint32_t h[4];
  e2m1x8_to_f16x2(codes, h);
  if (FMT == SHARQ_NVFP4) {
    // The s_g product uses the scalar __fmul_rn, which is never merged into a multiply-add:
    // ptxas contracts the packed mul.rn.f32x2 with a following sub.rn.f32x2 (r = x - deq)
    // into one fused operation, which skips this rounding.
    const __half2 sf2 = __float2half2_rn(b.sf);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(__hmul2(*reinterpret_cast<const __half2*>(&h[j]), sf2));
      out[2 * j] = __fmul_rn(f.x, s_g);
      out[2 * j + 1] = __fmul_rn(f.y, s_g);
    }
  } else {
    // E2M1 * 2^e is exact, so a fused x - deq downstream cannot change the result
    const float2 p2 = make_float2(b.sf, b.sf);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = mul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&h[j])), p2);
      out[2 * j] = f.x;
      out[2 * j + 1] = f.y;
    }
  }
}

__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float t;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(t) : "f"(a), "f"(b), "f"(c));
  return t;
}

// max |v| over N values (N = 16 or 32) with the three-input max of sm_100, as a tree of
// depth 3-4 (the preparation is latency-bound; a chain would be N/2 deep)
template <int N>
__device__ __forceinline__ float amax_n(const float* v) {
  static_assert(N == 16 || N == 32, "block of 16 or 32");
  constexpr int T = N / 3;  // full triples
  float m[T + 1];
#pragma unroll
  for (int i = 0; i < T; ++i) m[i] = max3_abs(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  m[T] = max3_abs(v[N - 2], v[N - 1], 0.f);  // N % 3 == 1 or 2: rest (overlap is harmless)
  if (N == 16) {  // 6 partial maxima
    return fmaxf(max3_abs(m[0], m[1], m[2]), max3_abs(m[3], m[4], m[5]));
  }
  // N == 32: 11 partial maxima
  const float n0 = max3_abs(m[0], m[1], m[2]), n1 = max3_abs(m[3], m[4], m[5]);
  const float n2 = max3_abs(m[6], m[7], m[8]), n3 = max3_abs(m[9], m[10], 0.f);
  return fmaxf(max3_abs(n0, n1, n2), n3);
}

// byte offset of (row r, column c) inside a staged tile of 128 rows x C scale columns
__device__ __forceinline__ int tile_off(int r, int c) {
  return (c >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (c & 3);
}

}  // namespace sharq

// Block quantisation recipes shared by the activation and weight kernels (device code).
//
// NVFP4: sf = E4M3_rne((a / 6) / s_g) with a the block's max |v|; d = E4M3(sf) * s_g;
// inv = 1 / d (one correctly rounded reciprocal per block); q = E2M1_rne(v * inv).
// MXFP4 (OCP MX): e = clamp(floor(log2 a) - 2, -127, 127); q = E2M1_rne(v * 2^-e).
// Every float operation is an explicit round-to-nearest intrinsic so that the compiler
// cannot contract or reassociate them.
#pragma once
#include <cstdint>

#include "fp4_device.cuh"
#include "sharq_internal.h"

namespace sharq {

// NVFP4 quantisation of N values with one E4M3 block scale:
//   sf = E4M3((a / 6) / s_g), d = E4M3(sf) * s_g, inv = 1 / d, q = E2M1(v * inv).
// Returns the scale code; codes (4 bits each, v[0] lowest) go to `packed`; deq[i] =
// (E2M1(q_i) * E4M3(sf)) * s_g when want_deq.
template <int N, bool WANT_DEQ>
__device__ __forceinline__ uint32_t quant_nv(const float* v, float s_g, uint32_t* packed,
                                             float* deq) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) a = fmaxf(a, fabsf(v[i]));
  uint32_t sf = 0;
  float sf_val = 0.f, inv = 0.f;
  bool live = false;
  if (s_g > 0.f) {
    sf = cvt_e4m3(__fdiv_rn(__fdiv_rn(a, 6.0f), s_g));
    sf_val = e4m3_value(sf);
    const float d = __fmul_rn(sf_val, s_g);
    live = d > 0.f;
    inv = live ? __frcp_rn(d) : 0.f;
  }
#pragma unroll
  for (int w = 0; w < N / 8; ++w) {
    const float* s = v + 8 * w;
    packed[w] = live ? cvt_e2m1x8(__fmul_rn(s[0], inv), __fmul_rn(s[1], inv),
                                  __fmul_rn(s[2], inv), __fmul_rn(s[3], inv),
                                  __fmul_rn(s[4], inv), __fmul_rn(s[5], inv),
                                  __fmul_rn(s[6], inv), __fmul_rn(s[7], inv))
                     : 0u;
  }
  if (WANT_DEQ) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const uint32_t c = (packed[i / 8] >> (4 * (i % 8))) & 0xFu;
      deq[i] = __fmul_rn(__fmul_rn(e2m1_value(c), sf_val), s_g);
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
#pragma unroll
  for (int w = 0; w < N / 8; ++w) {
    const float* s = v + 8 * w;
    packed[w] = live ? cvt_e2m1x8(__fmul_rn(s[0], scale), __fmul_rn(s[1], scale),
                                  __fmul_rn(s[2], scale), __fmul_rn(s[3], scale),
                                  __fmul_rn(s[4], scale), __fmul_rn(s[5], scale),
                                  __fmul_rn(s[6], scale), __fmul_rn(s[7], scale))
                     : 0u;
  }
  if (WANT_DEQ) {
    const float p2 = pow2f(e);
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const uint32_t c = (packed[i / 8] >> (4 * (i % 8))) & 0xFu;
      deq[i] = __fmul_rn(e2m1_value(c), p2);
    }
  }
  return uint32_t(e + 127);
}

template <int FMT, int N, bool WANT_DEQ>
__device__ __forceinline__ uint32_t quant_block(const float* v, float s_g, uint32_t* packed,
                                                float* deq) {
  if (FMT == SHARQ_NVFP4) return quant_nv<N, WANT_DEQ>(v, s_g, packed, deq);
  return quant_mx<N, WANT_DEQ>(v, packed, deq);
}

// byte offset of (row r, column c) inside a staged tile of 128 rows x C scale columns
__device__ __forceinline__ int tile_off(int r, int c) {
  return (c >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (c & 3);
}

}  // namespace sharq

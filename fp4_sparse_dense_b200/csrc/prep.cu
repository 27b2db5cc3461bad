// Fused SharQ activation preparation for sm_100a (HBM-bound).
//
// SharQ page (pith.science 2606.26587), "Core claim" and abstract: for every activation
// tensor an input-dependent N:M mask picks an outlier-heavy sparse backbone, the backbone
// is rounded to FP4, a dense residual is taken against the rounded backbone and rounded
// to FP4 as well, and the page builds mask selection and residual construction into a
// single fused preparation operator. This file is that operator (plus the tensor-amax
// pass that NVFP4's FP32 tensor scale needs).
//
// Work decomposition: one CTA owns 128 rows x 256 logical K (one metadata slice, whole
// 512-byte scale chunks); one thread owns a "unit" of 32 consecutive K of one row
// (4 mask groups, one backbone block of 16 kept values for the pair-wise mask, one or two
// residual blocks). X is read with 16-byte loads (8 threads cover a 512-byte row
// segment); codes are written with 8/16-byte stores, coalesced along the row; scales and
// metadata are staged in shared memory and written as contiguous 16-byte vectors.
#include <cstdint>
#include <cuda_runtime.h>

#include "fp4_device.cuh"
#include "fp4_quant.cuh"
#include "sharq_internal.h"

namespace sharq {

// ------------------------------------------------------------------------------ amax

// max |x| over the whole tensor, as float bits, combined into *amax_bits by atomicMax
// (non-negative floats order like their bit patterns). *amax_bits must be 0 on entry.
template <bool BF16>
__global__ void __launch_bounds__(512) amax_kernel(const uint4* __restrict__ X, size_t n16,
                                                  unsigned int* amax_bits) {
  uint32_t m = 0;  // two packed 15-bit magnitudes
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n16;
       i += size_t(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(X + i);
    m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
  }
  uint32_t h = max(m & 0xFFFFu, m >> 16);
  for (int off = 16; off; off >>= 1) h = max(h, __shfl_xor_sync(0xFFFFFFFFu, h, off));
  __shared__ uint32_t red[16];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = h;
  __syncthreads();
  if (threadIdx.x < 32) {
    h = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
    for (int off = 16; off; off >>= 1) h = max(h, __shfl_xor_sync(0xFFFFFFFFu, h, off));
    if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(in_to_float<BF16>(h)));
  }
}

// ------------------------------------------------------------------------------ prep

template <bool BF16, int FMT, int MASK, bool RESIDUAL>
__global__ void __launch_bounds__(256) prep_kernel(PrepParams p) {
  constexpr int RB = FMT == SHARQ_NVFP4 ? 16 : 32;                  // residual block
  constexpr int BB = MASK == SHARQ_MASK_PAIR_4_8 ? 32 : RB;         // backbone block (logical)
  constexpr int CB = 256 / BB;                                       // backbone scale cols / CTA
  constexpr int CR = 256 / RB;                                       // residual scale cols / CTA
  constexpr bool PAIR = MASK == SHARQ_MASK_PAIR_4_8;

  __shared__ __align__(16) uint8_t s_bs[128 * CB];
  __shared__ __align__(16) uint8_t s_rs[RESIDUAL ? 128 * CR : 16];
  __shared__ __align__(16) uint8_t s_bm[PAIR ? 128 * 16 : 16];

  const int q = blockIdx.x;           // 256-K slice
  const int rb = blockIdx.y;          // 128-row block
  const int u = threadIdx.x & 7;      // 32-K unit inside the slice
  const int k0 = q * 256 + u * 32;    // first logical K of the unit
  const int K = p.K;

  float s_g = 1.f;
  if (FMT == SHARQ_NVFP4) {
    s_g = __fdiv_rn(__uint_as_float(*reinterpret_cast<const unsigned int*>(p.amax)), 2688.0f);
    if (q == 0 && rb == 0 && threadIdx.x == 0) *p.tensor_scale = s_g;
  } else if (q == 0 && rb == 0 && threadIdx.x == 0) {
    *p.tensor_scale = 1.0f;
  }

#pragma unroll 1
  for (int it = 0; it < 4; ++it) {
    const int rl = it * 32 + (threadIdx.x >> 3);  // row inside the block
    const int r = rb * 128 + rl;
    if (r >= p.M) {  // padding row: zero scales, valid "pairs 0,1" metadata
      s_bs[tile_off(rl, u * (32 / BB))] = 0;
      if (BB == 16) s_bs[tile_off(rl, u * 2 + 1)] = 0;
      if (RESIDUAL) {
        s_rs[tile_off(rl, u * (32 / RB))] = 0;
        if (RB == 16) s_rs[tile_off(rl, u * 2 + 1)] = 0;
      }
      if (PAIR) *reinterpret_cast<uint16_t*>(s_bm + rl * 16 + u * 2) = 0x4444;
      continue;
    }
    // ---- load 32 input elements (64 bytes)
    const uint4* src = reinterpret_cast<const uint4*>(
        static_cast<const uint16_t*>(p.X) + size_t(r) * K + k0);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 t = __ldg(src + i);
      w[4 * i + 0] = t.x; w[4 * i + 1] = t.y; w[4 * i + 2] = t.z; w[4 * i + 3] = t.w;
    }
    float x[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      x[2 * i] = in_to_float<BF16>(w[i] & 0xFFFFu);
      x[2 * i + 1] = in_to_float<BF16>(w[i] >> 16);
    }

    float r_val[32];  // residual before quantisation
    uint32_t meta = 0;

    if (PAIR) {
      // ---- pair-wise 4:8 mask: per group of 8, keep the 2 of 4 adjacent pairs with the
      // largest (max |x|, min |x|), ties to the lower pair. Magnitudes compare as the
      // 15-bit patterns of the 16-bit inputs; the pair index breaks ties.
      float comp[16];
      int sel0[4], sel1[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t key[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t word = w[4 * g + j];
          const uint32_t a = word & 0x7FFFu, b = (word >> 16) & 0x7FFFu;
          key[j] = (max(a, b) << 17) | (min(a, b) << 2) | uint32_t(3 - j);
        }
        const int c01 = key[0] > key[1], c02 = key[0] > key[2], c03 = key[0] > key[3];
        const int c12 = key[1] > key[2], c13 = key[1] > key[3], c23 = key[2] > key[3];
        const bool k0p = (3 - c01 - c02 - c03) < 2;
        const bool k1p = (c01 + 2 - c12 - c13) < 2;
        const bool k2p = (c02 + c12 + 1 - c23) < 2;
        const int i0 = k0p ? 0 : (k1p ? 1 : 2);
        const int i1 = (c03 + c13 + c23) < 2 ? 3 : (k2p ? 2 : 1);
        (void)k2p;
        sel0[g] = i0;
        sel1[g] = i1;
        meta |= uint32_t(i0 | (i1 << 2)) << (4 * g);
        const float* xg = x + 8 * g;
        comp[4 * g + 0] = i0 == 0 ? xg[0] : (i0 == 1 ? xg[2] : xg[4]);
        comp[4 * g + 1] = i0 == 0 ? xg[1] : (i0 == 1 ? xg[3] : xg[5]);
        comp[4 * g + 2] = i1 == 3 ? xg[6] : (i1 == 2 ? xg[4] : xg[2]);
        comp[4 * g + 3] = i1 == 3 ? xg[7] : (i1 == 2 ? xg[5] : xg[3]);
      }
      // ---- backbone: one block of the 16 kept values
      uint32_t bcodes[2];
      float deq[16];
      const uint32_t bsf = quant_block<FMT, 16, RESIDUAL>(comp, s_g, bcodes, deq);
      s_bs[tile_off(rl, u)] = uint8_t(bsf);
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.bq) + size_t(r) * (K / 4) + k0 / 4) =
          make_uint2(bcodes[0], bcodes[1]);
      *reinterpret_cast<uint16_t*>(s_bm + rl * 16 + u * 2) = uint16_t(meta);
      if (RESIDUAL) {
        // ---- residual against the quantised backbone
#pragma unroll
        for (int g = 0; g < 4; ++g) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float xv = x[8 * g + 2 * j + e];
              const float d0 = deq[4 * g + e], d1 = deq[4 * g + 2 + e];
              r_val[8 * g + 2 * j + e] =
                  sel0[g] == j ? __fsub_rn(xv, d0) : (sel1[g] == j ? __fsub_rn(xv, d1) : xv);
            }
          }
        }
      }
    } else {
      // ---- element 2:4 mask: per group of 4 keep the 2 largest |x|, ties to the lower index
      float b[32];
      uint32_t kept = 0;  // bit i: element i of the unit is on the backbone
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint32_t key[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t h = (j & 1) ? (w[2 * g + (j >> 1)] >> 16) : (w[2 * g + (j >> 1)] & 0xFFFFu);
          key[j] = ((h & 0x7FFFu) << 2) | uint32_t(3 - j);
        }
        const int c01 = key[0] > key[1], c02 = key[0] > key[2], c03 = key[0] > key[3];
        const int c12 = key[1] > key[2], c13 = key[1] > key[3], c23 = key[2] > key[3];
        const bool kp[4] = {(3 - c01 - c02 - c03) < 2, (c01 + 2 - c12 - c13) < 2,
                            (c02 + c12 + 1 - c23) < 2, (c03 + c13 + c23) < 2};
        const int i0 = kp[0] ? 0 : (kp[1] ? 1 : 2);
        const int i1 = kp[3] ? 3 : (kp[2] ? 2 : 1);
        meta |= uint32_t(i0 | (i1 << 2)) << (4 * g);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          b[4 * g + j] = kp[j] ? x[4 * g + j] : 0.f;
          kept |= uint32_t(kp[j]) << (4 * g + j);
        }
      }
      uint32_t bcodes[4];
      float deq[32];
      if (BB == 16) {
        const uint32_t s0 = quant_block<FMT, 16, RESIDUAL>(b, s_g, bcodes, deq);
        const uint32_t s1 = quant_block<FMT, 16, RESIDUAL>(b + 16, s_g, bcodes + 2, deq + 16);
        s_bs[tile_off(rl, 2 * u)] = uint8_t(s0);
        s_bs[tile_off(rl, 2 * u + 1)] = uint8_t(s1);
      } else {
        const uint32_t s0 = quant_block<FMT, 32, RESIDUAL>(b, s_g, bcodes, deq);
        s_bs[tile_off(rl, u)] = uint8_t(s0);
      }
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.bq) + size_t(r) * (K / 2) + k0 / 2) =
          make_uint4(bcodes[0], bcodes[1], bcodes[2], bcodes[3]);
      *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.bm) + size_t(r) * (K / 8) + k0 / 8) =
          meta;
      if (RESIDUAL) {
#pragma unroll
        for (int i = 0; i < 32; ++i) r_val[i] = (kept >> i) & 1u ? __fsub_rn(x[i], deq[i]) : x[i];
      }
    }

    if (RESIDUAL) {
      uint32_t rcodes[4];
      if (RB == 16) {
        const uint32_t s0 = quant_block<FMT, 16, false>(r_val, s_g, rcodes, nullptr);
        const uint32_t s1 = quant_block<FMT, 16, false>(r_val + 16, s_g, rcodes + 2, nullptr);
        s_rs[tile_off(rl, 2 * u)] = uint8_t(s0);
        s_rs[tile_off(rl, 2 * u + 1)] = uint8_t(s1);
      } else {
        const uint32_t s0 = quant_block<FMT, 32, false>(r_val, s_g, rcodes, nullptr);
        s_rs[tile_off(rl, u)] = uint8_t(s0);
      }
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.rq) + size_t(r) * (K / 2) + k0 / 2) =
          make_uint4(rcodes[0], rcodes[1], rcodes[2], rcodes[3]);
    }
  }
  __syncthreads();

  // ---- write the staged scale / metadata tiles as contiguous 16-byte vectors
  const int Mp = p.Mp;
  {
    uint8_t* dst = static_cast<uint8_t*>(p.bs) +
                   (size_t(rb) * (K / BB / 4) + size_t(q) * (CB / 4)) * 512;
    for (int i = threadIdx.x; i < 128 * CB / 16; i += 256)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(s_bs)[i];
  }
  if (RESIDUAL) {
    uint8_t* dst = static_cast<uint8_t*>(p.rs) +
                   (size_t(rb) * (K / RB / 4) + size_t(q) * (CR / 4)) * 512;
    for (int i = threadIdx.x; i < 128 * CR / 16; i += 256)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(s_rs)[i];
  }
  if (PAIR) {
    uint8_t* dst = static_cast<uint8_t*>(p.bm) + size_t(q) * Mp * 16 + size_t(rb) * 2048;
    for (int i = threadIdx.x; i < 128; i += 256)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(s_bm)[i];
  }
}

// ------------------------------------------------------------------------------ launch

template <bool BF16, int FMT, int MASK, bool RES>
static cudaError_t launch_prep_t(const PrepParams& p, cudaStream_t st) {
  dim3 grid(p.K / 256, (p.M + 127) / 128);
  prep_kernel<BF16, FMT, MASK, RES><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

template <bool BF16, int FMT, int MASK>
static cudaError_t launch_prep_r(const PrepParams& p, bool res, cudaStream_t st) {
  return res ? launch_prep_t<BF16, FMT, MASK, true>(p, st)
             : launch_prep_t<BF16, FMT, MASK, false>(p, st);
}

template <bool BF16, int FMT>
static cudaError_t launch_prep_m(const PrepParams& p, int mask, bool res, cudaStream_t st) {
  return mask == SHARQ_MASK_PAIR_4_8 ? launch_prep_r<BF16, FMT, SHARQ_MASK_PAIR_4_8>(p, res, st)
                                     : launch_prep_r<BF16, FMT, SHARQ_MASK_ELEM_2_4>(p, res, st);
}

template <bool BF16>
static cudaError_t launch_prep_f(const PrepParams& p, int fmt, int mask, bool res,
                                 cudaStream_t st) {
  return fmt == SHARQ_NVFP4 ? launch_prep_m<BF16, SHARQ_NVFP4>(p, mask, res, st)
                            : launch_prep_m<BF16, SHARQ_MXFP4>(p, mask, res, st);
}

cudaError_t launch_amax(const void* X, bool bf16, size_t n_elems, unsigned int* amax_bits,
                        int num_sms, cudaStream_t st) {
  const size_t n16 = n_elems / 8;
  size_t blocks = (n16 + 511) / 512;
  const size_t cap = size_t(num_sms) * 4;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) blocks = 1;
  if (bf16)
    amax_kernel<true><<<unsigned(blocks), 512, 0, st>>>(static_cast<const uint4*>(X), n16, amax_bits);
  else
    amax_kernel<false><<<unsigned(blocks), 512, 0, st>>>(static_cast<const uint4*>(X), n16, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepParams& p, bool bf16, int fmt, int mask, bool residual,
                        cudaStream_t st) {
  return bf16 ? launch_prep_f<true>(p, fmt, mask, residual, st)
              : launch_prep_f<false>(p, fmt, mask, residual, st);
}

}  // namespace sharq

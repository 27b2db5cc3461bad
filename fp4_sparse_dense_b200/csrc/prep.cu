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
#include <type_traits>
#include <cuda_runtime.h>

#include "fp4_device.cuh"
#include "fp4_quant.cuh"
#include "sharq_internal.h"
#include "sm100_ptx.cuh"

namespace sharq {

// ------------------------------------------------------------------------------ amax

// max |x| over the whole tensor, as float bits, combined into *amax_bits by atomicMax
// (non-negative floats order like their bit patterns). *amax_bits must be 0 on entry.
template <bool BF16>
__global__ void __launch_bounds__(512) amax_kernel(const uint4* __restrict__ X, size_t n16,
                                                  unsigned int* amax_bits) {
  uint32_t m = 0;  // two packed 15-bit magnitudes
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  // four independent 16-byte loads in flight per thread
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      v[j] = i + j * stride < n16 ? __ldg(X + i + j * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = __vmaxu2(m, v[j].x & 0x7FFF7FFFu);
      m = __vmaxu2(m, v[j].y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v[j].z & 0x7FFF7FFFu);
      m = __vmaxu2(m, v[j].w & 0x7FFF7FFFu);
    }
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

// NVFP4 tensor amax across the two preparation kernels, in words 2..3 of the caller's
// tensor-scale buffer (zero before the first call): the first kernel (the mask kernel, or
// with RMSNorm absorbed the rstd kernel) folds max |x| into `acc` with atomicMax; every CTA of the quantisation kernel reads it once and counts
// itself in `done`, and the CTA that completes the count sets both back to zero for the
// next call. No CTA waits for another.
struct AmaxState {
  unsigned acc;   // max |x| as float bits (non-negative floats order like their bits)
  unsigned done;  // CTAs of the quantisation kernel that have read acc
};

// CTA max of the threads' packed 15-bit magnitudes (two per word), folded into st->acc.
template <bool BF16>
__device__ void block_max_to(uint32_t m, AmaxState* st) {
  __shared__ unsigned s_red[8];
  uint32_t h = max(m & 0xFFFFu, m >> 16);
  for (int off = 16; off; off >>= 1) h = max(h, __shfl_xor_sync(0xFFFFFFFFu, h, off));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = h;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) b = max(b, s_red[i]);
    atomicMax(&st->acc, __float_as_uint(in_to_float<BF16>(b)));
  }
}

// ------------------------------------------------------------------------------ RMSNorm

// One word of two 16-bit inputs x normalised with rstd r and weights g:
// y = round16((x * r) * g) per value (float32 products, one rounding each, then RNE to the
// input's 16-bit format).
template <bool BF16>
__device__ __forceinline__ uint32_t norm_word(uint32_t x, uint32_t g, float r) {
  const float lo = __fmul_rn(__fmul_rn(in_to_float<BF16>(x & 0xFFFFu), r),
                             in_to_float<BF16>(g & 0xFFFFu));
  const float hi = __fmul_rn(__fmul_rn(in_to_float<BF16>(x >> 16), r),
                             in_to_float<BF16>(g >> 16));
  uint32_t y;
  if (BF16) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(y) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(y) : "f"(hi), "f"(lo));
  }
  return y;
}

// Per-row rstd = 1 / sqrt(mean_k x^2 + eps), the RMSNorm that the preparation absorbs (the
// SharQ page's fused operator takes in layer normalisation; RMSNorm is that of the
// Llama/Qwen models it evaluates). One warp per row. The float32 order is fixed so that the
// result is reproducible: chunk c of 8 elements belongs to lane c mod 32, each lane adds
// its chunks' squares in increasing k, then a butterfly over lanes (xor 16, 8, 4, 2, 1).
// Squares of 16-bit inputs are exact; every addition and the division, square root and
// reciprocal round to nearest once. AMAX (NVFP4): a second pass over the row (from L1/L2)
// forms the normalised values y exactly as the quantisation kernel will and folds max |y|
// into the tensor amax, so that no separate mask kernel has to read X again; the
// quantisation kernel then computes the mask itself.
template <bool BF16, bool AMAX>
__global__ void __launch_bounds__(256) rms_kernel(PrepParams p) {
  ptx::griddep_wait();  // X may come from the kernel launched just before
  ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const uint32_t chunks = uint32_t(p.K) / 8;
  uint32_t mx = 0;  // AMAX: packed 15-bit magnitudes of y
  for (int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < p.M; row += warps) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.X) +
                                                      uint32_t(row) * uint32_t(p.K));
    float acc = 0.f;
#pragma unroll 4
    for (uint32_t c = lane; c < chunks; c += 32) {
      const uint4 v = __ldg(src + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = in_to_float<BF16>(w[i] & 0xFFFFu), hi = in_to_float<BF16>(w[i] >> 16);
        acc = __fadd_rn(acc, __fmul_rn(lo, lo));
        acc = __fadd_rn(acc, __fmul_rn(hi, hi));
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, off));
    // the butterfly leaves the same sum in every lane (each step adds the same two values)
    const float r = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(acc, float(p.K)), p.eps)));
    if (lane == 0) p.rstd[row] = r;
    if (AMAX) {
      const uint4* g4 = static_cast<const uint4*>(p.gamma);
#pragma unroll 4
      for (uint32_t c = lane; c < chunks; c += 32) {
        const uint4 v = __ldg(src + c), gv = __ldg(g4 + c);
        mx = __vmaxu2(mx, norm_word<BF16>(v.x, gv.x, r) & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, norm_word<BF16>(v.y, gv.y, r) & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, norm_word<BF16>(v.z, gv.z, r) & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, norm_word<BF16>(v.w, gv.w, r) & 0x7FFF7FFFu);
      }
    }
  }
  if (AMAX) block_max_to<BF16>(mx, reinterpret_cast<AmaxState*>(p.tensor_scale + 2));
}

// y = round16((x * rstd) * gamma) for the 32 inputs of one unit (16 words of two 16-bit
// values, k0 the unit's first column): the normalised input the preparation then sees.
template <bool BF16>
__device__ __forceinline__ void rms_apply(uint32_t* w, const PrepParams& p, int row,
                                          uint32_t k0) {
  const float r = __ldg(p.rstd + row);
  const uint4* g4 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.gamma) + k0);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 gv = __ldg(g4 + c);
    const uint32_t g[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) w[4 * c + i] = norm_word<BF16>(w[4 * c + i], g[i], r);
  }
}

// ------------------------------------------------------------------------------ pair 4:8

// Entry of the top-2-of-4 decision table. Bit b of `idx` is one comparison "candidate i
// beats candidate j" (i < j; a tie is won by i) in the order (0,1) (0,2) (0,3) (1,2)
// (1,3) (2,3). A candidate is kept when fewer than two others beat it. The entry packs
//   bits  0..15  byte selector that keeps the kept pairs' code bytes and zeroes the others
//   bits 16..23  byte selector of the two kept bytes (i0, i1) in order
//   bits 24..27  metadata nibble i0 | i1 << 2 (i0 < i1)
__device__ __forceinline__ uint32_t top2_entry(int idx) {
  const int c01 = idx & 1, c02 = (idx >> 1) & 1, c03 = (idx >> 2) & 1;
  const int c12 = (idx >> 3) & 1, c13 = (idx >> 4) & 1, c23 = (idx >> 5) & 1;
  const int rank[4] = {3 - c01 - c02 - c03, c01 + 2 - c12 - c13, c02 + c12 + 1 - c23,
                       c03 + c13 + c23};
  int i0 = -1, i1 = -1;
  for (int j = 0; j < 4; ++j)
    if (rank[j] < 2) {
      if (i0 < 0) i0 = j;
      else if (i1 < 0) i1 = j;
    }
  if (i0 < 0 || i1 < 0) {  // not reachable from a total order
    i0 = 0;
    i1 = 1;
  }
  uint32_t keep = 0;
  for (int j = 0; j < 4; ++j) keep |= uint32_t(j == i0 || j == i1 ? j : 4) << (4 * j);
  return keep | (uint32_t(i0 | (i1 << 4)) << 16) | (uint32_t(i0 | (i1 << 2)) << 24);
}

template <bool BF16>
__device__ __forceinline__ float lo16(uint32_t w) {
  return BF16 ? __uint_as_float(w << 16) : in_to_float<false>(w & 0xFFFFu);
}
template <bool BF16>
__device__ __forceinline__ float hi16(uint32_t w) {
  return BF16 ? __uint_as_float(w & 0xFFFF0000u) : in_to_float<false>(w >> 16);
}


// Table entry of a metadata nibble i0 | i1 << 2 (same packing as top2_entry); nibbles that
// the mask never produces map to pairs (0, 1).
__device__ __forceinline__ uint32_t nibble_entry(int nib) {
  int i0 = nib & 3, i1 = nib >> 2;
  if (!(i0 < i1)) {
    i0 = 0;
    i1 = 1;
  }
  uint32_t keep = 0;
  for (int j = 0; j < 4; ++j) keep |= uint32_t(j == i0 || j == i1 ? j : 4) << (4 * j);
  return keep | (uint32_t(i0 | (i1 << 4)) << 16) | (uint32_t(i0 | (i1 << 2)) << 24);
}

// Pair-wise 4:8 mask of one 32-K unit (16 words of two 16-bit inputs): one table entry per
// group of 4 pairs from the pair keys (max |x| << 16 | min |x|, as 15-bit magnitudes); the
// comparison bits are the sign bits of key_j - key_i - 1, shifted in from (2,3) down to
// (0,1). Returns the unit's 4 metadata nibbles; folds the magnitudes into *mx.
__device__ __forceinline__ uint32_t pair_mask(const uint32_t* w, const uint32_t* top2,
                                              uint32_t* L, uint32_t* mx) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t k[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t m = w[4 * g + j] & 0x7FFF7FFFu;
      *mx = __vmaxu2(*mx, m);
      k[j] = max(m, __byte_perm(m, 0, 0x1032));
    }
    uint32_t idx = (k[3] - k[2] - 1u) >> 31;
    idx = __funnelshift_l(k[3] - k[1] - 1u, idx, 1);
    idx = __funnelshift_l(k[2] - k[1] - 1u, idx, 1);
    idx = __funnelshift_l(k[3] - k[0] - 1u, idx, 1);
    idx = __funnelshift_l(k[2] - k[0] - 1u, idx, 1);
    idx = __funnelshift_l(k[1] - k[0] - 1u, idx, 1);
    L[g] = top2[idx];
  }
  return ((L[0] >> 24) & 0xFu) | ((L[1] >> 20) & 0xF0u) | ((L[2] >> 16) & 0xF00u) |
         ((L[3] >> 12) & 0xF000u);
}

// Warp items of the pair-mask kernels: an item is 4 rows x 256 K (lane = row * 8 + unit,
// unit = 32 K); warps walk the items with a grid stride. Offsets are 32-bit: sharq_prepare
// admits M * K < 2^31 only.
struct PairWalk {
  int K, M, Mp, KS, n_items, u, stride, stride_q, stride_r, first, q0, row0;
  const uint16_t* X;
  uint8_t* bm;

  __device__ __forceinline__ PairWalk(const PrepParams& p) {
    K = p.K;
    M = p.M;
    Mp = p.Mp;
    KS = K / 256;
    n_items = (Mp / 4) * KS;
    const int lane = threadIdx.x & 31;
    u = lane & 7;
    stride = gridDim.x * (blockDim.x >> 5);
    stride_q = stride % KS;
    stride_r = (stride / KS) * 4;
    first = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    q0 = first % KS;
    row0 = (first / KS) * 4 + (lane >> 3);
    X = static_cast<const uint16_t*>(p.X);
    bm = static_cast<uint8_t*>(p.bm);
  }
  __device__ __forceinline__ void load(int it, int r, int q, uint4* dst) const {
    if (it < n_items && r < M) {
      const uint4* src = reinterpret_cast<const uint4*>(
          X + (uint32_t(r) * uint32_t(K) + uint32_t(q) * 256u + uint32_t(u) * 32u));
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = __ldg(src + i);
    }
  }
  __device__ __forceinline__ void advance(int& q, int& r) const {
    q += stride_q;
    r += stride_r;
    if (q >= KS) {
      q -= KS;
      r += 4;
    }
  }
  // metadata: 4 nibbles per lane, the row's 16 bytes at slice q
  __device__ __forceinline__ uint32_t meta_off(int q, int r) const {
    return uint32_t(q) * uint32_t(Mp) * 16u + uint32_t(r) * 16u + uint32_t(u) * 2u;
  }
  // lanes u, u+1 -> one 32-bit store (whole warp)
  __device__ __forceinline__ void store_meta(int q, int r, uint32_t meta) const {
    const uint32_t m16 = meta & 0xFFFFu;
    const uint32_t word = m16 | (__shfl_down_sync(0xFFFFFFFFu, m16, 1) << 16);
    if ((u & 1) == 0) *reinterpret_cast<uint32_t*>(bm + meta_off(q, r)) = word;
  }
};

__device__ __forceinline__ void unpack16(const uint4* c, uint32_t* w) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[4 * i + 0] = c[i].x; w[4 * i + 1] = c[i].y;
    w[4 * i + 2] = c[i].z; w[4 * i + 3] = c[i].w;
  }
}

// First NVFP4 preparation kernel (pair mask): streams X from HBM, computes the mask, writes
// the metadata (padding rows included) and folds max |x| into the tensor amax. Its integer
// work hides under the HBM reads.
template <bool BF16, bool NORM, bool ABL>
__global__ void __launch_bounds__(256) prep_mask_kernel(PrepParams p) {
  const bool mask_given = ABL && p.mask_given;  // ablation flags compile away unless ABL
  __shared__ uint32_t s_top2[64];
  if (threadIdx.x < 64) s_top2[threadIdx.x] = top2_entry(threadIdx.x);
  __syncthreads();
  ptx::griddep_wait();  // X (and rstd) come from the kernels launched before
  // Only now may the quantisation kernel start: once it runs, the kernels that produced X
  // have completed, so it may read X before its own wait. It waits (griddepcontrol.wait)
  // for this grid's completion before it reads anything written here.
  ptx::griddep_launch_dependents();
  const PairWalk wk(p);
  uint32_t mx = 0;
  int q = wk.q0, row = wk.row0;
  uint4 cur[4];
  wk.load(wk.first, row, q, cur);
#pragma unroll 1
  for (int item = wk.first; item < wk.n_items; item += wk.stride) {
    int nq = q, nrow = row;
    wk.advance(nq, nrow);
    uint4 nxt[4];
    wk.load(item + wk.stride, nrow, nq, nxt);
    uint32_t meta = 0x4444u;  // padding rows: pairs 0, 1
    if (row < wk.M) {
      uint32_t w[16], L[4];
      unpack16(cur, w);
      if (NORM) rms_apply<BF16>(w, p, row, uint32_t(q) * 256u + uint32_t(wk.u) * 32u);
      if (mask_given) {  // ablation: the caller's mask stays in bm; only max |x| here
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = __vmaxu2(mx, w[i] & 0x7FFF7FFFu);
      } else {
        meta = pair_mask(w, s_top2, L, &mx);
      }
    }
    if (!mask_given) wk.store_meta(q, row, meta);
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    q = nq;
    row = nrow;
  }
  block_max_to<BF16>(mx, reinterpret_cast<AmaxState*>(p.tensor_scale + 2));
}

// Pair-wise 4:8 mask: in every 8 consecutive K keep the 2 of the 4 adjacent pairs with the
// largest (max |x|, min |x|), ties to the lower pair; the kept values (compressed, 16 per
// 32 K) form one backbone block; the residual is taken against their dequantised values.
//
// Persistent and warp-independent (PairWalk), loading the next item while computing the
// current one. Scale and metadata bytes of neighbouring lanes are gathered with shuffles
// into 32-bit stores, so no CTA barrier is needed inside the loop. NVFP4 runs after
// prep_mask_kernel and takes the mask from its metadata and the tensor amax from its
// reduction; MXFP4 (no tensor scale), NVFP4 with RMSNorm absorbed (the amax comes from the
// rstd kernel) and NVFP4 with a supplied amax compute the mask inline.
//
// Per unit the backbone is encoded at all 32 positions with the block's scale (its max
// |x| is the unit's max |x|: the largest element of every group of 8 lies in its top pair,
// which is kept); byte permutes then keep the kept pairs' code bytes, either compressed
// (the backbone operand) or in place with zeros elsewhere, which dequantise to the backbone
// at kept positions and +0 elsewhere, so r = x - deq needs no per-element selection.
//
// GIVEN (NVFP4): the tensor amax is supplied by the caller (p.amax_in), so this is the
// only kernel of the call and it computes the mask itself.
template <bool BF16, int FMT, bool RESIDUAL, bool NORM, bool ABL, bool GIVEN = false>
__global__ void __launch_bounds__(256, ABL ? 1 : 3) prep_pair_kernel(PrepParams p) {
  constexpr bool NV = FMT == SHARQ_NVFP4;
  // ablation flags compile away unless ABL (the method's instantiation stays lean)
  const bool mask_given = ABL && p.mask_given, res_unquant = ABL && p.res_unquant;
  // residual with its own tensor scale (NVFP4, the two-accumulator variant): phase 1 writes
  // the backbone and folds max |r| into a second amax state; phase 2 recomputes the same
  // backbone and r and writes the residual quantised with s_r = amax|r| / 2688
  const int res_phase = (ABL && NV && RESIDUAL) ? p.res_phase : 0;
  constexpr int RB = NV ? 16 : 32;  // residual block
  __shared__ uint32_t s_top2[64];
  __shared__ uint32_t s_nib[16];
  __shared__ NvScaleTable s_nv;
  struct NoTable {};
  __shared__ std::conditional_t<ABL && NV && RESIDUAL, NvScaleTable, NoTable> s_nvr;
  __shared__ float s_amax, s_amax_r;
  __shared__ unsigned s_rmax[8];
  if (threadIdx.x < 64) s_top2[threadIdx.x] = top2_entry(threadIdx.x);
  if (threadIdx.x < 16) s_nib[threadIdx.x] = nibble_entry(threadIdx.x);
  const PairWalk wk(p);
  int q = wk.q0, row = wk.row0;
  uint4 cur[4];
  // NVFP4: launched as a programmatic dependent of prep_mask_kernel, which releases it only
  // after its own wait, so X is final here and the first item's load overlaps that kernel's
  // tail; the wait below returns once the mask kernel's writes (amax, metadata) are visible.
  // MXFP4 is the first kernel of the call: X may come from the kernel launched just before.
  if (NV && !GIVEN) wk.load(wk.first, row, q, cur);
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();  // the GEMM that follows may start its prologue
  if (!NV || GIVEN) wk.load(wk.first, row, q, cur);
  AmaxState* const amax_st = reinterpret_cast<AmaxState*>(p.tensor_scale + 2);
  AmaxState* const amax_r_st = reinterpret_cast<AmaxState*>(p.tensor_scale + 4);
  if (NV && threadIdx.x == 0) {
    if (GIVEN) {
      s_amax = *p.amax_in;
    } else if (res_phase == 2) {  // amax|X| as phase 1 wrote it; amax|r| from phase 1's reduction
      s_amax = *reinterpret_cast<volatile float*>(p.tensor_scale + 1);
      s_amax_r = __uint_as_float(*reinterpret_cast<volatile unsigned*>(&amax_r_st->acc));
    } else {
      s_amax = __uint_as_float(*reinterpret_cast<volatile unsigned*>(&amax_st->acc));
    }
  }
  __syncthreads();
  TensorConsts tc{1.f, 1.f}, tcr{1.f, 1.f};
  if constexpr (NV) {
    tc = tensor_consts(s_amax);
    nv_table_fill(&s_nv, tc.s_g, threadIdx.x);
    if (res_phase == 2) {
      tcr = tensor_consts(s_amax_r);
      if constexpr (ABL && RESIDUAL) nv_table_fill(&s_nvr, tcr.s_g, threadIdx.x);
      if (blockIdx.x == 0 && threadIdx.x == 0) {
        p.tensor_scale[6] = tcr.s_g;
        p.tensor_scale[7] = s_amax_r;
      }
    } else if (blockIdx.x == 0 && threadIdx.x == 0) {
      p.tensor_scale[0] = tc.s_g;
      p.tensor_scale[1] = s_amax;
    }
  } else if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.tensor_scale[0] = 1.0f;
  }
  __syncthreads();  // decision and scale tables ready
  float r_max = 0.f;  // phase 1: running max |r| of this thread

  const int K = wk.K, M = wk.M, u = wk.u;
  const uint32_t scols_b = uint32_t(K) / 32 / 4;  // 512-byte chunks per 128 rows (backbone)
  const uint32_t scols_r = uint32_t(K) / RB / 4;  // (residual)

  // one block's scale; NVFP4 through the per-tensor table
  auto scale_of = [&](float a) {
    if constexpr (NV) return nv_block_scale(a, tc, &s_nv);
    else return block_scale<FMT>(a, tc);
  };
  // the residual's blocks: the backbone's table, or phase 2's table of s_r
  auto scale_of_r = [&](float a) {
    if constexpr (NV && ABL && RESIDUAL) {
      if (res_phase == 2) return nv_block_scale(a, tcr, &s_nvr);
    }
    return scale_of(a);
  };
  auto decode_of = [&](uint32_t codes, const BlockScale& b, float* out) {
    if constexpr (NV) decode8_nv(codes, b, tc.s_g, out);
    else decode8<FMT>(codes, b, tc.s_g, out);
  };
  // mask read back from bm (written by prep_mask_kernel, or supplied), else computed here
  // (MXFP4, and NVFP4 with RMSNorm absorbed, where the rstd kernel supplies the amax)
  const bool meta_in = (NV && !(NORM && !ABL) && !GIVEN) || mask_given;
  auto load_meta = [&](int it, int r, int q) -> uint32_t {
    if (!meta_in || it >= wk.n_items || r >= M) return 0x4444u;
    return __ldcg(reinterpret_cast<const unsigned short*>(wk.bm + wk.meta_off(q, r)));
  };

  uint32_t cmeta = load_meta(wk.first, row, q);

  // two items per loop trip for the NVFP4 method (measured about 2 % faster on a
  // 4096 x 4096 tensor), one otherwise
#pragma unroll (NV && !ABL ? 2 : 1)
  for (int item = wk.first; item < wk.n_items; item += wk.stride) {
    int nq = q, nrow = row;
    wk.advance(nq, nrow);
    uint4 nxt[4];
    wk.load(item + wk.stride, nrow, nq, nxt);
    const uint32_t nmeta = load_meta(item + wk.stride, nrow, nq);
    const uint32_t k0 = uint32_t(q) * 256u + uint32_t(u) * 32u;
    const bool live = row < M;

    uint32_t meta = 0x4444u, bsf = 0, rsf0 = 0, rsf1 = 0;
    if (live) {
      uint32_t w[16], L[4];
      unpack16(cur, w);
      if (NORM) rms_apply<BF16>(w, p, row, k0);
      if (meta_in) {
        meta = cmeta;
#pragma unroll
        for (int g = 0; g < 4; ++g) L[g] = s_nib[(meta >> (4 * g)) & 0xFu];
      } else {
        uint32_t unused = 0;
        meta = pair_mask(w, s_top2, L, &unused);
      }

      float x[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        x[2 * i] = lo16<BF16>(w[i]);
        x[2 * i + 1] = hi16<BF16>(w[i]);
      }
      // ---- backbone: one block of 32 logical K. With the adaptive mask its max |x| is the
      // unit's; a supplied mask may drop a group's largest element, so then the max runs
      // over the kept values only.
      float a_b;
      if (mask_given) {
        float xk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          xk[i] = ((L[i >> 3] >> (4 * ((i & 7) >> 1))) & 0xFu) != 4u ? x[i] : 0.f;
        a_b = amax_n<32>(xk);
      } else {
        a_b = amax_n<32>(x);
      }
      const BlockScale bb = scale_of(a_b);
      bsf = bb.code;
      uint32_t c[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) c[g] = encode8(x + 8 * g, bb);
      // compressed backbone codes: the kept bytes of groups 0, 1 and of groups 2, 3 (the
      // selector takes bytes i0, i1 of the first word and 4 + i0, 4 + i1 of the second)
      const uint32_t sel01 = __byte_perm(L[0], L[1], 0x0062u) + 0x4400u;
      const uint32_t sel23 = __byte_perm(L[2], L[3], 0x0062u) + 0x4400u;
      if (res_phase != 2)
        *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.bq) +
                                  (uint32_t(row) * uint32_t(K / 4) + k0 / 4)) =
            make_uint2(__byte_perm(c[0], c[1], sel01), __byte_perm(c[2], c[3], sel23));
      if (RESIDUAL) {
        // ---- residual against the quantised backbone
        float r[32];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float d[8];
          if (res_unquant) {  // ablation: against the unquantised backbone
#pragma unroll
            for (int j = 0; j < 8; ++j)
              d[j] = ((L[g] >> (4 * (j >> 1))) & 0xFu) != 4u ? x[8 * g + j] : 0.f;
          } else {
            decode_of(__byte_perm(c[g], 0u, L[g]), bb, d);
          }
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            const float2 t = sub2_rn(make_float2(x[8 * g + j], x[8 * g + j + 1]),
                                     make_float2(d[j], d[j + 1]));
            r[8 * g + j] = t.x;
            r[8 * g + j + 1] = t.y;
          }
        }
        uint32_t rc[4];
        if (res_phase == 1) {
          r_max = fmaxf(r_max, amax_n<32>(r));
        } else {
#pragma unroll
          for (int hb = 0; hb < 32 / RB; ++hb) {
            const BlockScale rb = scale_of_r(amax_n<RB>(r + hb * RB));
            if (hb == 0) rsf0 = rb.code; else rsf1 = rb.code;
#pragma unroll
            for (int g = 0; g < RB / 8; ++g)
              rc[hb * (RB / 8) + g] = encode8(r + hb * RB + 8 * g, rb);
          }
          *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.rq) +
                                    (uint32_t(row) * uint32_t(K / 2) + k0 / 2)) =
              make_uint4(rc[0], rc[1], rc[2], rc[3]);
        }
      }
    }

    // ---- scales (and MXFP4 metadata): gather neighbouring lanes' bytes into 32-bit stores
    const uint32_t rq32 = uint32_t(row & 31) * 16u + uint32_t((row >> 5) & 3) * 4u;
    if (res_phase != 2) {
      // backbone scale column q*8+u: lanes u..u+3 form one 4-byte word
      uint32_t word = bsf;
      word |= __shfl_down_sync(0xFFFFFFFFu, bsf, 1) << 8;
      word |= __shfl_down_sync(0xFFFFFFFFu, bsf, 2) << 16;
      word |= __shfl_down_sync(0xFFFFFFFFu, bsf, 3) << 24;
      if ((u & 3) == 0) {
        const uint32_t chunk = uint32_t(row >> 7) * scols_b + uint32_t(q) * 2u + uint32_t(u >> 2);
        *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.bs) + (chunk * 512u + rq32)) = word;
      }
    }
    if (RESIDUAL && res_phase != 1) {
      if constexpr (RB == 16) {
        // residual scale columns q*16+2u, +1: lanes u, u+1 form one 4-byte word
        const uint32_t two = rsf0 | (rsf1 << 8);
        const uint32_t word = two | (__shfl_down_sync(0xFFFFFFFFu, two, 1) << 16);
        if ((u & 1) == 0) {
          const uint32_t chunk = uint32_t(row >> 7) * scols_r + uint32_t(q) * 4u + uint32_t(u >> 1);
          *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.rs) + (chunk * 512u + rq32)) = word;
        }
      } else {
        uint32_t word = rsf0;
        word |= __shfl_down_sync(0xFFFFFFFFu, rsf0, 1) << 8;
        word |= __shfl_down_sync(0xFFFFFFFFu, rsf0, 2) << 16;
        word |= __shfl_down_sync(0xFFFFFFFFu, rsf0, 3) << 24;
        if ((u & 3) == 0) {
          const uint32_t chunk = uint32_t(row >> 7) * scols_r + uint32_t(q) * 2u + uint32_t(u >> 2);
          *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.rs) + (chunk * 512u + rq32)) = word;
        }
      }
    }
    if (!meta_in) wk.store_meta(q, row, meta);
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    cmeta = nmeta;
    q = nq;
    row = nrow;
  }
  if (res_phase == 1) {  // fold max |r| into the second amax state (one atomic per CTA)
    uint32_t h = __float_as_uint(r_max);
    for (int off = 16; off; off >>= 1) h = max(h, __shfl_xor_sync(0xFFFFFFFFu, h, off));
    if ((threadIdx.x & 31) == 0) s_rmax[threadIdx.x >> 5] = h;
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t b = 0;
      for (int i = 0; i < int(blockDim.x >> 5); ++i) b = max(b, s_rmax[i]);
      atomicMax(&amax_r_st->acc, b);
    }
  }
  // NVFP4: the last CTA to finish resets the amax state it read for the next call (every
  // CTA read acc at its start; the fence orders that read before this CTA is counted)
  if (NV && !GIVEN && threadIdx.x == 0) {
    AmaxState* const st = res_phase == 2 ? amax_r_st : amax_st;
    __threadfence();
    if (atomicAdd(&st->done, 1u) == gridDim.x - 1) {
      st->acc = 0u;
      st->done = 0u;
    }
  }
}


// ------------------------------------------------------------------------------ element 2:4

// Element-wise 2:4 mask (every 4 consecutive K keep the 2 largest |x|, ties to the lower
// index); the backbone is stored zero-filled for the dense MMA.

template <bool BF16, int FMT, bool RESIDUAL>
__global__ void __launch_bounds__(256) prep_elem_kernel(PrepParams p) {
  constexpr int MASK = SHARQ_MASK_ELEM_2_4;
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

  TensorConsts tc{1.f, 1.f};
  if (FMT == SHARQ_NVFP4) {
    tc = tensor_consts(__uint_as_float(*reinterpret_cast<const unsigned int*>(p.amax)));
    if (q == 0 && rb == 0 && threadIdx.x == 0) *p.tensor_scale = tc.s_g;
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

    {
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
        const bool all = p.keep_all != 0;  // ablation: no mask, plain FP4 of x
        const bool kp[4] = {all || (3 - c01 - c02 - c03) < 2, all || (c01 + 2 - c12 - c13) < 2,
                            all || (c02 + c12 + 1 - c23) < 2, all || (c03 + c13 + c23) < 2};
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
        const uint32_t s0 = quant_block<FMT, 16, RESIDUAL>(b, tc, bcodes, deq);
        const uint32_t s1 = quant_block<FMT, 16, RESIDUAL>(b + 16, tc, bcodes + 2, deq + 16);
        s_bs[tile_off(rl, 2 * u)] = uint8_t(s0);
        s_bs[tile_off(rl, 2 * u + 1)] = uint8_t(s1);
      } else {
        const uint32_t s0 = quant_block<FMT, 32, RESIDUAL>(b, tc, bcodes, deq);
        s_bs[tile_off(rl, u)] = uint8_t(s0);
      }
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.bq) + size_t(r) * (K / 2) + k0 / 2) =
          make_uint4(bcodes[0], bcodes[1], bcodes[2], bcodes[3]);
      if (!p.keep_all)
        *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.bm) + size_t(r) * (K / 8) + k0 / 8) =
            meta;
      if (RESIDUAL) {
        // ablation res_unquant: against the unquantised backbone (x - x = +0 where kept)
#pragma unroll
        for (int i = 0; i < 32; ++i)
          r_val[i] = (kept >> i) & 1u ? __fsub_rn(x[i], p.res_unquant ? x[i] : deq[i]) : x[i];
      }
    }

    if (RESIDUAL) {
      uint32_t rcodes[4];
      if (RB == 16) {
        const uint32_t s0 = quant_block<FMT, 16, false>(r_val, tc, rcodes, nullptr);
        const uint32_t s1 = quant_block<FMT, 16, false>(r_val + 16, tc, rcodes + 2, nullptr);
        s_rs[tile_off(rl, 2 * u)] = uint8_t(s0);
        s_rs[tile_off(rl, 2 * u + 1)] = uint8_t(s1);
      } else {
        const uint32_t s0 = quant_block<FMT, 32, false>(r_val, tc, rcodes, nullptr);
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

// launch with the programmatic-stream-serialization attribute: the kernel may start while
// the previous one in the stream finishes and waits (griddepcontrol.wait) for its results
// Beside a GEMM (alongside) the launch also asks for the largest shared-memory carveout, so
// that an SM running one of these CTAs can still take a GEMM CTA that needs nearly all of
// its shared memory without reconfiguring; alone the default split keeps L1 large for the
// X stream.
template <typename... Args>
static cudaError_t launch_pdl_t(void (*kern)(Args...), unsigned blocks, unsigned threads,
                                bool alongside, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributePreferredSharedMemoryCarveout;
  attr[1].val.sharedMemCarveout = unsigned(cudaSharedmemCarveoutMaxShared);
  cfg.attrs = attr;
  cfg.numAttrs = alongside ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}
template <typename... Args>
static cudaError_t launch_pdl(void (*kern)(Args...), unsigned blocks, cudaStream_t st,
                              Args... args) {
  return launch_pdl_t(kern, blocks, 256u, false, st, args...);
}

// CTAs of a persistent preparation kernel: enough warp items for every warp, at most what
// fits on the GPU at once (resident CTAs per SM from the occupancy calculator, cached).
// Beside a GEMM (p.alongside): one CTA per SM of `threads` threads.
template <typename Kern>
static cudaError_t persistent_blocks(Kern kern, int* per_sm, const PrepParams& p, int num_sms,
                                     unsigned* blocks, unsigned threads = 256) {
  if (*per_sm == 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, kern, 256, 0);
    if (e != cudaSuccess) return e;
    if (*per_sm < 1) *per_sm = 1;
  }
  const long items = long(p.Mp / 4) * (p.K / 256);
  const long warps = threads / 32;
  long b = (items + warps - 1) / warps;
  const long cap = long(num_sms) * (p.alongside ? 1 : *per_sm);
  *blocks = unsigned(b < cap ? b : cap);
  return cudaSuccess;
}

// threads per CTA of the quantisation kernel: beside a GEMM the SM has about 16 K registers
// left, so 128 threads (4 warps at up to 80 registers); alone 256
static unsigned quant_threads(const PrepParams& p) { return p.alongside ? 128u : 256u; }

template <bool BF16, int FMT, bool RES, bool NORM, bool ABL>
static cudaError_t launch_prep_t(const PrepParams& p, int mask, int num_sms, cudaStream_t st) {
  if (FMT == SHARQ_NVFP4 && !NORM && !ABL && p.amax_in && is_pair_mask(mask)) {
    // the caller's tensor amax: one kernel, mask computed inline
    auto kern = prep_pair_kernel<BF16, FMT, RES, false, false, true>;
    static int per_sm = 0;
    unsigned blocks = 0;
    const unsigned qt = quant_threads(p);
    cudaError_t e = persistent_blocks(kern, &per_sm, p, num_sms, &blocks, qt);
    if (e != cudaSuccess) return e;
    if ((e = launch_pdl_t(kern, blocks, qt, p.alongside != 0, st, p)) != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (is_pair_mask(mask)) {
    cudaError_t e = cudaSuccess;
    // NVFP4 + RMSNorm (the method): the rstd kernel also reduces the tensor amax of the
    // normalised X, and the quantisation kernel computes the mask (no mask kernel)
    constexpr bool NORM_AMAX = NORM && !ABL && FMT == SHARQ_NVFP4;
    if (NORM && p.res_phase != 2) {  // per-row rstd first: one warp per row
      long rb = (long(p.M) + 7) / 8;
      if (rb > long(num_sms) * 8) rb = long(num_sms) * 8;
      e = launch_pdl(rms_kernel<BF16, NORM_AMAX>, unsigned(rb), st, p);
      if (e != cudaSuccess) return e;
    }
    if (FMT == SHARQ_NVFP4 && !NORM_AMAX && p.res_phase != 2) {
      auto mk = prep_mask_kernel<BF16, NORM, ABL>;
      static int mk_per_sm = 0;
      unsigned mb = 0;
      if ((e = persistent_blocks(mk, &mk_per_sm, p, num_sms, &mb)) != cudaSuccess) return e;
      if ((e = launch_pdl_t(mk, mb, 256u, p.alongside != 0, st, p)) != cudaSuccess) return e;
    }
    auto kern = prep_pair_kernel<BF16, FMT, RES, NORM, ABL>;
    static int per_sm = 0;
    unsigned blocks = 0;
    const unsigned qt = quant_threads(p);
    if ((e = persistent_blocks(kern, &per_sm, p, num_sms, &blocks, qt)) != cudaSuccess) return e;
    e = launch_pdl_t(kern, blocks, qt, p.alongside != 0, st, p);
    if (e != cudaSuccess) return e;
  } else {
    if (NORM) return cudaErrorNotSupported;
    dim3 grid(p.K / 256, (p.M + 127) / 128);
    prep_elem_kernel<BF16, FMT, RES><<<grid, 256, 0, st>>>(p);
  }
  return cudaGetLastError();
}

template <bool BF16, int FMT, bool RES, bool NORM>
static cudaError_t launch_prep_a(const PrepParams& p, int mask, int num_sms, cudaStream_t st) {
  const bool abl = p.mask_given || p.res_unquant || p.res_phase != 0;
  return abl ? launch_prep_t<BF16, FMT, RES, NORM, true>(p, mask, num_sms, st)
             : launch_prep_t<BF16, FMT, RES, NORM, false>(p, mask, num_sms, st);
}

template <bool BF16, int FMT, bool RES>
static cudaError_t launch_prep_n(const PrepParams& p, int mask, bool norm, int n, cudaStream_t st) {
  return norm ? launch_prep_a<BF16, FMT, RES, true>(p, mask, n, st)
              : launch_prep_a<BF16, FMT, RES, false>(p, mask, n, st);
}

template <bool BF16, int FMT>
static cudaError_t launch_prep_r(const PrepParams& p, int mask, bool res, bool norm, int n,
                                 cudaStream_t st) {
  return res ? launch_prep_n<BF16, FMT, true>(p, mask, norm, n, st)
             : launch_prep_n<BF16, FMT, false>(p, mask, norm, n, st);
}

template <bool BF16>
static cudaError_t launch_prep_f(const PrepParams& p, int fmt, int mask, bool res, bool norm,
                                 int n, cudaStream_t st) {
  return fmt == SHARQ_NVFP4 ? launch_prep_r<BF16, SHARQ_NVFP4>(p, mask, res, norm, n, st)
                            : launch_prep_r<BF16, SHARQ_MXFP4>(p, mask, res, norm, n, st);
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
                        int num_sms, cudaStream_t st) {
  const bool norm = p.gamma != nullptr;
  return bf16 ? launch_prep_f<true>(p, fmt, mask, residual, norm, num_sms, st)
              : launch_prep_f<false>(p, fmt, mask, residual, norm, num_sms, st);
}

}  // namespace sharq

// Offline weight quantisation for the SharQ linear layer (sm_100a).
//
// SharQ page (pith.science 2606.26587), abstract: the sparse and the dense GEMM read one
// FP4 weight payload, each through its own view of the scales. W[K x N] is transposed to
// K-major FP4 codes [N][K/2] once; its block scales are written twice, in the layout and
// granularity each MMA consumes: the dense view (one scale per 16 K for NVFP4, 32 for
// MXFP4) and, for the pair-wise sparse path, the sparse view (one scale per 32 logical
// K). With the pair-wise mask the codes are quantised with 32-element blocks so that the
// same codes are exact under both views (the dense view repeats each scale twice).
//
// One CTA quantises 32 output rows x 256 K: the W tile is staged in shared memory
// (coalesced along N), then each thread quantises 32 consecutive K of one output row.
#include <cstdint>
#include <cuda_runtime.h>

#include "fp4_device.cuh"
#include "fp4_quant.cuh"
#include "sharq_internal.h"

namespace sharq {

// byte offset of scale (row r, column c) in the 128x4-tiled layout with `ncols` columns
__device__ __forceinline__ size_t tiled_offset(int r, int c, int ncols) {
  const size_t chunk = size_t(r >> 7) * size_t(ncols >> 2) + size_t(c >> 2);
  return chunk * 512 + size_t(r & 31) * 16 + size_t((r >> 5) & 3) * 4 + size_t(c & 3);
}

template <bool BF16, int FMT, int BW, bool SPARSE_VIEW>
__global__ void __launch_bounds__(256) weight_quant_kernel(WeightQuantParams p) {
  constexpr int GD = FMT == SHARQ_NVFP4 ? 16 : 32;  // dense-view granularity
  constexpr int PITCH = 34;                          // 32 columns + 2 (bank spread)
  __shared__ uint16_t tile[256 * PITCH];
  const int n0 = blockIdx.x * 32, k_base = blockIdx.y * 256;
  const int K = p.K, N = p.N;
  {
    // row k_base + t: 32 consecutive N elements (64 bytes)
    const int k = k_base + threadIdx.x;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.W) +
                                                      size_t(k) * N + n0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        tile[threadIdx.x * PITCH + 8 * i + 2 * h] = uint16_t(w[h] & 0xFFFFu);
        tile[threadIdx.x * PITCH + 8 * i + 2 * h + 1] = uint16_t(w[h] >> 16);
      }
    }
  }
  TensorConsts tc{1.f, 1.f};
  if (FMT == SHARQ_NVFP4) {
    tc = tensor_consts(p.tensor_scale[1]);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) p.tensor_scale[0] = tc.s_g;
  } else if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    p.tensor_scale[0] = 1.0f;
  }
  __syncthreads();

  const int nl = threadIdx.x & 31, u = threadIdx.x >> 5;
  const int n = n0 + nl, k0 = k_base + u * 32;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = in_to_float<BF16>(tile[(u * 32 + i) * PITCH + nl]);

  uint32_t codes[4];
  uint32_t sc[2];
  if (BW == 16) {
    sc[0] = quant_block<FMT, 16, false>(v, tc, codes, nullptr);
    sc[1] = quant_block<FMT, 16, false>(v + 16, tc, codes + 2, nullptr);
  } else {
    sc[0] = sc[1] = quant_block<FMT, 32, false>(v, tc, codes, nullptr);
  }
  *reinterpret_cast<uint4*>(p.codes + size_t(n) * (K / 2) + k0 / 2) =
      make_uint4(codes[0], codes[1], codes[2], codes[3]);
  if (GD == 16) {
    p.scales_dense[tiled_offset(n, k0 / 16, K / 16)] = uint8_t(sc[0]);
    p.scales_dense[tiled_offset(n, k0 / 16 + 1, K / 16)] = uint8_t(sc[1]);
  } else {
    p.scales_dense[tiled_offset(n, k0 / 32, K / 32)] = uint8_t(sc[0]);
  }
  if (SPARSE_VIEW) p.scales_sparse[tiled_offset(n, k0 / 32, K / 32)] = uint8_t(sc[0]);
}

template <bool BF16, int FMT, int BW, bool SV>
static cudaError_t launch_wq_t(const WeightQuantParams& p, cudaStream_t st) {
  dim3 grid(p.N / 32, p.K / 256);
  weight_quant_kernel<BF16, FMT, BW, SV><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

template <bool BF16>
static cudaError_t launch_wq_b(const WeightQuantParams& p, int fmt, int mask, cudaStream_t st) {
  const bool pair = is_pair_mask(mask);
  if (fmt == SHARQ_NVFP4)
    return pair ? launch_wq_t<BF16, SHARQ_NVFP4, 32, true>(p, st)
                : launch_wq_t<BF16, SHARQ_NVFP4, 16, false>(p, st);
  return pair ? launch_wq_t<BF16, SHARQ_MXFP4, 32, true>(p, st)
              : launch_wq_t<BF16, SHARQ_MXFP4, 32, false>(p, st);
}

cudaError_t launch_weight_quant(const WeightQuantParams& p, bool bf16, int fmt, int mask,
                                cudaStream_t st) {
  return bf16 ? launch_wq_b<true>(p, fmt, mask, st) : launch_wq_b<false>(p, fmt, mask, st);
}

}  // namespace sharq

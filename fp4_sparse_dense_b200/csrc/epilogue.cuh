// GEMM epilogue store of one warp's accumulator rows (device code shared by both GEMMs).
//
// A warp owns 32 output rows (its tensor-memory lane quarter) and `COLS` columns held as
// unscaled FP32 in registers, one row per lane. bf16 output: every 32-column slice is
// scaled, converted and written to a 2 KB shared staging box (64-byte swizzle, so that the
// 32 lanes' row writes spread over all banks) and sent to global memory by one tensor
// store: whole 64-byte row segments instead of per-lane scattered 16-byte pieces, and the
// warp goes on while the copy engine writes. float output (a debugging aid) is stored
// directly.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace sharq {

template <int COLS>
__device__ __forceinline__ void store_rows_bf16(const CUtensorMap* ymap, uint32_t stage_smem,
                                                const uint32_t* v, float alpha, int row0,
                                                int col0, int lane) {
#pragma unroll
  for (int c = 0; c < COLS / 32; ++c) {
    // the previous box must have been read out of the staging buffer
    if (lane == 0) ptx::bulk_wait_read_all();
    __syncwarp();
    uint32_t w[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) {
      const __nv_bfloat162 b2 =
          __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[32 * c + 2 * h]), alpha),
                                __fmul_rn(__uint_as_float(v[32 * c + 2 * h + 1]), alpha));
      w[h] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    const uint32_t row_base = stage_smem + uint32_t(lane) * 64u;
    const uint32_t sw = uint32_t((lane >> 1) & 3);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t addr = row_base + ((uint32_t(j) ^ sw) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * j]),
                   "r"(w[4 * j + 1]), "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                   : "memory");
    }
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      ptx::tma_store_2d(ymap, stage_smem, col0 + 32 * c, row0);
      ptx::bulk_commit_group();
    }
  }
}

template <int COLS>
__device__ __forceinline__ void store_rows_f32(float* Y, int M, int N, const uint32_t* v,
                                               float alpha, int row, int col0) {
  if (row >= M) return;
  float4* dst = reinterpret_cast<float4*>(Y + size_t(row) * N + col0);
#pragma unroll
  for (int i = 0; i < COLS / 4; ++i)
    dst[i] = make_float4(__fmul_rn(__uint_as_float(v[4 * i]), alpha),
                         __fmul_rn(__uint_as_float(v[4 * i + 1]), alpha),
                         __fmul_rn(__uint_as_float(v[4 * i + 2]), alpha),
                         __fmul_rn(__uint_as_float(v[4 * i + 3]), alpha));
}

}  // namespace sharq

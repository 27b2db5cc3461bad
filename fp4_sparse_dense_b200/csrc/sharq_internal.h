// Internal declarations shared by the SharQ CUDA translation units (not part of the ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sharq.h"

namespace sharq {

struct PrepParams {
  const void* X;        // [M][K] 16-bit
  void* bq;
  void* bs;
  void* bm;
  void* rq;
  void* rs;
  float* tensor_scale;  // [0] = s_g, [1] = amax (written); [2..5] amax state (pair mask, NVFP4)
  const float* amax;    // = tensor_scale + 1 (element mask, NVFP4: written by amax_kernel)
  int M, K, Mp;
  unsigned* status;     // device status word (bounded-wait timeouts)
  unsigned long long timeout_ns;
  // RMSNorm absorbed into the preparation (null gamma: X is prepared as given)
  const void* gamma;    // [K] 16-bit, same dtype as X
  float* rstd;          // [M] per-row 1 / sqrt(mean x^2 + eps), written by rms_kernel
  float eps;
  // ablation modes (runtime flags: not on the method's path)
  int mask_given;       // pair mask read from bm instead of chosen per row
  int keep_all;         // no mask: every element on the (dense) backbone
  int res_unquant;      // residual against the unquantised backbone
  int alongside;        // launch sized to run beside a GEMM on another stream
  int res_phase;        // residual with its own tensor scale: 1 backbone + amax|r|, 2 residual
  const float* amax_in; // NVFP4: the caller's tensor amax (device), else nullptr
};

struct WeightQuantParams {
  const void* W;           // [K][N] 16-bit
  uint8_t* codes;          // [N][K/2]
  uint8_t* scales_dense;   // tiled N x K/GD
  uint8_t* scales_sparse;  // tiled N x K/32 (pair mask) or null
  float* tensor_scale;     // [0] = s_gw (written), [1] = amax (NVFP4, read)
  int K, N;
};

struct GemmParams {
  const uint8_t* bs;   // backbone scales (tiled)
  const uint8_t* bm;   // pair metadata
  const uint8_t* rs;   // residual scales (tiled)
  const uint8_t* wsd;  // weight scales, dense view
  const uint8_t* wss;  // weight scales, sparse view
  const float* act_ts;
  const float* w_ts;
  void* Y;
  int M, N, K, Mp;
  int tiles_m, tiles_n;
  // tile order of the persistent CTA-pair kernel: 0 = M fastest (consecutive tiles share a
  // weight tile; the whole activation operand is reused from L2 across the N columns),
  // 1 = N fastest (consecutive tiles share activation rows; the whole weight is reused)
  int n_fast;
  // one-CTA kernel: load the weight part of the first stages before waiting for the kernel
  // launched before it (decode-sized M, where the weight stream dominates)
  int prefetch_w;
  int splits;  // K ranges per output tile (1: no split; >1: partials in ws, then a reduction)
  float* ws;   // split-K partials [splits][M][N] (caller-owned workspace)
  unsigned int* status;
  unsigned long long timeout_ns;
};

cudaError_t launch_amax(const void* X, bool bf16, size_t n_elems, unsigned int* amax_bits,
                        int num_sms, cudaStream_t st);
cudaError_t launch_prep(const PrepParams& p, bool bf16, int fmt, int mask, bool residual,
                        int num_sms, cudaStream_t st);
cudaError_t launch_weight_quant(const WeightQuantParams& p, bool bf16, int fmt, int mask,
                                cudaStream_t st);

// maps for the three FP4 operands, built by the host side
struct GemmMaps {
  CUtensorMap w, b, r, y;  // y: bf16 output, 32 x 32 boxes (unused for float output)
};
// residual with its own tensor scale (two accumulators), NVFP4 pair mask, 128-wide tiles
cudaError_t launch_gemm_two(const GemmMaps& maps, const GemmParams& p, bool out_f32, int num_sms,
                            cudaStream_t st);
cudaError_t launch_gemm(const GemmMaps& maps, const GemmParams& p, int fmt, int mask,
                        bool residual, bool out_f32, int num_sms, cudaStream_t st);

// maps of the CTA-pair kernel: the three FP4 operands plus byte views [bytes/256][256] of
// the scale and metadata buffers (loaded by tensor copies so that both CTAs can count them
// on the pair leader's barrier)
struct GemmPairMaps {
  CUtensorMap w, b, r, rs, bs, bm, wsd, wss, y;
};
cudaError_t launch_gemm_pair(const GemmPairMaps& maps, const GemmParams& p, int fmt, int mask,
                             bool residual, bool out_f32, int num_sms, cudaStream_t st);

// Unique id of the current CUDA context (initialises the primary context if none is
// current); per-context caches key on it.
sharq_status current_context_id(unsigned long long* id);

// masks whose backbone is stored compressed and runs through the sparse MMA
inline bool is_pair_mask(int mask) {
  return mask == SHARQ_MASK_PAIR_4_8 || mask == SHARQ_MASK_PAIR_4_8_GIVEN;
}

// block sizes along K
inline int residual_block(int fmt) { return fmt == SHARQ_NVFP4 ? 16 : 32; }
inline int backbone_block(int fmt, int mask) {
  return is_pair_mask(mask) ? 32 : residual_block(fmt);
}
inline int weight_block(int fmt, int mask) {
  if (fmt == SHARQ_MXFP4) return 32;
  return is_pair_mask(mask) ? 32 : 16;
}
inline int dense_view_block(int fmt) { return fmt == SHARQ_NVFP4 ? 16 : 32; }

// Split-K plan of the one-CTA kernel: when the output has too few tiles to occupy the SMs,
// split K so that tiles x splits roughly covers them (each split keeps >= 2 K steps).
inline int plan_splits(int M, int N, int K, int num_sms) {
  if (M >= 256 && N % 256 == 0) return 1;  // CTA-pair kernel, enough tiles
  const int BN = (N % 256 == 0) ? 256 : 128;
  const int tiles = ((M + 127) / 128) * (N / BN);
  const int KT = K / 256;
  if (tiles * 2 > num_sms || KT < 4) return 1;
  int s = num_sms / tiles;
  if (s > KT / 2) s = KT / 2;
  return s < 1 ? 1 : s;
}

}  // namespace sharq

// SharQ sparse + dense FP4 GEMM over CTA pairs (tcgen05 cta_group::2), for M >= 256.
//
// Same computation as gemm.cu (SharQ page, pith.science 2606.26587, "Core claim": the
// backbone through a structured-sparse FP4 GEMM and the residual through a dense FP4 GEMM,
// both over one FP4 weight payload, summed into one accumulator), on a 256 x 256 output
// tile shared by the two CTAs of a cluster. Each CTA holds its own 128 activation rows
// and one half (128 rows along N) of the weight tile; the pair MMA reads the weight halves
// of both CTAs, so each CTA streams only half of the weight from L2 (the one-CTA kernel
// is bound by L2 -> SM traffic at prefill sizes).
//
// Protocol (leader = cluster rank 0):
//   * every load of both CTAs (FP4 tiles, scales, metadata; all tensor maps) counts
//     its bytes on the leader's `full` barrier of the stage; the leader arms it for the
//     bytes of both CTAs;
//   * the leader's single MMA thread copies scales / metadata into both CTAs' tensor
//     memory (tcgen05.cp cta_group::2), issues the pair MMAs and releases the stage in both
//     CTAs with one multicast tcgen05.commit; after the last K step a second multicast
//     commit tells both epilogues that their accumulator rows are ready;
//   * each CTA's epilogue drains its own 128 accumulator rows and reports to the leader's
//     `tempty` barrier (one arrival per warp), then scales, converts and stores.
// No load uses cluster multicast. Every wait is bounded (see sm100_ptx.cuh).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sharq_internal.h"
#include "epilogue.cuh"
#include "sm100_ptx.cuh"

namespace sharq {

namespace {

constexpr int kPairMaxSmem = 232448;
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;

template <int FMT, bool PAIR, bool RES>
struct PairCfg {
  static constexpr bool NV = FMT == SHARQ_NVFP4;
  static constexpr int BN = 256;                 // N of the pair tile
  static constexpr int GD = NV ? 16 : 32;        // dense-view scale granularity
  static constexpr int DCH = 256 / GD / 4;       // 512-byte scale chunks per K step (dense)
  static constexpr bool DENSE_W = RES || !PAIR;  // any dense MMA issued
  // bytes per stage in ONE CTA
  static constexpr int W_BYTES = 128 * 128;      // this CTA's half of the weight tile
  static constexpr int R_BYTES = RES ? 128 * 128 : 0;
  static constexpr int B_BYTES = PAIR ? 128 * 64 : 128 * 128;
  static constexpr int SFR_BYTES = RES ? DCH * 512 : 0;
  static constexpr int SFB_BYTES = PAIR ? 2 * 512 : DCH * 512;
  static constexpr int SWD_BYTES = DENSE_W ? 2 * DCH * 512 : 0;  // both weight halves
  static constexpr int SWS_BYTES = PAIR ? 2 * 2 * 512 : 0;
  static constexpr int E_BYTES = PAIR ? 2048 : 0;
  static constexpr int OFF_W = 0;
  static constexpr int OFF_R = OFF_W + W_BYTES;
  static constexpr int OFF_B = OFF_R + R_BYTES;
  static constexpr int OFF_SFR = OFF_B + B_BYTES;
  static constexpr int OFF_SFB = OFF_SFR + SFR_BYTES;
  static constexpr int OFF_SWD = OFF_SFB + SFB_BYTES;
  static constexpr int OFF_SWS = OFF_SWD + SWD_BYTES;
  static constexpr int OFF_E = OFF_SWS + SWS_BYTES;
  static constexpr int STAGE_RAW = OFF_E + E_BYTES;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int TX_PAIR = 2 * STAGE_RAW;  // bytes of both CTAs, counted by the leader
  static constexpr int EPI_BYTES = kPairEpiWarps * 2048;  // 32 x 32 bf16 box per warp
  static constexpr int STAGES_FIT = (kPairMaxSmem - 2048 - EPI_BYTES) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  // stages, 1 KB of barriers, the epilogue staging, 1 KB alignment slack
  static constexpr int SMEM = STAGES * STAGE + 1024 + EPI_BYTES + 1024;
  // tensor-memory columns (same in both CTAs)
  static constexpr int COL_SFR = 256;
  static constexpr int COL_SFB = COL_SFR + (RES ? DCH * 4 : 0);
  static constexpr int COL_SWD = COL_SFB + (PAIR ? 8 : DCH * 4);
  static constexpr int COL_SWS = COL_SWD + (DENSE_W ? DCH * (BN / 32) : 0);
  static constexpr int COL_E = COL_SWS + (PAIR ? 2 * (BN / 32) : 0);
  static constexpr int COL_END = COL_E + (PAIR ? 4 : 0);
  static constexpr int SF_SPAN = (COL_END - COL_SFR + 3) / 4 * 4;
  static_assert(COL_SFR + 2 * SF_SPAN <= 512, "tensor memory overflow");
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  // block-scaled instruction descriptor: E2M1 A and B, M = 256 (pair), N = 256
  static constexpr uint32_t IDESC_BASE =
      (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(256 >> 4) << 24);
  static constexpr uint32_t SCALE_FMT = NV ? 0u : (1u << 23);
};

// Shared-memory matrix descriptors of one stage buffer at one add each (the MMA thread
// issues some thirty per K step, alone in its warp, so their arithmetic is on its critical
// path). Every address in a stage is 16-byte aligned and below 256 KB, so the descriptor's
// 14-bit address field of base + off is the base's plus off >> 4 with no carry; the leading
// byte offset is 16 bytes throughout. Same bits as ptx::smem_desc.
struct StageDesc {
  uint32_t lo;  // address field of the stage base | leading byte offset field
  __device__ __forceinline__ explicit StageDesc(uint32_t base) : lo((base >> 4) | (1u << 16)) {}
  template <uint32_t SBO, uint32_t LAYOUT>
  __device__ __forceinline__ uint64_t at(uint32_t off) const {
    constexpr uint32_t hi = ((SBO >> 4) & 0x3FFFu) | (1u << 14) | ((LAYOUT & 7u) << 29);
    return (uint64_t(hi) << 32) | uint64_t(lo + (off >> 4));
  }
};

}  // namespace

template <int FMT, bool PAIR, bool RES, bool OUT_F32>
__global__ void __launch_bounds__(kPairThreads, 1)
    sharq_gemm_pair_kernel(const __grid_constant__ GemmPairMaps m, const GemmParams p) {
  using C = PairCfg<FMT, PAIR, RES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + C::STAGES * C::STAGE;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty_bar = full_bar + C::STAGES;
  uint64_t* tfull_bar = empty_bar + C::STAGES;
  uint64_t* tempty_bar = tfull_bar + 1;
  uint64_t* drain_bar = tempty_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int KT = p.K / 256;
  const int tiles_m2 = (p.M + 255) / 256;
  const int pair_tiles = tiles_m2 * p.tiles_n;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int last_rb = p.Mp / 128 - 1;  // last 128-row block the padded scale buffers hold

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(ptx::smem_u32(full_bar + s), 1);
      ptx::mbar_init(ptx::smem_u32(empty_bar + s), 1);
    }
    ptx::mbar_init(ptx::smem_u32(tfull_bar), 1);
    ptx::mbar_init(ptx::smem_u32(tempty_bar), 2 * kPairEpiWarps);
    ptx::mbar_init(ptx::smem_u32(drain_bar), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tensormap(&m.w);
    ptx::prefetch_tensormap(&m.b);
    if (RES) ptx::prefetch_tensormap(&m.r);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
  ptx::tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t limit = p.timeout_ns;
  // launched as a programmatic dependent: the set-up above overlapped the previous kernel;
  // nothing it wrote (the operands) is read before this point
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  // the leader's copies of the barriers (the pair's loads and epilogues report there)
  const uint32_t lead_full0 = ptx::mapa(ptx::smem_u32(full_bar), 0);
  const uint32_t lead_tempty = ptx::mapa(ptx::smem_u32(tempty_bar), 0);

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    if (ptx::elect_one()) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = cluster; t < pair_tiles && ok; t += n_clusters) {
        const int mb2 = p.n_fast ? t / p.tiles_n : t % tiles_m2;
        const int nb = p.n_fast ? t % p.tiles_n : t / tiles_m2;
        const int rb = mb2 * 2 + int(rank);               // this CTA's 128-row block
        const int rb_sf = rb < last_rb ? rb : last_rb;    // in-bounds block for scales
        for (int kt = 0; kt < KT; ++kt) {
          if (!ptx::mbar_wait(ptx::smem_u32(empty_bar + s), ph ^ 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          if (rank == 0) ptx::mbar_arrive_expect_tx(ptx::smem_u32(full_bar + s), C::TX_PAIR);
          const uint32_t fb = lead_full0 + uint32_t(s) * 8u;
          const uint32_t st = ptx::smem_u32(smem + s * C::STAGE);
          ptx::tma_load_2d_pair(st + C::OFF_W, &m.w, kt * 128, nb * 256 + int(rank) * 128, fb);
          if (RES) ptx::tma_load_2d_pair(st + C::OFF_R, &m.r, kt * 128, rb * 128, fb);
          ptx::tma_load_2d_pair(st + C::OFF_B, &m.b, kt * (PAIR ? 64 : 128), rb * 128, fb);
          // scales and metadata: byte views [bytes / 256][256]
          if (RES)
            ptx::tma_load_2d_pair(st + C::OFF_SFR, &m.rs, 0,
                                  (rb_sf * (p.K / C::GD / 4) + kt * C::DCH) * 2, fb);
          if (PAIR) {
            ptx::tma_load_2d_pair(st + C::OFF_SFB, &m.bs, 0, (rb_sf * (p.K / 128) + kt * 2) * 2, fb);
            ptx::tma_load_2d_pair(st + C::OFF_E, &m.bm, 0,
                                  (kt * p.Mp * 16 + rb_sf * 2048) / 256, fb);
            // both 128-row halves of the weight tile's sparse-view scales in one box
            ptx::tma_load_4d_pair(st + C::OFF_SWS, &m.wss, 0, 0, kt, nb * 2, fb);
          } else {
            ptx::tma_load_2d_pair(st + C::OFF_SFB, &m.bs, 0,
                                  (rb_sf * (p.K / C::GD / 4) + kt * C::DCH) * 2, fb);
          }
          if (C::DENSE_W)  // both halves of the dense-view weight scales in one box
            ptx::tma_load_4d_pair(st + C::OFF_SWD, &m.wsd, 0, 0, kt, nb * 2, fb);
          if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) atomicExch(p.status, unsigned(SHARQ_ERR_TIMEOUT));
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (rank == 0 && ptx::elect_one()) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int tcount = 0;
      const uint32_t idesc_d = C::IDESC_BASE | C::SCALE_FMT;
      const uint32_t idesc_s = C::IDESC_BASE | C::SCALE_FMT | (1u << 2);
      for (int t = cluster; t < pair_tiles && ok; t += n_clusters, ++tcount) {
        if (tcount > 0) {
          if (!ptx::mbar_wait(ptx::smem_u32(tempty_bar), uint32_t(tcount - 1) & 1u, abort_flag,
                              limit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
        }
        for (int kt = 0; kt < KT; ++kt) {
          if (!ptx::mbar_wait(ptx::smem_u32(full_bar + s), ph, abort_flag, limit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const StageDesc sd(ptx::smem_u32(smem + s * C::STAGE));
          const uint32_t tb = tbase + uint32_t(kt & 1) * C::SF_SPAN;
          // ---- scales and metadata of this K step into both CTAs' tensor memory
          if (PAIR) {
            ptx::tmem_cp_128x128b_pair(tb + C::COL_E, sd.at<128, 0>(C::OFF_E));
            for (int j = 0; j < 2; ++j) {
              ptx::tmem_cp_32x128b_x4_pair(tb + C::COL_SFB + 4 * j,
                                           sd.at<128, 0>(C::OFF_SFB + 512 * j));
              for (int h = 0; h < 2; ++h)
                ptx::tmem_cp_32x128b_x4_pair(
                    tb + C::COL_SWS + j * (C::BN / 32) + 4 * h,
                    sd.at<128, 0>(C::OFF_SWS + (h * 2 + j) * 512));
            }
          } else {
            for (int c = 0; c < C::DCH; ++c)
              ptx::tmem_cp_32x128b_x4_pair(tb + C::COL_SFB + 4 * c,
                                           sd.at<128, 0>(C::OFF_SFB + 512 * c));
          }
          if (RES)
            for (int c = 0; c < C::DCH; ++c)
              ptx::tmem_cp_32x128b_x4_pair(tb + C::COL_SFR + 4 * c,
                                           sd.at<128, 0>(C::OFF_SFR + 512 * c));
          if (C::DENSE_W)
            for (int c = 0; c < C::DCH; ++c)
              for (int h = 0; h < 2; ++h)
                ptx::tmem_cp_32x128b_x4_pair(
                    tb + C::COL_SWD + c * (C::BN / 32) + 4 * h,
                    sd.at<128, 0>(C::OFF_SWD + (h * C::DCH + c) * 512));
          // ---- pair MMAs: backbone then residual, one accumulator
          uint32_t acc = kt > 0 ? 1u : 0u;
          if (PAIR) {
            for (int j = 0; j < 2; ++j) {
              const uint64_t a = sd.at<512, 4>(C::OFF_B + 32 * j);
              const uint64_t b = sd.at<1024, 2>(C::OFF_W + 64 * j);
              ptx::mma_sp_nvf4_pair(tbase, a, b, tb + C::COL_E + 2 * j, idesc_s,
                                    tb + C::COL_SFB + 4 * j, tb + C::COL_SWS + j * (C::BN / 32), acc);
              acc = 1u;
            }
          } else {
            for (int i = 0; i < 4; ++i) {
              const uint64_t a = sd.at<1024, 2>(C::OFF_B + 32 * i);
              const uint64_t b = sd.at<1024, 2>(C::OFF_W + 32 * i);
              if (C::NV) {
                ptx::mma_nvf4_pair(tbase, a, b, idesc_d, tb + C::COL_SFB + 4 * i,
                                   tb + C::COL_SWD + i * (C::BN / 32), acc);
              } else {
                const uint32_t id = 2u * uint32_t(i & 1);
                ptx::mma_mxf4_pair(tbase, a, b, idesc_d | (id << 29) | (id << 4),
                                   (tb + C::COL_SFB + 4 * (i >> 1)) | (id << 30),
                                   (tb + C::COL_SWD + (i >> 1) * (C::BN / 32)) | (id << 30), acc);
              }
              acc = 1u;
            }
          }
          if (RES) {
            for (int i = 0; i < 4; ++i) {
              const uint64_t a = sd.at<1024, 2>(C::OFF_R + 32 * i);
              const uint64_t b = sd.at<1024, 2>(C::OFF_W + 32 * i);
              if (C::NV) {
                ptx::mma_nvf4_pair(tbase, a, b, idesc_d, tb + C::COL_SFR + 4 * i,
                                   tb + C::COL_SWD + i * (C::BN / 32), 1u);
              } else {
                const uint32_t id = 2u * uint32_t(i & 1);
                ptx::mma_mxf4_pair(tbase, a, b, idesc_d | (id << 29) | (id << 4),
                                   (tb + C::COL_SFR + 4 * (i >> 1)) | (id << 30),
                                   (tb + C::COL_SWD + (i >> 1) * (C::BN / 32)) | (id << 30), 1u);
              }
            }
          }
          ptx::mma_commit_pair(ptx::smem_u32(empty_bar + s), 0x3);
          if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        ptx::mma_commit_pair(ptx::smem_u32(tfull_bar), 0x3);
      }
      // drain: everything issued above has completed once this arrives
      ptx::mma_commit_pair(ptx::smem_u32(drain_bar), 0x1);
      if (!ptx::mbar_wait(ptx::smem_u32(drain_bar), 0, abort_flag, limit)) ok = false;
      if (!ok) atomicExch(p.status, unsigned(SHARQ_ERR_TIMEOUT));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    constexpr int HALF = C::BN / 2;
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const float alpha = __fmul_rn(p.act_ts[0], p.w_ts[0]);
    const uint32_t epi_stage = ptx::smem_u32(ctrl + 1024 + (warp - 2) * 2048);
    int tcount = 0;
    bool ok = true;
    for (int t = cluster; t < pair_tiles; t += n_clusters, ++tcount) {
      const int mb2 = p.n_fast ? t / p.tiles_n : t % tiles_m2;
      const int nb = p.n_fast ? t % p.tiles_n : t / tiles_m2;
      if (!ptx::mbar_wait(ptx::smem_u32(tfull_bar), uint32_t(tcount) & 1u, abort_flag, limit)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int row = (mb2 * 2 + int(rank)) * 128 + quarter * 32 + lane;
      const uint32_t taddr = tbase + (uint32_t(quarter * 32) << 16) + uint32_t(half * HALF);
      uint32_t v[HALF];
#pragma unroll
      for (int c = 0; c < HALF / 32; ++c) ptx::tmem_ld_32x32b_x32(taddr + c * 32, v + 32 * c);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(lead_tempty);
      if (OUT_F32)
        store_rows_f32<HALF>(static_cast<float*>(p.Y), p.M, p.N, v, alpha, row, nb * C::BN + half * HALF);
      else
        store_rows_bf16<HALF>(&m.y, epi_stage, v, alpha, (mb2 * 2 + int(rank)) * 128 + quarter * 32, nb * C::BN + half * HALF, lane);
    }
    if (!OUT_F32 && lane == 0) ptx::bulk_wait_all();  // stores complete before exit
    if (!ok && lane == 0) atomicExch(p.status, unsigned(SHARQ_ERR_TIMEOUT));
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // no CTA leaves while its partner may still signal or read it
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tbase, 512);
  }
}

template <int FMT, bool PAIR, bool RES, bool OUT_F32>
static cudaError_t launch_pair_t(const GemmPairMaps& m, const GemmParams& p, int num_sms,
                                 cudaStream_t st) {
  using C = PairCfg<FMT, PAIR, RES>;
  auto kern = sharq_gemm_pair_kernel<FMT, PAIR, RES, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int pair_tiles = ((p.M + 255) / 256) * p.tiles_n;
  int clusters = num_sms / 2;
  if (clusters > pair_tiles) clusters = pair_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(2 * clusters));
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, m, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT, bool PAIR, bool RES>
static cudaError_t launch_pair_o(const GemmPairMaps& m, const GemmParams& p, bool f32, int n,
                                 cudaStream_t st) {
  return f32 ? launch_pair_t<FMT, PAIR, RES, true>(m, p, n, st)
             : launch_pair_t<FMT, PAIR, RES, false>(m, p, n, st);
}

template <int FMT, bool PAIR>
static cudaError_t launch_pair_r(const GemmPairMaps& m, const GemmParams& p, bool res, bool f32,
                                 int n, cudaStream_t st) {
  return res ? launch_pair_o<FMT, PAIR, true>(m, p, f32, n, st)
             : launch_pair_o<FMT, PAIR, false>(m, p, f32, n, st);
}

template <int FMT>
static cudaError_t launch_pair_m(const GemmPairMaps& m, const GemmParams& p, int mask, bool res,
                                 bool f32, int n, cudaStream_t st) {
  return is_pair_mask(mask) ? launch_pair_r<FMT, true>(m, p, res, f32, n, st)
                                     : launch_pair_r<FMT, false>(m, p, res, f32, n, st);
}

cudaError_t launch_gemm_pair(const GemmPairMaps& maps, const GemmParams& p, int fmt, int mask,
                             bool residual, bool out_f32, int num_sms, cudaStream_t st) {
  return fmt == SHARQ_NVFP4
             ? launch_pair_m<SHARQ_NVFP4>(maps, p, mask, residual, out_f32, num_sms, st)
             : launch_pair_m<SHARQ_MXFP4>(maps, p, mask, residual, out_f32, num_sms, st);
}

}  // namespace sharq

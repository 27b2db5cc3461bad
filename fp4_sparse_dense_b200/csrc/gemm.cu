// SharQ sparse + dense FP4 GEMM on sm_100a tensor cores (tcgen05, TMEM, TMA).
//
// SharQ page (pith.science 2606.26587), "Core claim" and abstract: the backbone goes
// through a structured-sparse FP4 GEMM, the residual through a dense FP4 GEMM that makes
// up for what the mask dropped and for the backbone's rounding, and both read the same
// FP4 weight codes, each with its own view of the weight scales. Here both GEMMs are one
// kernel: for every 256-wide K step the same weight tile in shared memory feeds two
// structured-sparse block-scaled MMAs (backbone, 128 logical K each) and four dense
// block-scaled MMAs (residual, 64 K each), all accumulating into one FP32 accumulator in
// tensor memory, which one epilogue scales by alpha = s_g * s_gw and writes once.
//
// CTA organisation (persistent, one CTA per SM, 10 warps):
//   warp 0      TMA producer: FP4 tiles by tensor-map loads, scales and metadata by
//               1-D bulk copies, all completing on the stage's "full" mbarrier;
//   warp 1      tensor-memory owner and single-thread MMA issuer: copies the stage's
//               scales / metadata into tensor memory (tcgen05.cp) and issues the MMAs;
//               tcgen05.commit releases the stage and, after the last K step, the
//               accumulator;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator into registers, release of the
//               accumulator, then scale, convert and store (overlapping the next tile).
// Tensor memory: columns [0, BN) accumulator; from column 256 two buffers of the scale
// factors and sparse metadata, used by alternate K steps, so that the copies of step k+1
// never write columns the MMAs of step k may still read.
// TWO (the variant whose residual has its own tensor scale s_r, BN = 128): the residual's
// MMAs accumulate in columns [128, 256) and the epilogue forms
// s_gw * (s_g * acc_backbone + s_r * acc_residual).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sharq_internal.h"
#include "epilogue.cuh"
#include "sm100_ptx.cuh"

namespace sharq {

constexpr int kMaxSmem = 232448;  // 227 KB opt-in dynamic shared memory per CTA
constexpr int kEpiThreads = 256;  // 8 epilogue warps
constexpr int kThreads = 64 + kEpiThreads;

template <int FMT, bool PAIR, bool RES, int BN>
struct GemmCfg {
  static constexpr bool NV = FMT == SHARQ_NVFP4;
  static constexpr int GD = NV ? 16 : 32;        // dense-view scale granularity (A and W)
  static constexpr int DCH = 256 / GD / 4;       // 512-byte scale chunks per K step (dense)
  static constexpr bool DENSE_W = RES || !PAIR;  // any dense MMA issued
  // bytes per stage
  static constexpr int W_BYTES = BN * 128;
  static constexpr int R_BYTES = RES ? 128 * 128 : 0;
  static constexpr int B_BYTES = PAIR ? 128 * 64 : 128 * 128;
  static constexpr int SFR_BYTES = RES ? DCH * 512 : 0;
  static constexpr int SFB_BYTES = PAIR ? 2 * 512 : DCH * 512;
  static constexpr int SWD_BYTES = DENSE_W ? (BN / 128) * DCH * 512 : 0;
  static constexpr int SWS_BYTES = PAIR ? (BN / 128) * 2 * 512 : 0;
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
  static constexpr int TX = STAGE_RAW;  // every byte of the stage arrives by copy
  static constexpr int TX_W = W_BYTES + SWD_BYTES + SWS_BYTES;  // the weight's part of it
  static constexpr int TX_A = TX - TX_W;                         // the activations' part
  static constexpr int EPI_BYTES = 8 * 2048;  // one 32 x 32 bf16 staging box per epilogue warp
  static constexpr int STAGES_FIT = (kMaxSmem - 2048 - EPI_BYTES) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  // stages, 1 KB of barriers, the epilogue staging, 1 KB alignment slack
  static constexpr int SMEM = STAGES * STAGE + 1024 + EPI_BYTES + 1024;
  // tensor-memory columns
  static constexpr int COL_SFR = 256;
  static constexpr int COL_SFB = COL_SFR + (RES ? DCH * 4 : 0);
  static constexpr int COL_SWD = COL_SFB + (PAIR ? 8 : DCH * 4);
  static constexpr int COL_SWS = COL_SWD + (DENSE_W ? DCH * (BN / 32) : 0);
  static constexpr int COL_E = COL_SWS + (PAIR ? 2 * (BN / 32) : 0);
  static constexpr int COL_END = COL_E + (PAIR ? 4 : 0);
  // scales / metadata are double-buffered: K step kt uses columns + (kt & 1) * SF_SPAN
  static constexpr int SF_SPAN = (COL_END - COL_SFR + 3) / 4 * 4;
  static_assert(COL_SFR + 2 * SF_SPAN <= 512, "tensor memory overflow");
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  // instruction descriptors (block-scaled kinds): E2M1 A and B, M = 128, N = BN
  static constexpr uint32_t IDESC_BASE =
      (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static constexpr uint32_t SCALE_FMT = NV ? 0u : (1u << 23);  // E4M3 or E8M0 scales
};

template <int FMT, bool PAIR, bool RES, int BN, bool OUT_F32, bool TWO = false>
__global__ void __launch_bounds__(kThreads, 1)
    sharq_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_r,
                      const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using C = GemmCfg<FMT, PAIR, RES, BN>;
  static_assert(!TWO || (RES && BN == 128), "second accumulator: residual on, BN = 128");
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
  const int KT = p.K / 256;
  const int tiles_mn = p.tiles_m * p.tiles_n;
  const int tiles = tiles_mn * p.splits;  // split-K: `splits` K ranges per output tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(ptx::smem_u32(full_bar + s), 1);
      ptx::mbar_init(ptx::smem_u32(empty_bar + s), 1);
    }
    ptx::mbar_init(ptx::smem_u32(tfull_bar), 1);
    ptx::mbar_init(ptx::smem_u32(tempty_bar), kEpiThreads);
    ptx::mbar_init(ptx::smem_u32(drain_bar), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tensormap(&tm_w);
    ptx::prefetch_tensormap(&tm_b);
    if (RES) ptx::prefetch_tensormap(&tm_r);
  }
  // the weight's part of K step kt of N block nb into stage buffer st (codes and scales)
  auto load_w = [&](uint8_t* st, int kt, int nb, uint32_t fb) {
    ptx::tma_load_2d(ptx::smem_u32(st + C::OFF_W), &tm_w, kt * 128, nb * BN, fb);
    if (PAIR) {
      for (int rb = 0; rb < BN / 128; ++rb) {
        const uint8_t* w =
            p.wss + (size_t(nb * (BN / 128) + rb) * (p.K / 32 / 4) + size_t(kt) * 2) * 512;
        ptx::bulk_load(ptx::smem_u32(st + C::OFF_SWS + rb * 1024), w, 1024, fb);
      }
    }
    if (C::DENSE_W) {
      for (int rb = 0; rb < BN / 128; ++rb) {
        const uint8_t* w = p.wsd + (size_t(nb * (BN / 128) + rb) * (p.K / C::GD / 4) +
                                    size_t(kt) * C::DCH) * 512;
        ptx::bulk_load(ptx::smem_u32(st + C::OFF_SWD + rb * C::DCH * 512), w, C::DCH * 512, fb);
      }
    }
  };
  // Decode-sized M: the weight part of the first tile's first stages is loaded now, while the
  // kernel launched just before (the preparation) may still run. The weight is not among its
  // outputs: it was written before that kernel started (sharq_linear's contract). The
  // stages' barriers only get the bytes to expect here; their arrival, with the
  // activations' bytes, comes after the wait, so no stage completes early.
  int n_pre = 0;
  if (p.prefetch_w && warp == 0) {
    if (lane == 0 && int(blockIdx.x) < tiles) {
      const int t = blockIdx.x;
      const int tmn = t % tiles_mn, ks = t / tiles_mn;
      const int nb = tmn / p.tiles_m;
      const int kt0 = ks * KT / p.splits, kt1 = (ks + 1) * KT / p.splits;
      n_pre = kt1 - kt0 < C::STAGES ? kt1 - kt0 : C::STAGES;
      for (int i = 0; i < n_pre; ++i) {
        const uint32_t fb = ptx::smem_u32(full_bar + i);
        ptx::mbar_expect_tx(fb, C::TX_W);
        load_w(smem + i * C::STAGE, kt0 + i, nb, fb);
      }
    }
    n_pre = __shfl_sync(0xFFFFFFFFu, n_pre, 0);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t limit = p.timeout_ns;
  // launched as a programmatic dependent: the set-up above overlapped the previous kernel;
  // nothing it wrote (the activation operands) is read before this point
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (ptx::elect_one()) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool first = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, first = false) {
        const int tmn = t % tiles_mn, ks = t / tiles_mn;
        const int mb = tmn % p.tiles_m, nb = tmn / p.tiles_m;
        const int kt0 = ks * KT / p.splits, kt1 = (ks + 1) * KT / p.splits;
        for (int kt = kt0; kt < kt1; ++kt) {
          if (!ptx::mbar_wait(ptx::smem_u32(empty_bar + s), ph ^ 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          const uint32_t fb = ptx::smem_u32(full_bar + s);
          uint8_t* st = smem + s * C::STAGE;
          if (first && kt - kt0 < n_pre) {  // weight part already on its way (see above)
            ptx::mbar_arrive_expect_tx(fb, C::TX_A);
          } else {
            ptx::mbar_arrive_expect_tx(fb, C::TX);
            load_w(st, kt, nb, fb);
          }
          if (RES) ptx::tma_load_2d(ptx::smem_u32(st + C::OFF_R), &tm_r, kt * 128, mb * 128, fb);
          ptx::tma_load_2d(ptx::smem_u32(st + C::OFF_B), &tm_b, kt * (PAIR ? 64 : 128), mb * 128,
                           fb);
          if (RES) {
            const uint8_t* src = p.rs + (size_t(mb) * (p.K / C::GD / 4) + size_t(kt) * C::DCH) * 512;
            ptx::bulk_load(ptx::smem_u32(st + C::OFF_SFR), src, C::SFR_BYTES, fb);
          }
          if (PAIR) {
            const uint8_t* src = p.bs + (size_t(mb) * (p.K / 32 / 4) + size_t(kt) * 2) * 512;
            ptx::bulk_load(ptx::smem_u32(st + C::OFF_SFB), src, C::SFB_BYTES, fb);
            const uint8_t* e = p.bm + size_t(kt) * p.Mp * 16 + size_t(mb) * 2048;
            ptx::bulk_load(ptx::smem_u32(st + C::OFF_E), e, 2048, fb);
          } else {
            const uint8_t* src = p.bs + (size_t(mb) * (p.K / C::GD / 4) + size_t(kt) * C::DCH) * 512;
            ptx::bulk_load(ptx::smem_u32(st + C::OFF_SFB), src, C::SFB_BYTES, fb);
          }
          if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) atomicExch(p.status, unsigned(SHARQ_ERR_TIMEOUT));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (ptx::elect_one()) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int tcount = 0;
      const uint32_t idesc_d = C::IDESC_BASE | C::SCALE_FMT;
      const uint32_t idesc_s = C::IDESC_BASE | C::SCALE_FMT | (1u << 2);
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tcount) {
        if (tcount > 0) {
          if (!ptx::mbar_wait(ptx::smem_u32(tempty_bar), uint32_t(tcount - 1) & 1u, abort_flag,
                              limit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
        }
        const int ks = t / tiles_mn;
        const int kt0 = ks * KT / p.splits, kt1 = (ks + 1) * KT / p.splits;
        for (int kt = kt0; kt < kt1; ++kt) {
          if (!ptx::mbar_wait(ptx::smem_u32(full_bar + s), ph, abort_flag, limit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t st = ptx::smem_u32(smem + s * C::STAGE);
          // this K step's half of the double-buffered scale / metadata columns
          const uint32_t tb = tbase + uint32_t(kt & 1) * C::SF_SPAN;
          // ---- scale factors and metadata of this K step into tensor memory
          if (PAIR) {
            ptx::tmem_cp_128x128b(tb + C::COL_E, ptx::smem_desc(st + C::OFF_E, 16, 128, 0));
            for (int j = 0; j < 2; ++j) {
              ptx::tmem_cp_32x128b_x4(tb + C::COL_SFB + 4 * j,
                                      ptx::smem_desc(st + C::OFF_SFB + 512 * j, 16, 128, 0));
              for (int rb = 0; rb < BN / 128; ++rb)
                ptx::tmem_cp_32x128b_x4(
                    tb + C::COL_SWS + j * (BN / 32) + 4 * rb,
                    ptx::smem_desc(st + C::OFF_SWS + (rb * 2 + j) * 512, 16, 128, 0));
            }
          } else {
            for (int c = 0; c < C::DCH; ++c)
              ptx::tmem_cp_32x128b_x4(tb + C::COL_SFB + 4 * c,
                                      ptx::smem_desc(st + C::OFF_SFB + 512 * c, 16, 128, 0));
          }
          if (RES) {
            for (int c = 0; c < C::DCH; ++c)
              ptx::tmem_cp_32x128b_x4(tb + C::COL_SFR + 4 * c,
                                      ptx::smem_desc(st + C::OFF_SFR + 512 * c, 16, 128, 0));
          }
          if (C::DENSE_W) {
            for (int c = 0; c < C::DCH; ++c)
              for (int rb = 0; rb < BN / 128; ++rb)
                ptx::tmem_cp_32x128b_x4(
                    tb + C::COL_SWD + c * (BN / 32) + 4 * rb,
                    ptx::smem_desc(st + C::OFF_SWD + (rb * C::DCH + c) * 512, 16, 128, 0));
          }
          // ---- MMAs: backbone then residual, one accumulator
          uint32_t acc = kt > kt0 ? 1u : 0u;
          if (PAIR) {
            for (int j = 0; j < 2; ++j) {
              const uint64_t a = ptx::smem_desc(st + C::OFF_B + 32 * j, 16, 512, 4);
              const uint64_t b = ptx::smem_desc(st + C::OFF_W + 64 * j, 16, 1024, 2);
              ptx::mma_sp_nvf4(tbase, a, b, tb + C::COL_E + 2 * j, idesc_s,
                               tb + C::COL_SFB + 4 * j, tb + C::COL_SWS + j * (BN / 32), acc);
              acc = 1u;
            }
          } else {
            for (int i = 0; i < 4; ++i) {
              const uint64_t a = ptx::smem_desc(st + C::OFF_B + 32 * i, 16, 1024, 2);
              const uint64_t b = ptx::smem_desc(st + C::OFF_W + 32 * i, 16, 1024, 2);
              if (C::NV) {
                ptx::mma_nvf4(tbase, a, b, idesc_d, tb + C::COL_SFB + 4 * i,
                              tb + C::COL_SWD + i * (BN / 32), acc);
              } else {
                const uint32_t id = 2u * uint32_t(i & 1);
                ptx::mma_mxf4(tbase, a, b, idesc_d | (id << 29) | (id << 4),
                              (tb + C::COL_SFB + 4 * (i >> 1)) | (id << 30),
                              (tb + C::COL_SWD + (i >> 1) * (BN / 32)) | (id << 30), acc);
              }
              acc = 1u;
            }
          }
          if (RES) {
            // one accumulator, or (TWO) the residual's own, starting at the range's first step
            const uint32_t tacc = TWO ? tbase + uint32_t(BN) : tbase;
            uint32_t acc_r = TWO ? (kt > kt0 ? 1u : 0u) : 1u;
            for (int i = 0; i < 4; ++i) {
              const uint64_t a = ptx::smem_desc(st + C::OFF_R + 32 * i, 16, 1024, 2);
              const uint64_t b = ptx::smem_desc(st + C::OFF_W + 32 * i, 16, 1024, 2);
              if (C::NV) {
                ptx::mma_nvf4(tacc, a, b, idesc_d, tb + C::COL_SFR + 4 * i,
                              tb + C::COL_SWD + i * (BN / 32), acc_r);
              } else {
                const uint32_t id = 2u * uint32_t(i & 1);
                ptx::mma_mxf4(tacc, a, b, idesc_d | (id << 29) | (id << 4),
                              (tb + C::COL_SFR + 4 * (i >> 1)) | (id << 30),
                              (tb + C::COL_SWD + (i >> 1) * (BN / 32)) | (id << 30), acc_r);
              }
              acc_r = 1u;
            }
          }
          ptx::mma_commit(ptx::smem_u32(empty_bar + s));
          if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_u32(tfull_bar));
      }
      // drain: every tcgen05 operation issued above has finished once this arrives
      ptx::mma_commit(ptx::smem_u32(drain_bar));
      if (!ptx::mbar_wait(ptx::smem_u32(drain_bar), 0, abort_flag, limit)) ok = false;
      if (!ok) atomicExch(p.status, unsigned(SHARQ_ERR_TIMEOUT));
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Eight warps: warp w reads tensor-memory lane quarter w % 4 (rows) and column half
    // (w - 2) / 4. Each thread pulls its row's BN/2 accumulator columns into registers,
    // releases the accumulator (so the next tile's MMAs start at once), then scales,
    // converts and stores while the tensor cores run ahead.
    constexpr int HALF = BN / 2;
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const float alpha = __fmul_rn(p.act_ts[0], p.w_ts[0]);
    const uint32_t epi_stage = ptx::smem_u32(ctrl + 1024 + (warp - 2) * 2048);
    int tcount = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tcount) {
      const int tmn = t % tiles_mn, ks = t / tiles_mn;
      const int mb = tmn % p.tiles_m, nb = tmn / p.tiles_m;
      if (!ptx::mbar_wait(ptx::smem_u32(tfull_bar), uint32_t(tcount) & 1u, abort_flag, limit)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int row = mb * 128 + quarter * 32 + lane;
      const uint32_t taddr = tbase + (uint32_t(quarter * 32) << 16) + uint32_t(half * HALF);
      uint32_t v[HALF];
#pragma unroll
      for (int c = 0; c < HALF / 32; ++c) ptx::tmem_ld_32x32b_x32(taddr + c * 32, v + 32 * c);
      if constexpr (TWO) {
        uint32_t vr[HALF];
#pragma unroll
        for (int c = 0; c < HALF / 32; ++c)
          ptx::tmem_ld_32x32b_x32(taddr + uint32_t(BN) + c * 32, vr + 32 * c);
        ptx::tmem_ld_wait();
        // s_gw * (s_g * b + s_r * r), then stored with a unit scale
        const float ab = alpha, ar = __fmul_rn(p.act_ts[6], p.w_ts[0]);
#pragma unroll
        for (int i = 0; i < HALF; ++i)
          v[i] = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(v[i]), ab),
                                           __fmul_rn(__uint_as_float(vr[i]), ar)));
      }
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(ptx::smem_u32(tempty_bar));
      const float out_scale = TWO ? 1.0f : alpha;
      if (p.splits > 1)  // unscaled FP32 partial of this K range, reduced by a second kernel
        store_rows_f32<HALF>(p.ws + size_t(ks) * p.M * p.N, p.M, p.N, v, 1.0f, row,
                             nb * BN + half * HALF);
      else if (OUT_F32)
        store_rows_f32<HALF>(static_cast<float*>(p.Y), p.M, p.N, v, out_scale, row, nb * BN + half * HALF);
      else
        store_rows_bf16<HALF>(&tm_y, epi_stage, v, out_scale, mb * 128 + quarter * 32, nb * BN + half * HALF, lane);
    }
    if (!OUT_F32 && p.splits == 1 && lane == 0) ptx::bulk_wait_all();  // stores done before exit
    if (!ok && lane == 0) atomicExch(p.status, unsigned(SHARQ_ERR_TIMEOUT));
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, 512);
  }
}

template <int FMT, bool PAIR, bool RES, int BN, bool OUT_F32, bool TWO = false>
static cudaError_t launch_t(const GemmMaps& m, const GemmParams& p, int num_sms, cudaStream_t st) {
  using C = GemmCfg<FMT, PAIR, RES, BN>;
  auto kern = sharq_gemm_kernel<FMT, PAIR, RES, BN, OUT_F32, TWO>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n * p.splits;
  const int grid = tiles < num_sms ? tiles : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, m.w, m.b, m.r, m.y, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Split-K reduction: Y = alpha * sum over the K ranges of the FP32 partials, in a fixed
// order (deterministic). One thread per 2 consecutive outputs, so that decode-sized outputs
// spread over several SMs; the partials of up to 16 splits are loaded before any is added
// (one L2 round trip for the usual split counts), then added in split order.
constexpr int kReduceOut = 2;    // outputs per thread
constexpr int kReduceBatch = 16; // splits loaded together
template <bool OUT_F32>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ ws,
                                                            int splits, int M, int N,
                                                            const float* act_ts, const float* w_ts,
                                                            void* Y) {
  ptx::griddep_wait();  // the partials of the GEMM launched just before
  const size_t total = size_t(M) * N;
  const size_t i = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) * kReduceOut;
  if (i >= total) return;
  const float alpha = __fmul_rn(act_ts[0], w_ts[0]);
  float2 acc = make_float2(0.f, 0.f);
  for (int base = 0; base < splits; base += kReduceBatch) {
    float2 v[kReduceBatch];
#pragma unroll
    for (int j = 0; j < kReduceBatch; ++j)
      if (base + j < splits)
        v[j] = __ldcg(reinterpret_cast<const float2*>(ws + size_t(base + j) * total + i));
#pragma unroll
    for (int j = 0; j < kReduceBatch; ++j) {
      if (base + j >= splits) break;
      if (base + j == 0) {
        acc = v[j];
      } else {
        acc.x = __fadd_rn(acc.x, v[j].x);
        acc.y = __fadd_rn(acc.y, v[j].y);
      }
    }
  }
  if (OUT_F32) {
    *reinterpret_cast<float2*>(static_cast<float*>(Y) + i) =
        make_float2(__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha));
  } else {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha));
    *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(Y) + i) = b2;
  }
}

template <int FMT, bool PAIR, bool RES, int BN>
static cudaError_t launch_o(const GemmMaps& m, const GemmParams& p, bool f32, int n, cudaStream_t st) {
  return f32 ? launch_t<FMT, PAIR, RES, BN, true>(m, p, n, st)
             : launch_t<FMT, PAIR, RES, BN, false>(m, p, n, st);
}

template <int FMT, bool PAIR, bool RES>
static cudaError_t launch_n(const GemmMaps& m, const GemmParams& p, bool f32, int n, cudaStream_t st) {
  return (p.N % 256 == 0) ? launch_o<FMT, PAIR, RES, 256>(m, p, f32, n, st)
                          : launch_o<FMT, PAIR, RES, 128>(m, p, f32, n, st);
}

template <int FMT, bool PAIR>
static cudaError_t launch_r(const GemmMaps& m, const GemmParams& p, bool res, bool f32, int n,
                            cudaStream_t st) {
  return res ? launch_n<FMT, PAIR, true>(m, p, f32, n, st)
             : launch_n<FMT, PAIR, false>(m, p, f32, n, st);
}

template <int FMT>
static cudaError_t launch_m(const GemmMaps& m, const GemmParams& p, int mask, bool res, bool f32,
                            int n, cudaStream_t st) {
  return is_pair_mask(mask) ? launch_r<FMT, true>(m, p, res, f32, n, st)
                                     : launch_r<FMT, false>(m, p, res, f32, n, st);
}

// The variant whose residual has its own tensor scale: NVFP4, pair mask, BN = 128, two
// accumulators, no split-K.
cudaError_t launch_gemm_two(const GemmMaps& maps, const GemmParams& p, bool out_f32, int num_sms,
                            cudaStream_t st) {
  if (p.splits != 1 || p.tiles_n * 128 != p.N) return cudaErrorInvalidValue;
  return out_f32 ? launch_t<SHARQ_NVFP4, true, true, 128, true, true>(maps, p, num_sms, st)
                 : launch_t<SHARQ_NVFP4, true, true, 128, false, true>(maps, p, num_sms, st);
}

cudaError_t launch_gemm(const GemmMaps& maps, const GemmParams& p, int fmt, int mask,
                        bool residual, bool out_f32, int num_sms, cudaStream_t st) {
  cudaError_t e =
      fmt == SHARQ_NVFP4 ? launch_m<SHARQ_NVFP4>(maps, p, mask, residual, out_f32, num_sms, st)
                         : launch_m<SHARQ_MXFP4>(maps, p, mask, residual, out_f32, num_sms, st);
  if (e != cudaSuccess || p.splits <= 1) return e;
  const size_t total = size_t(p.M) * p.N;
  const unsigned blocks = unsigned((total / kReduceOut + 255) / 256);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = out_f32 ? cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<true>, (const float*)p.ws, p.splits,
                                   p.M, p.N, p.act_ts, p.w_ts, p.Y)
              : cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<false>, (const float*)p.ws, p.splits,
                                   p.M, p.N, p.act_ts, p.w_ts, p.Y);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sharq

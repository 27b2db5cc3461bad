/*
 * sharq.h - C ABI of the SharQ sparse-dense FP4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The operation is the one stated on the SharQ page ("SharQ: Bridging Activation
 * Sparsity and FP4 Quantization for LLM Inference", pith.science 2606.26587, "Core
 * claim" and arXiv abstract): for each activation tensor an input-adaptive N:M mask
 * extracts an outlier-dominated sparse backbone, the backbone is quantised to FP4, a
 * dense residual is defined against the quantised backbone and quantised to FP4 with its
 * own scales, and Y = sparse-FP4-GEMM(backbone, W) + dense-FP4-GEMM(residual, W), the two
 * GEMMs sharing one FP4 weight payload with path-specific scale views.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor arguments are DEVICE pointers into memory the caller owns. The library
 *   never allocates or frees device memory and keeps no pointer after a call returns,
 *   except a small host-side cache of TMA descriptors keyed by (pointer, shape).
 * - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *   stream) and the call returns without synchronising, except the two status reads.
 * - Every device pointer must be 16-byte aligned (TMA / 128-bit access); a misaligned
 *   pointer returns SHARQ_ERR_MISALIGNED before anything is enqueued.
 * - Shapes: K % 256 == 0, N % 128 == 0, M >= 1 (no upper bound other than int32 sizes).
 * - Errors are returned by value; no call aborts the process. A CUDA launch error is
 *   reported as SHARQ_ERR_CUDA. A kernel that gives up on a bounded wait records
 *   SHARQ_ERR_TIMEOUT in the status word of its stream, read back by
 *   sharq_read_device_status(stream) (or, device-wide, sharq_device_status()).
 * - The library needs an sm_100 device (B200); on anything else the compute calls return
 *   SHARQ_ERR_ARCH. The size queries and sharq_status_string need no GPU.
 */
#ifndef SHARQ_H
#define SHARQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SHARQ_API __attribute__((visibility("default")))
#else
#define SHARQ_API
#endif

typedef enum {
  SHARQ_OK = 0,
  SHARQ_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, mismatched configs */
  SHARQ_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
  SHARQ_ERR_MISALIGNED = 3,   /* a device pointer is not 16-byte aligned */
  SHARQ_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  SHARQ_ERR_TIMEOUT = 5,      /* a kernel hit its bounded-wait limit and exited */
  SHARQ_ERR_ARCH = 6          /* the current device is not sm_100 */
} sharq_status;

/* FP4 encodings. NVFP4: E2M1 codes, E4M3 block scales, FP32 tensor scale.
 * MXFP4 (OCP MX): E2M1 codes, E8M0 block scales, no tensor scale. */
typedef enum { SHARQ_NVFP4 = 0, SHARQ_MXFP4 = 1 } sharq_format;

/* Backbone masks along K. PAIR_4_8: in every 8 consecutive K elements keep 2 of the 4
 * adjacent pairs (the structured sparsity of the sm_100a sparse FP4 MMA); pairs ranked by
 * (max |x|, then min |x|), ties to the lower pair. ELEM_2_4: in every 4 keep the 2 largest
 * |x|, ties to the lower index; the backbone is then stored zero-filled and runs through
 * the dense MMA (sm_100a has no element-wise 2:4 pattern for block-scaled FP4). */
typedef enum {
  SHARQ_MASK_PAIR_4_8 = 0,
  SHARQ_MASK_ELEM_2_4 = 1,
  /* Ablation modes (the page's referee asks for them; not part of the method):
   * PAIR_4_8_GIVEN: the pair-wise 4:8 mask is not chosen per row but read from act->bm,
   * which the caller fills in the PAIR metadata layout before sharq_prepare (a static
   * mask: one channel set for the whole tensor, e.g. from calibration statistics); the
   * rest is PAIR_4_8. NONE: no mask, every element is on the "backbone", i.e. plain FP4
   * of x in the residual's block size through the dense MMA (with residual on, a second
   * dense FP4 term r = x - deq(Q(x))). */
  SHARQ_MASK_PAIR_4_8_GIVEN = 2,
  SHARQ_MASK_NONE = 3
} sharq_mask;

typedef enum { SHARQ_F16 = 0, SHARQ_BF16 = 1, SHARQ_F32 = 2 } sharq_dtype;

typedef struct {
  int32_t fmt;      /* sharq_format */
  int32_t mask;     /* sharq_mask */
  int32_t residual; /* 1: backbone + residual (the method); 0: backbone only;
                       2: ablation, residual against the unquantised backbone
                       (r = x - backbone: 0 where the mask keeps, x elsewhere);
                       3: the residual with its own tensor scale s_r = amax|r| / 2688
                       instead of sharing s_g (NVFP4 with a pair mask, else
                       SHARQ_ERR_UNSUPPORTED): two accumulators, Y = s_gw * (s_g *
                       acc_backbone + s_r * acc_residual) */
} sharq_config;

/* Block sizes along K (logical positions per scale), fixed by the MMA consuming them:
 *   residual:  16 (NVFP4) | 32 (MXFP4)
 *   backbone:  32 for PAIR_4_8 (16 kept values); the residual's size for ELEM_2_4
 *   weight:    32 for PAIR_4_8(_GIVEN) or MXFP4; 16 for NVFP4 + ELEM_2_4 / NONE
 *   (PAIR_4_8_GIVEN has the sizes and layouts of PAIR_4_8; NONE those of ELEM_2_4,
 *   without metadata: act->bm is unused and may be NULL)
 *
 * Byte layouts (all row-major in the sense given):
 *   FP4 codes:  two per byte, even K index in the low nibble, rows K-major.
 *   Scales:     one byte per (row, block); rows grouped by 128 and block columns by 4;
 *               each 128x4 tile is a 512-byte chunk where (r, c) sits at
 *               (r%32)*16 + ((r/32)%4)*4 + c%4; chunks run along the columns first,
 *               then along the 128-row groups. Rows padded to 128, columns to 4.
 *   PAIR metadata: one nibble per 8 logical K, i0 | i1<<2 (kept pair indices i0 < i1).
 *               Per 256 logical K, rows padded to 128 are stored one after another,
 *               16 bytes each (lower group in the low nibble); the 256-K slices follow
 *               each other. Padding rows hold 0x44 (pairs 0 and 1).
 *   ELEM metadata: one nibble per 4 K (element indices), row-major, K/8 bytes per row.
 */

/* Quantised weight. Filled by sharq_quantize_weight; the caller allocates the buffers
 * with the sizes from sharq_weight_sizes and keeps them for every later sharq_linear. */
typedef struct {
  void* codes;         /* [N][K/2] bytes: W^T K-major, E2M1 */
  void* scales_dense;  /* tiled scales, N x K/16 (NVFP4) or N x K/32 (MXFP4): the dense
                          MMA's view */
  void* scales_sparse; /* tiled scales, N x K/32: the sparse MMA's view (PAIR_4_8 only,
                          else unused and may be NULL) */
  float* tensor_scale; /* 2 floats: [0] s_gw = amax|W| / 2688 (NVFP4) or 1.0 (MXFP4);
                          [1] amax|W| (NVFP4; written by the first pass) */
  int32_t K, N;
  sharq_config cfg;
} sharq_weight;

/* Prepared activations. Filled by sharq_prepare from X[M x K]. */
typedef struct {
  void* bq;            /* backbone codes: [M][K/4] bytes (PAIR, compressed) or
                          [M][K/2] (ELEM, zero-filled) */
  void* bs;            /* backbone scales, tiled, M x K/backbone_block */
  void* bm;            /* metadata: PAIR layout (M_pad*K/16 bytes) or ELEM (M*K/8) */
  void* rq;            /* residual codes [M][K/2] (unused when residual == 0) */
  void* rs;            /* residual scales, tiled, M x K/residual_block */
  float* tensor_scale; /* 8 floats (32 bytes): [0] s_g = amax|X| / 2688 (NVFP4) or 1.0
                          (MXFP4); [1] amax|X| (NVFP4); both written by sharq_prepare.
                          [6] s_r = amax|r| / 2688 and [7] amax|r|, written when
                          residual == 3. [2..5] library state of the amax reductions: set
                          [2..7] to zero once when the buffer is allocated and never write
                          [2..5] afterwards (re-zero them if a call was interrupted by a
                          device error). */
  int32_t M, K;
  sharq_config cfg;
} sharq_act;

typedef struct { size_t bq, bs, bm, rq, rs; } sharq_act_bytes;
typedef struct { size_t codes, scales_dense, scales_sparse; } sharq_weight_bytes;

/* Byte sizes of the buffers of a sharq_act for X[M x K] under cfg. No GPU needed.
 * Errors: INVALID_ARG (bad shape/config or out == NULL). */
SHARQ_API sharq_status sharq_act_sizes(int32_t M, int32_t K, sharq_config cfg, sharq_act_bytes* out);

/* Byte sizes of the buffers of a sharq_weight for W[K x N] under cfg. No GPU needed. */
SHARQ_API sharq_status sharq_weight_sizes(int32_t K, int32_t N, sharq_config cfg, sharq_weight_bytes* out);

/* Offline weight quantisation (SharQ page, abstract: one FP4 weight payload serves both
 * GEMMs, each with its own view of the scales). W: device pointer to W[K x N] row-major
 * in `dtype` (F16 or BF16). Writes w->codes, w->scales_dense, w->scales_sparse (PAIR) and
 * w->tensor_scale, whose shapes/config are taken from *w. */
SHARQ_API sharq_status sharq_quantize_weight(const void* W, sharq_dtype dtype, const sharq_weight* w,
                                   void* stream);

/* Online activation preparation (SharQ page, "Core claim": adaptive N:M mask, backbone
 * quantisation, residual against the quantised backbone, residual quantisation, fused
 * into one operator). X: device pointer to X[M x K] row-major in `dtype` (F16 or BF16).
 * Computes the tensor scale (NVFP4) in a first pass over X, then writes every buffer of
 * *act, including padding rows of the tiled scale and metadata layouts. With the pair
 * mask the first pass also computes the mask and metadata, and the second reads them back;
 * the two kernels hand the tensor amax over through act->tensor_scale[2..3], so calls
 * that share one act->tensor_scale buffer must be ordered (one stream). With the pair
 * mask M * K must be below 2^31 (else SHARQ_ERR_UNSUPPORTED). X must be finite: an infinite
 * or NaN element gives unspecified codes and scales (the kernels have no data-dependent
 * control flow, so nothing faults or waits on it). */
SHARQ_API sharq_status sharq_prepare(const void* X, sharq_dtype dtype, const sharq_act* act, void* stream);

/* The preparation with the NVFP4 tensor amax supplied by the caller instead of reduced from
 * X in the call (a deployment option the SharQ page does not discuss: a static amax from
 * calibration, or one a producer kernel has already reduced). amax: DEVICE pointer to one
 * float (4-byte aligned), read by the kernel; s_g = amax / 2688 and every code, scale and
 * metadata byte are those sharq_prepare would write if max |X| were that value (values of X
 * above it saturate: E4M3 block scales clamp at 448, E2M1 codes at 6). With the amax known
 * before X is read, the preparation is a single kernel that also computes the mask.
 * NVFP4 with SHARQ_MASK_PAIR_4_8 and residual 0 or 1 only (else SHARQ_ERR_UNSUPPORTED);
 * act->tensor_scale[0..1] receive s_g and amax as with sharq_prepare. */
SHARQ_API sharq_status sharq_prepare_given_amax(const void* X, sharq_dtype dtype, const float* amax,
                                    const sharq_act* act, void* stream);

/* The same preparation, with results identical to sharq_prepare, launched to share the GPU
 * with a sharq_linear GEMM that runs at the same time on another stream (the overlap of
 * one batch's preparation with another batch's GEMM: the SharQ page's Fig. 4a latency
 * breakdown puts the preparation beside the two GEMMs). The persistent pair-mask kernels
 * run one CTA per SM, small enough in registers and shared memory to sit beside a GEMM
 * CTA, so neither waits for the other to leave the SMs. Alone on the GPU it is slower than
 * sharq_prepare. Arguments, buffers and errors as for sharq_prepare; the caller orders the
 * two streams (the GEMM that reads *act waits for this call, and a call that rewrites *act
 * waits for the GEMMs reading it). The element 2:4 mask runs its usual kernel. */
SHARQ_API sharq_status sharq_prepare_alongside(const void* X, sharq_dtype dtype, const sharq_act* act,
                                   void* stream);

/* Preparation with the layer's RMSNorm absorbed (SharQ page, abstract: the fused
 * preparation operator takes in layer normalisation; RMSNorm is that of the Llama/Qwen
 * models the page evaluates). The prepared input is y = round16((x * rstd) * gamma) per
 * element, rstd = 1 / sqrt(mean_k x^2 + eps) per row, and *act is filled exactly as
 * sharq_prepare(y) would fill it. Float32 throughout, one rounding per operation; the sum
 * of squares in a fixed order (chunk c of 8 elements to accumulator c mod 32, in increasing
 * k; then accumulators combined by xor 16, 8, 4, 2, 1), so results are reproducible.
 * X: device [M x K] row-major in `dtype` (F16 or BF16, 16-byte aligned); gamma: device [K]
 * in the same dtype; eps >= 0; rstd: device float[M], written. Pair mask only (element mask:
 * SHARQ_ERR_UNSUPPORTED); M * K < 2^31. Nothing is written to X. */
SHARQ_API sharq_status sharq_prepare_rmsnorm(const void* X, const void* gamma, float eps,
                                             sharq_dtype dtype, float* rstd,
                                             const sharq_act* act, void* stream);

/* Y[M x N] = alpha * (sparse-FP4-GEMM(backbone, W) + dense-FP4-GEMM(residual, W)) with
 * alpha = s_g * s_gw, accumulated in FP32 tensor memory and written once (SharQ page, "Core
 * claim": a sparse FP4 GEMM for the backbone and a dense FP4 GEMM for the compensation,
 * sharing one weight payload). With residual == 3 the two GEMMs accumulate separately and
 * Y = s_gw * (s_g * acc_backbone + s_r * acc_residual) (128-wide tiles, no split-K). Y: device pointer, row-major, y_dtype BF16 (the product) or
 * F32. act->cfg must equal w->cfg and act->K == w->K.
 * workspace / workspace_bytes: optional caller-owned device scratch (16-byte aligned) for
 * the split-K path used when the output has too few tiles to occupy the GPU (decode-sized
 * M); sharq_linear_workspace_size gives the bytes it wants. With a NULL or too small
 * workspace the call runs without splitting K (same result up to summation order, slower
 * for small M).
 * Ordering: the GEMM is launched as a programmatic dependent of the kernel launched just
 * before it on `stream`. It reads nothing of *act before that kernel has completed. For
 * M < 256 it may start loading w's codes and scales while that kernel still runs, when
 * this library's previous launch on `stream` was a preparation or a linear call. It does
 * not do this on a stream it has not seen before, nor after sharq_quantize_weight. So w
 * must be complete before the kernel launched just before this call starts. A caller's
 * own kernel that writes w must not come between a preparation and this call on `stream`.
 * A copy (cudaMemcpyAsync) or a write ordered through an event is fine. */
SHARQ_API sharq_status sharq_linear(const sharq_act* act, const sharq_weight* w, void* Y,
                                    sharq_dtype y_dtype, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Bytes of workspace sharq_linear uses for this shape on the current device (0 when it does
 * not split K). Needs the device's SM count: returns SHARQ_ERR_CUDA / SHARQ_ERR_ARCH
 * without a usable sm_100 device. */
SHARQ_API sharq_status sharq_linear_workspace_size(int32_t M, int32_t N, int32_t K,
                                                   sharq_config cfg, size_t* bytes);

/* sharq_linear for callers that cannot allocate device memory (the SharQ page has no
 * counterpart: this is a deployment aid, not part of the method). Some callers cannot pass
 * a workspace: code that runs inside a CUDA graph or an allocator-free runtime, or a host
 * whose memory manager forbids allocation on the hot path. For decode-sized M, the linear
 * layer splits K and sums FP32 partials in scratch memory; here that scratch is a fixed
 * device array compiled into the library, 16 MiB per GPU, held by every GPU that loads
 * the library until the process exits. The call itself allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine).
 * - Arguments and result are those of sharq_linear without the workspace; shapes that
 *   sharq_linear does not split run exactly as sharq_linear with no workspace.
 * - A shape whose split-K scratch would exceed 16 MiB returns SHARQ_ERR_UNSUPPORTED
 *   (use sharq_linear with a workspace of sharq_linear_workspace_size bytes instead).
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *   with that device current) and caches it per CUDA context, so a device reset (a new
 *   context) triggers a fresh lookup; make the first call in each context before any stream
 *   capture.
 * - Every call uses the same array and leaves its partial sums there; nothing in it has to
 *   start at zero (each call overwrites every value it reads). Calls that overlap on the
 *   GPU (different streams, or different host threads) race on the array. */
SHARQ_API sharq_status sharq_linear_noalloc(const sharq_act* act, const sharq_weight* w, void* Y,
                                            sharq_dtype y_dtype, void* stream);

/* Failure-detection self-test (no counterpart in the pages): launches one thread that
 * waits until the device word *flag equals `expected`, for at most limit_ns nanoseconds
 * (1 ms ... 10 s). On expiry it records SHARQ_ERR_TIMEOUT in the status word of `stream`
 * and returns, exactly as the GEMM's bounded pipeline waits do, so that a test can exercise
 * the detection path (sharq_read_device_status reports the timeout, the context stays
 * usable) without a fault. flag: device pointer, 4-byte aligned. Asynchronous on `stream`. */
SHARQ_API sharq_status sharq_wait_probe(const uint32_t* flag, uint32_t expected,
                                        uint64_t limit_ns, void* stream);

/* Status of the work enqueued on `stream` (no counterpart in the pages: failure detection).
 * A kernel that gives up on a bounded wait records SHARQ_ERR_TIMEOUT in the status word of
 * the stream it was launched on (one word per stream: the NULL stream has its own, the
 * first 63 other streams a context uses get one each, further streams share them round
 * robin). This call enqueues a one-thread kernel on `stream` that reads and clears that word
 * in one atomic exchange, copies the value back on `stream` and synchronises `stream` only
 * (other streams keep running). Returns SHARQ_OK or SHARQ_ERR_TIMEOUT for the work enqueued
 * on `stream` before the call (each timeout is reported once), or SHARQ_ERR_CUDA if the
 * launch, copy or synchronisation fails. Work on another stream that shares the slot
 * reports to it as well. Not for use while `stream` is being captured into a graph. */
SHARQ_API sharq_status sharq_read_device_status(void* stream);

/* Device-wide variant: synchronises the device, then reads and clears every stream's status
 * word (atomically, one exchange per word) and returns the first non-zero one (SHARQ_OK if
 * none), or SHARQ_ERR_CUDA if the synchronisation fails. */
SHARQ_API sharq_status sharq_device_status(void);

/* Static, human-readable name of a status code. */
SHARQ_API const char* sharq_status_string(sharq_status s);

#ifdef __cplusplus
}
#endif
#endif /* SHARQ_H */

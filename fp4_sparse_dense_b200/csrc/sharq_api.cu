// C ABI of the SharQ library: argument checks, buffer-size queries, TMA descriptor
// construction and the launches of the preparation, weight-quantisation and GEMM
// kernels. See include/sharq.h for the contract of every entry point.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include <cuda.h>
#include <cuda_runtime.h>

#include "sharq_internal.h"

namespace sharq {

// Unique id of the calling thread's current CUDA context (CUDA 12 context ids are never
// reused within a process, unlike context handles, so caches keyed on them are not fooled
// by a device reset that creates a new primary context). Initialises the device's primary
// context if none is current.
sharq_status current_context_id(unsigned long long* id) {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  if (!get_current || !get_id) return SHARQ_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return SHARQ_ERR_CUDA;
  if (!ctx) {  // no context yet: cudaSetDevice initialises the device's primary context
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess ||
        get_current(&ctx) != CUDA_SUCCESS || !ctx)
      return SHARQ_ERR_CUDA;
  }
  return get_id(ctx, id) == CUDA_SUCCESS ? SHARQ_OK : SHARQ_ERR_CUDA;
}

// Status words written by kernels that give up on a bounded wait: one word per stream
// slot (a stream's launches report to its slot), read and cleared by
// sharq_read_device_status (the stream's slot, in stream order) and sharq_device_status
// (every slot, after a device synchronisation). The arrays are per device image.
constexpr int kStatusSlots = 64;
__device__ unsigned int g_status_words[kStatusSlots];
__device__ unsigned int g_status_taken[kStatusSlots + 1];  // [kStatusSlots]: all slots

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per mbarrier wait

struct DeviceInfo {
  bool ok = false;
  int num_sms = 0;
  unsigned long long ctx_id = 0;
  unsigned int* status_words = nullptr;  // device addresses of the arrays above
  unsigned int* status_taken = nullptr;
};

std::mutex g_mu;
std::unordered_map<unsigned long long, DeviceInfo> g_dev;  // context id -> device facts
struct StreamKey {
  unsigned long long ctx;
  const void* stream;
  bool operator==(const StreamKey& o) const { return ctx == o.ctx && stream == o.stream; }
};
struct StreamKeyHash {
  size_t operator()(const StreamKey& k) const {
    return size_t(k.ctx * 0x9E3779B97F4A7C15ull) ^ reinterpret_cast<size_t>(k.stream);
  }
};
// Per stream: its status slot, and whether the GEMM may load its weight before waiting for
// the kernel launched just before it. That holds when the last launch of this library on the
// stream was a preparation or a linear call: each of their kernels waits for its own
// predecessor before it lets a dependent start, and none of them writes a weight. It does not
// hold on a stream not seen before, nor after sharq_quantize_weight.
struct StreamState {
  int slot = 0;
  bool weight_early = false;
};
std::unordered_map<StreamKey, StreamState, StreamKeyHash> g_streams;
std::unordered_map<unsigned long long, int> g_next_slot;  // context id -> next slot to hand out

sharq_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SHARQ_ERR_CUDA;
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) != SHARQ_OK) return SHARQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_dev.find(ctx);
  if (it != g_dev.end()) {
    *out = it->second;
    return out->ok ? SHARQ_OK : SHARQ_ERR_ARCH;
  }
  DeviceInfo d;
  d.ctx_id = ctx;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SHARQ_ERR_CUDA;
  d.ok = (major == 10 && minor == 0);
  if (d.ok) {
    void* w = nullptr;
    void* t = nullptr;
    if (cudaGetSymbolAddress(&w, g_status_words) != cudaSuccess ||
        cudaGetSymbolAddress(&t, g_status_taken) != cudaSuccess)
      return SHARQ_ERR_CUDA;
    d.status_words = static_cast<unsigned int*>(w);
    d.status_taken = static_cast<unsigned int*>(t);
  }
  g_dev[ctx] = d;
  *out = d;
  return d.ok ? SHARQ_OK : SHARQ_ERR_ARCH;
}

// State of `stream` (g_mu held). The NULL (legacy default) stream has slot 0; other streams
// get slots 1 .. kStatusSlots-1 in the order they are first seen, round robin beyond that.
StreamState& stream_state_locked(const DeviceInfo& d, cudaStream_t stream) {
  const StreamKey key{d.ctx_id, stream};
  auto it = g_streams.find(key);
  if (it != g_streams.end()) return it->second;
  if (g_streams.size() > 4096) g_streams.clear();
  StreamState st;
  if (stream != nullptr) {
    int& next = g_next_slot[d.ctx_id];
    st.slot = 1 + next % (kStatusSlots - 1);
    ++next;
  }
  return g_streams.emplace(key, st).first->second;
}

int stream_slot(const DeviceInfo& d, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  return stream_state_locked(d, stream).slot;
}

// Records the kind of this library's latest launch on `stream` and returns whether the one
// before it allowed the weight to be loaded early (see StreamState).
bool note_launch(const DeviceInfo& d, cudaStream_t stream, bool weight_early_after) {
  std::lock_guard<std::mutex> lk(g_mu);
  StreamState& st = stream_state_locked(d, stream);
  const bool before = st.weight_early;
  st.weight_early = weight_early_after;
  return before;
}

unsigned int* status_word(const DeviceInfo& d, cudaStream_t stream) {
  return d.status_words + stream_slot(d, stream);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sharq_status check_cfg(sharq_config c) {
  if (c.fmt != SHARQ_NVFP4 && c.fmt != SHARQ_MXFP4) return SHARQ_ERR_INVALID_ARG;
  if (c.mask < SHARQ_MASK_PAIR_4_8 || c.mask > SHARQ_MASK_NONE) return SHARQ_ERR_INVALID_ARG;
  if (c.residual < 0 || c.residual > 3) return SHARQ_ERR_INVALID_ARG;
  // the residual's own tensor scale exists for NVFP4 (MXFP4 has no tensor scale) and is
  // built for the pair mask
  if (c.residual == 3 && (c.fmt != SHARQ_NVFP4 || !is_pair_mask(c.mask)))
    return SHARQ_ERR_UNSUPPORTED;
  return SHARQ_OK;
}

size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }
size_t tiled_bytes(size_t rows, size_t cols) { return round_up(rows, 128) * round_up(cols, 4); }

sharq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA; }

// ------------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct MapKey {
  const void* ptr;
  int rank, dtype, swz;
  uint64_t dims[4], strides[3];
  uint32_t box[4];
  bool operator==(const MapKey& o) const {
    if (ptr != o.ptr || rank != o.rank || dtype != o.dtype || swz != o.swz) return false;
    for (int i = 0; i < 4; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    for (int i = 0; i < 3; ++i)
      if (strides[i] != o.strides[i]) return false;
    return true;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = reinterpret_cast<uint64_t>(k.ptr) * 0x9E3779B97F4A7C15ull;
    auto mix = [&](uint64_t v) { h ^= v + 0x9E3779B97F4A7C15ull + (h << 6) + (h >> 2); };
    mix(uint64_t(k.rank) | uint64_t(k.dtype) << 8 | uint64_t(k.swz) << 16);
    for (int i = 0; i < 4; ++i) mix(k.dims[i] ^ (uint64_t(k.box[i]) << 40));
    for (int i = 0; i < 3; ++i) mix(k.strides[i]);
    return size_t(h);
  }
};
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

// Tensor map of a `rank`-dimensional tensor: dims in elements (innermost first), strides
// in bytes of dimensions 1..rank-1, box in elements. Cached by (pointer, shape).
sharq_status make_map_nd(CUtensorMap* out, const void* ptr, CUtensorMapDataType dtype, int rank,
                         const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                         CUtensorMapSwizzle swz) {
  MapKey key{};
  key.ptr = ptr;
  key.rank = rank;
  key.dtype = int(dtype);
  key.swz = int(swz);
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i > 0) key.strides[i - 1] = strides[i - 1];
  }
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return SHARQ_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return SHARQ_ERR_CUDA;
  cuuint64_t d[4], st[3];
  cuuint32_t b[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    if (i > 0) st[i - 1] = strides[i - 1];
  }
  CUresult r = fn(out, dtype, cuuint32_t(rank), const_cast<void*>(ptr), d, st, b, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return SHARQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps[key] = *out;
  return SHARQ_OK;
}

// 2-D byte matrix [rows][inner] (row pitch = inner), box [box_rows][box_inner]
sharq_status make_map(CUtensorMap* out, const void* ptr, uint64_t inner, uint64_t rows,
                      uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  const uint64_t dims[2] = {inner, rows};
  const uint64_t strides[1] = {inner};
  const uint32_t box[2] = {box_inner, box_rows};
  return make_map_nd(out, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, dims, strides, box, swz);
}

// bf16 output Y[M][N]: 32 x 32 boxes with the 64-byte swizzle of the epilogue staging
sharq_status make_y_map(CUtensorMap* out, const void* Y, int M, int N) {
  const uint64_t dims[2] = {uint64_t(N), uint64_t(M)};
  const uint64_t strides[1] = {uint64_t(N) * 2};
  const uint32_t box[2] = {32, 32};
  return make_map_nd(out, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_64B);
}

// weight scales seen as [N/128 row blocks][K/256 steps][rows_per_step][256 bytes], so that
// one box fetches the chunks of both 128-row halves of a 256-row tile for one K step
sharq_status make_wscale_map(CUtensorMap* out, const void* ptr, int K, int N, uint32_t rows_per_step) {
  const uint64_t KT = uint64_t(K) / 256;
  const uint64_t dims[4] = {256, rows_per_step, KT, uint64_t(N) / 128};
  const uint64_t strides[3] = {256, uint64_t(rows_per_step) * 256, KT * rows_per_step * 256};
  const uint32_t box[4] = {256, rows_per_step, 1, 2};
  return make_map_nd(out, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
}

sharq_status act_sizes(int32_t M, int32_t K, sharq_config c, sharq_act_bytes* o) {
  if (!o || M < 1 || K < 256 || K % 256 != 0) return SHARQ_ERR_INVALID_ARG;
  sharq_status s = check_cfg(c);
  if (s != SHARQ_OK) return s;
  const bool pair = is_pair_mask(c.mask);
  const size_t m = size_t(M), k = size_t(K);
  o->bq = pair ? m * k / 4 : m * k / 2;
  o->bs = tiled_bytes(m, k / size_t(backbone_block(c.fmt, c.mask)));
  o->bm = pair ? round_up(m, 128) * k / 16 : (c.mask == SHARQ_MASK_NONE ? 0 : m * k / 8);
  o->rq = c.residual ? m * k / 2 : 0;
  o->rs = c.residual ? tiled_bytes(m, k / size_t(residual_block(c.fmt))) : 0;
  return SHARQ_OK;
}

sharq_status weight_sizes(int32_t K, int32_t N, sharq_config c, sharq_weight_bytes* o) {
  if (!o || K < 256 || K % 256 != 0 || N < 128 || N % 128 != 0) return SHARQ_ERR_INVALID_ARG;
  sharq_status s = check_cfg(c);
  if (s != SHARQ_OK) return s;
  const size_t k = size_t(K), n = size_t(N);
  o->codes = n * k / 2;
  o->scales_dense = tiled_bytes(n, k / size_t(dense_view_block(c.fmt)));
  o->scales_sparse = is_pair_mask(c.mask) ? tiled_bytes(n, k / 32) : 0;
  return SHARQ_OK;
}

}  // namespace
}  // namespace sharq

using namespace sharq;

namespace sharq {
namespace {
// The preparation entry points: gamma == nullptr prepares X as given; otherwise the
// RMSNorm of X with (gamma, eps), writing the per-row rstd. alongside: launch sized to
// share the SMs with a GEMM running on another stream (same results).
sharq_status prepare_impl(const void* X, sharq_dtype dtype, const sharq_act* a, const void* gamma,
                          float eps, float* rstd, void* stream, bool alongside = false,
                          const float* amax_in = nullptr) {
  if (!X || !a) return SHARQ_ERR_INVALID_ARG;
  if (dtype != SHARQ_F16 && dtype != SHARQ_BF16) return SHARQ_ERR_INVALID_ARG;
  sharq_act_bytes sz;
  sharq_status s = act_sizes(a->M, a->K, a->cfg, &sz);
  if (s != SHARQ_OK) return s;
  const bool res = a->cfg.residual != 0;
  const bool norm = gamma != nullptr;
  const bool pair = is_pair_mask(a->cfg.mask), none = a->cfg.mask == SHARQ_MASK_NONE;
  if (norm && !pair) return SHARQ_ERR_UNSUPPORTED;
  // a supplied tensor amax: NVFP4, the method's pair mask, a residual with the shared s_g
  // (or none), no RMSNorm
  if (amax_in && ((reinterpret_cast<uintptr_t>(amax_in) & 3u) != 0)) return SHARQ_ERR_MISALIGNED;
  if (amax_in && (a->cfg.fmt != SHARQ_NVFP4 || a->cfg.mask != SHARQ_MASK_PAIR_4_8 ||
                  a->cfg.residual == 2 || a->cfg.residual == 3 || norm))
    return SHARQ_ERR_UNSUPPORTED;
  // the pair-mask kernels address X and their outputs with 32-bit offsets
  if (pair && size_t(a->M) * size_t(a->K) >= (size_t(1) << 31)) return SHARQ_ERR_UNSUPPORTED;
  if (!a->bq || !a->bs || (!a->bm && !none) || !a->tensor_scale || (res && (!a->rq || !a->rs)) ||
      (norm && !rstd))
    return SHARQ_ERR_INVALID_ARG;
  if (norm && !(eps >= 0.f && eps < 1e30f)) return SHARQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(a->bq) || !aligned16(a->bs) || !aligned16(a->bm) ||
      !aligned16(a->tensor_scale) || (res && (!aligned16(a->rq) || !aligned16(a->rs))) ||
      (norm && (!aligned16(gamma) || !aligned16(rstd))))
    return SHARQ_ERR_MISALIGNED;
  DeviceInfo d;
  if ((s = device_info(&d)) != SHARQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == SHARQ_BF16;
  // the pair-mask kernels reduce the NVFP4 tensor amax themselves (state in
  // tensor_scale[2..3]); the element-mask kernel takes it from a separate pass into
  // tensor_scale[1]
  if (a->cfg.fmt == SHARQ_NVFP4 && !pair) {
    if (cudaMemsetAsync(a->tensor_scale + 1, 0, sizeof(float), st) != cudaSuccess)
      return SHARQ_ERR_CUDA;
    s = from_cuda(launch_amax(X, bf16, size_t(a->M) * size_t(a->K),
                              reinterpret_cast<unsigned int*>(a->tensor_scale + 1), d.num_sms, st));
    if (s != SHARQ_OK) return s;
  }
  PrepParams p;
  p.X = X;
  p.bq = a->bq;
  p.bs = a->bs;
  p.bm = a->bm;
  p.rq = a->rq;
  p.rs = a->rs;
  p.tensor_scale = a->tensor_scale;
  p.amax = a->tensor_scale + 1;
  p.M = a->M;
  p.K = a->K;
  p.Mp = int(round_up(size_t(a->M), 128));
  p.status = status_word(d, st);
  p.timeout_ns = kWaitLimitNs;
  p.gamma = gamma;
  p.rstd = rstd;
  p.eps = eps;
  p.mask_given = a->cfg.mask == SHARQ_MASK_PAIR_4_8_GIVEN;
  p.keep_all = none;
  p.res_unquant = a->cfg.residual == 2;
  p.alongside = alongside ? 1 : 0;
  p.res_phase = 0;
  p.amax_in = amax_in;
  if (a->cfg.residual != 3) {
    s = from_cuda(launch_prep(p, bf16, a->cfg.fmt, a->cfg.mask, res, d.num_sms, st));
  } else {
    // the residual's own tensor scale: amax|r| is a grid-wide reduction that follows the
    // backbone's quantisation, so the quantisation runs twice (backbone + amax|r|, then the
    // residual with s_r)
    p.res_phase = 1;
    s = from_cuda(launch_prep(p, bf16, a->cfg.fmt, a->cfg.mask, res, d.num_sms, st));
    if (s == SHARQ_OK) {
      p.res_phase = 2;
      s = from_cuda(launch_prep(p, bf16, a->cfg.fmt, a->cfg.mask, res, d.num_sms, st));
    }
  }
  note_launch(d, st, s == SHARQ_OK);
  return s;
}
}  // namespace
}  // namespace sharq

namespace sharq {
namespace {
// One thread waits for *flag == expected with the same bounded-wait discipline as the
// GEMM's pipeline waits; on expiry the status word gets SHARQ_ERR_TIMEOUT.
__global__ void wait_probe_kernel(const uint32_t* flag, uint32_t expected, uint64_t limit_ns,
                                  unsigned int* status) {
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t it = 0;; ++it) {
    if (*reinterpret_cast<const volatile uint32_t*>(flag) == expected) return;
    if ((it & 63u) == 0) {
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > limit_ns) {
        atomicExch(status, unsigned(SHARQ_ERR_TIMEOUT));
        return;
      }
    }
    __nanosleep(1000);
  }
}

// Reads and clears status words atomically: slot >= 0 moves that slot's word into
// taken[slot]; slot < 0 clears every slot and leaves the first non-zero word (in slot
// order) in taken[kStatusSlots]. One thread: at most kStatusSlots atomics.
__global__ void status_take_kernel(unsigned int* words, unsigned int* taken, int slot) {
  if (slot >= 0) {
    taken[slot] = atomicExch(words + slot, 0u);
    return;
  }
  unsigned int first = 0;
  for (int i = 0; i < kStatusSlots; ++i) {
    const unsigned int v = atomicExch(words + i, 0u);
    if (first == 0) first = v;
  }
  taken[kStatusSlots] = first;
}
}  // namespace
}  // namespace sharq

extern "C" {

const char* sharq_status_string(sharq_status s) {
  switch (s) {
    case SHARQ_OK: return "SHARQ_OK";
    case SHARQ_ERR_INVALID_ARG: return "SHARQ_ERR_INVALID_ARG";
    case SHARQ_ERR_UNSUPPORTED: return "SHARQ_ERR_UNSUPPORTED";
    case SHARQ_ERR_MISALIGNED: return "SHARQ_ERR_MISALIGNED";
    case SHARQ_ERR_CUDA: return "SHARQ_ERR_CUDA";
    case SHARQ_ERR_TIMEOUT: return "SHARQ_ERR_TIMEOUT";
    case SHARQ_ERR_ARCH: return "SHARQ_ERR_ARCH";
  }
  return "SHARQ_ERR_UNKNOWN";
}

sharq_status sharq_act_sizes(int32_t M, int32_t K, sharq_config cfg, sharq_act_bytes* out) {
  return act_sizes(M, K, cfg, out);
}

sharq_status sharq_weight_sizes(int32_t K, int32_t N, sharq_config cfg, sharq_weight_bytes* out) {
  return weight_sizes(K, N, cfg, out);
}

sharq_status sharq_quantize_weight(const void* W, sharq_dtype dtype, const sharq_weight* w,
                                   void* stream) {
  if (!W || !w) return SHARQ_ERR_INVALID_ARG;
  if (dtype != SHARQ_F16 && dtype != SHARQ_BF16) return SHARQ_ERR_INVALID_ARG;
  sharq_weight_bytes sz;
  sharq_status s = weight_sizes(w->K, w->N, w->cfg, &sz);
  if (s != SHARQ_OK) return s;
  const bool pair = is_pair_mask(w->cfg.mask);
  if (!w->codes || !w->scales_dense || !w->tensor_scale || (pair && !w->scales_sparse))
    return SHARQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(w->codes) || !aligned16(w->scales_dense) ||
      !aligned16(w->tensor_scale) || (pair && !aligned16(w->scales_sparse)))
    return SHARQ_ERR_MISALIGNED;
  DeviceInfo d;
  if ((s = device_info(&d)) != SHARQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  note_launch(d, st, false);  // a GEMM launched next must not read this weight early
  const bool bf16 = dtype == SHARQ_BF16;
  if (w->cfg.fmt == SHARQ_NVFP4) {
    if (cudaMemsetAsync(w->tensor_scale + 1, 0, sizeof(float), st) != cudaSuccess)
      return SHARQ_ERR_CUDA;
    s = from_cuda(launch_amax(W, bf16, size_t(w->K) * size_t(w->N),
                              reinterpret_cast<unsigned int*>(w->tensor_scale + 1), d.num_sms, st));
    if (s != SHARQ_OK) return s;
  }
  WeightQuantParams p;
  p.W = W;
  p.codes = static_cast<uint8_t*>(w->codes);
  p.scales_dense = static_cast<uint8_t*>(w->scales_dense);
  p.scales_sparse = static_cast<uint8_t*>(w->scales_sparse);
  p.tensor_scale = w->tensor_scale;
  p.K = w->K;
  p.N = w->N;
  return from_cuda(launch_weight_quant(p, bf16, w->cfg.fmt, w->cfg.mask, st));
}

sharq_status sharq_prepare(const void* X, sharq_dtype dtype, const sharq_act* a, void* stream) {
  return sharq::prepare_impl(X, dtype, a, nullptr, 0.f, nullptr, stream);
}

sharq_status sharq_prepare_alongside(const void* X, sharq_dtype dtype, const sharq_act* a,
                                    void* stream) {
  return sharq::prepare_impl(X, dtype, a, nullptr, 0.f, nullptr, stream, true);
}

sharq_status sharq_prepare_given_amax(const void* X, sharq_dtype dtype, const float* amax,
                                      const sharq_act* a, void* stream) {
  if (!amax) return SHARQ_ERR_INVALID_ARG;
  return sharq::prepare_impl(X, dtype, a, nullptr, 0.f, nullptr, stream, false, amax);
}

sharq_status sharq_prepare_rmsnorm(const void* X, const void* gamma, float eps, sharq_dtype dtype,
                                   float* rstd, const sharq_act* a, void* stream) {
  if (!gamma) return SHARQ_ERR_INVALID_ARG;
  return sharq::prepare_impl(X, dtype, a, gamma, eps, rstd, stream);
}

sharq_status sharq_linear_workspace_size(int32_t M, int32_t N, int32_t K, sharq_config cfg,
                                         size_t* bytes) {
  if (!bytes) return SHARQ_ERR_INVALID_ARG;
  sharq_act_bytes asz;
  sharq_weight_bytes wsz;
  sharq_status s = act_sizes(M, K, cfg, &asz);
  if (s != SHARQ_OK) return s;
  if ((s = weight_sizes(K, N, cfg, &wsz)) != SHARQ_OK) return s;
  DeviceInfo d;
  if ((s = device_info(&d)) != SHARQ_OK) return s;
  const int splits = cfg.residual == 3 ? 1 : plan_splits(M, N, K, d.num_sms);
  *bytes = splits > 1 ? size_t(splits) * size_t(M) * size_t(N) * sizeof(float) : 0;
  return SHARQ_OK;
}

sharq_status sharq_linear(const sharq_act* a, const sharq_weight* w, void* Y, sharq_dtype y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!a || !w || !Y) return SHARQ_ERR_INVALID_ARG;
  if (y_dtype != SHARQ_BF16 && y_dtype != SHARQ_F32) return SHARQ_ERR_INVALID_ARG;
  if (std::memcmp(&a->cfg, &w->cfg, sizeof(sharq_config)) != 0 || a->K != w->K)
    return SHARQ_ERR_INVALID_ARG;
  sharq_act_bytes asz;
  sharq_weight_bytes wsz;
  sharq_status s = act_sizes(a->M, a->K, a->cfg, &asz);
  if (s != SHARQ_OK) return s;
  if ((s = weight_sizes(w->K, w->N, w->cfg, &wsz)) != SHARQ_OK) return s;
  const bool res = a->cfg.residual != 0, pair = is_pair_mask(a->cfg.mask);
  if (!a->bq || !a->bs || !a->tensor_scale || (pair && !a->bm) || (res && (!a->rq || !a->rs)) ||
      !w->codes || !w->tensor_scale || ((res || !pair) && !w->scales_dense) ||
      (pair && !w->scales_sparse))
    return SHARQ_ERR_INVALID_ARG;
  if (!aligned16(Y) || !aligned16(a->bq) || !aligned16(a->bs) || !aligned16(a->bm) ||
      !aligned16(a->rq) || !aligned16(a->rs) || !aligned16(w->codes) ||
      !aligned16(w->scales_dense) || !aligned16(w->scales_sparse))
    return SHARQ_ERR_MISALIGNED;
  DeviceInfo d;
  if ((s = device_info(&d)) != SHARQ_OK) return s;
  const int M = a->M, K = a->K, N = w->N;
  GemmParams p;
  p.bs = static_cast<const uint8_t*>(a->bs);
  p.bm = static_cast<const uint8_t*>(a->bm);
  p.rs = static_cast<const uint8_t*>(a->rs);
  p.wsd = static_cast<const uint8_t*>(w->scales_dense);
  p.wss = static_cast<const uint8_t*>(w->scales_sparse);
  p.act_ts = a->tensor_scale;
  p.w_ts = w->tensor_scale;
  p.Y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.Mp = int(round_up(size_t(M), 128));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  p.status = status_word(d, st);
  p.timeout_ns = kWaitLimitNs;
  p.splits = 1;
  p.n_fast = 0;
  p.prefetch_w = 0;
  p.ws = nullptr;

  const bool own = a->cfg.residual == 3;  // residual with its own tensor scale
  if (M >= 256 && N % 256 == 0 && !own) {
    // CTA-pair kernel: 256 x 256 tiles, half of the weight tile per CTA
    const bool nv = a->cfg.fmt == SHARQ_NVFP4;
    const uint32_t dch_rows = uint32_t(256 / (nv ? 16 : 32) / 4) * 2;  // 256-byte rows per K step
    GemmPairMaps pm;
    std::memset(&pm, 0, sizeof(pm));
    if ((s = make_map(&pm.w, w->codes, uint64_t(K) / 2, uint64_t(N), 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != SHARQ_OK)
      return s;
    if (pair)
      s = make_map(&pm.b, a->bq, uint64_t(K) / 4, uint64_t(M), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B);
    else
      s = make_map(&pm.b, a->bq, uint64_t(K) / 2, uint64_t(M), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != SHARQ_OK) return s;
    if (res && (s = make_map(&pm.r, a->rq, uint64_t(K) / 2, uint64_t(M), 128, 128,
                             CU_TENSOR_MAP_SWIZZLE_128B)) != SHARQ_OK)
      return s;
    if (!res) pm.r = pm.b;
    auto view = [&](CUtensorMap* mp, const void* ptr, size_t bytes, uint32_t rows) {
      return make_map(mp, ptr, 256, uint64_t(bytes / 256), 256, rows, CU_TENSOR_MAP_SWIZZLE_NONE);
    };
    if (res && (s = view(&pm.rs, a->rs, asz.rs, dch_rows)) != SHARQ_OK) return s;
    if ((s = view(&pm.bs, a->bs, asz.bs, pair ? 4 : dch_rows)) != SHARQ_OK) return s;
    if (pair && (s = view(&pm.bm, a->bm, asz.bm, 8)) != SHARQ_OK) return s;
    if ((res || !pair) &&
        (s = make_wscale_map(&pm.wsd, w->scales_dense, K, N, dch_rows)) != SHARQ_OK)
      return s;
    if (pair && (s = make_wscale_map(&pm.wss, w->scales_sparse, K, N, 4)) != SHARQ_OK) return s;
    if (y_dtype == SHARQ_BF16 && (s = make_y_map(&pm.y, Y, M, N)) != SHARQ_OK) return s;
    if (!res) pm.rs = pm.bs;
    if (!pair) pm.bm = pm.bs, pm.wss = pm.wsd;
    if (pair && !res) pm.wsd = pm.wss;
    p.tiles_m = (M + 127) / 128;
    p.tiles_n = N / 256;
    // Raster order: the operand whose whole payload is smaller stays in L2 while the other
    // streams through once. With M fastest every wave touches all activation rows (reused
    // across the weight's column tiles), with N fastest every wave touches the whole weight.
    {
      const double act_bytes = double(asz.bq) + double(asz.bs) + double(asz.bm) +
                               double(asz.rq) + double(asz.rs);
      const double w_bytes = double(wsz.codes) + double(wsz.scales_dense) +
                             double(pair ? wsz.scales_sparse : 0);
      p.n_fast = act_bytes > w_bytes ? 1 : 0;
    }
    return from_cuda(launch_gemm_pair(pm, p, a->cfg.fmt, a->cfg.mask, res, y_dtype == SHARQ_F32,
                                      d.num_sms, st));
  }

  // two accumulators (own residual scale) take 128 + 128 tensor-memory columns: BN = 128
  const int BN = (N % 256 == 0 && !own) ? 256 : 128;
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if ((s = make_map(&maps.w, w->codes, uint64_t(K) / 2, uint64_t(N), 128, uint32_t(BN),
                    CU_TENSOR_MAP_SWIZZLE_128B)) != SHARQ_OK)
    return s;
  if (pair)
    s = make_map(&maps.b, a->bq, uint64_t(K) / 4, uint64_t(M), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  else
    s = make_map(&maps.b, a->bq, uint64_t(K) / 2, uint64_t(M), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SHARQ_OK) return s;
  if (res && (s = make_map(&maps.r, a->rq, uint64_t(K) / 2, uint64_t(M), 128, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SHARQ_OK)
    return s;
  if (!res) maps.r = maps.b;
  if (y_dtype == SHARQ_BF16 && (s = make_y_map(&maps.y, Y, M, N)) != SHARQ_OK) return s;
  {
    const int splits = plan_splits(M, N, K, d.num_sms);
    const size_t need = size_t(splits) * size_t(M) * size_t(N) * sizeof(float);
    if (splits > 1 && !own && workspace && workspace_bytes >= need && aligned16(workspace)) {
      p.splits = splits;
      p.ws = static_cast<float*>(workspace);
    }
  }
  p.tiles_m = (M + 127) / 128;
  p.tiles_n = N / BN;
  // decode-sized M: the weight stream dominates; its first stages are loaded while the
  // kernel launched just before (normally the preparation) is still running, when that kernel
  // is one of this library's that writes no weight (see StreamState)
  const bool weight_early = note_launch(d, st, true);
  p.prefetch_w = (M < 256 && weight_early) ? 1 : 0;
  if (own) return from_cuda(launch_gemm_two(maps, p, y_dtype == SHARQ_F32, d.num_sms, st));
  return from_cuda(launch_gemm(maps, p, a->cfg.fmt, a->cfg.mask, res, y_dtype == SHARQ_F32,
                               d.num_sms, st));
}

sharq_status sharq_wait_probe(const uint32_t* flag, uint32_t expected, uint64_t limit_ns,
                              void* stream) {
  if (!flag || (reinterpret_cast<uintptr_t>(flag) & 3u) != 0) return SHARQ_ERR_INVALID_ARG;
  if (limit_ns < 1000000ull || limit_ns > 10000000000ull) return SHARQ_ERR_INVALID_ARG;
  DeviceInfo d;
  sharq_status s = device_info(&d);
  if (s != SHARQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  wait_probe_kernel<<<1, 1, 0, st>>>(flag, expected, limit_ns, status_word(d, st));
  return from_cuda(cudaGetLastError());
}

sharq_status sharq_read_device_status(void* stream) {
  DeviceInfo d;
  sharq_status s = device_info(&d);
  if (s != SHARQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int slot = stream_slot(d, st);
  // in stream order: after every kernel this stream launched before the call
  status_take_kernel<<<1, 1, 0, st>>>(d.status_words, d.status_taken, slot);
  if (cudaGetLastError() != cudaSuccess) return SHARQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, d.status_taken + slot, sizeof(v), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SHARQ_ERR_CUDA;
  return v == 0 ? SHARQ_OK : static_cast<sharq_status>(v);
}

sharq_status sharq_device_status(void) {
  DeviceInfo d;
  sharq_status s = device_info(&d);
  if (s != SHARQ_OK) return s;
  if (cudaDeviceSynchronize() != cudaSuccess) return SHARQ_ERR_CUDA;
  status_take_kernel<<<1, 1>>>(d.status_words, d.status_taken, -1);
  if (cudaGetLastError() != cudaSuccess) return SHARQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, d.status_taken + kStatusSlots, sizeof(v), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return SHARQ_ERR_CUDA;
  return v == 0 ? SHARQ_OK : static_cast<sharq_status>(v);
}

}  // extern "C"

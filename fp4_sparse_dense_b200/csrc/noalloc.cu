// sharq_linear_noalloc: the linear layer for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a scratch buffer: code running inside a CUDA graph
// that must not grow the memory pool, allocator-free inference runtimes, or hosts whose
// memory manager forbids allocation on the hot path. For decode-sized M, sharq_linear
// splits K and needs an FP32 workspace for the partial sums. This entry point gives such
// callers the same result without any allocation: the workspace is a fixed device array
// compiled into the library (kNoAllocScratchBytes per GPU, held by every GPU that loads the
// library until the process exits). No cudaMalloc / cudaFree or allocating library routine
// is called.
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <unordered_map>

#include <cuda_runtime.h>

#include "sharq_internal.h"

namespace sharq {
namespace {

// Maximum split-K scratch served by sharq_linear_noalloc: 16 MiB per device.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

// The scratch itself. Host code must not use this symbol as an address: its device
// address comes from cudaGetSymbolAddress, taken once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
// context id -> device address of the array in that context. A device reset creates a new
// primary context with a new id, so an address from before the reset is never reused.
std::unordered_map<unsigned long long, void*> g_scratch_addr;

// Device address of the scratch in the current context; looked up with
// cudaGetSymbolAddress on the first call in each context (with that device current) and
// cached.
sharq_status scratch_address(void** out) {
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) != SHARQ_OK) return SHARQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  auto it = g_scratch_addr.find(ctx);
  if (it != g_scratch_addr.end()) {
    *out = it->second;
    return SHARQ_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return SHARQ_ERR_CUDA;
  g_scratch_addr[ctx] = p;
  *out = p;
  return SHARQ_OK;
}

}  // namespace
}  // namespace sharq

extern "C" sharq_status sharq_linear_noalloc(const sharq_act* act, const sharq_weight* w, void* Y,
                                             sharq_dtype y_dtype, void* stream) {
  using namespace sharq;
  if (!act || !w) return SHARQ_ERR_INVALID_ARG;
  size_t need = 0;
  sharq_status s = sharq_linear_workspace_size(act->M, w->N, act->K, act->cfg, &need);
  if (s != SHARQ_OK) return s;
  if (need > kNoAllocScratchBytes) return SHARQ_ERR_UNSUPPORTED;  // shape needs more scratch
  void* scratch = nullptr;
  if (need > 0 && (s = scratch_address(&scratch)) != SHARQ_OK) return s;
  return sharq_linear(act, w, Y, y_dtype, scratch, need > 0 ? kNoAllocScratchBytes : 0, stream);
}

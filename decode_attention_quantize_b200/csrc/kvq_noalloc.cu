// Allocation-free decode attention: the existing decode path with its workspace taken
// from a static device array instead of caller memory.
#include <cuda.h>

#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace {

// Split partials and the paged plan of kvq_decode_attention, for callers that cannot allocate.
// Held by every GPU that loads the library until the process exits.
static __device__ __align__(256) uint8_t g_decode_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
// Device address of g_decode_scratch per device ordinal, and the CUDA context it was looked up
// in: the address belongs to that context, so a different current context (after a device
// reset, or a caller's own driver context) looks it up again.
void* g_scratch_ptr[kMaxDevices];
CUcontext g_scratch_ctx[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  return fn;
}

// Device address of the array on the current device, looked up once per (device, context).
// In host code g_decode_scratch names a host-side stand-in, never the device memory itself.
kvq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return KVQ_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    // the look-up makes the runtime's context current when no context is yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return KVQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_cache_desc* desc, const void* q, int32_t q_dtype,
                                                   float softmax_scale, float* out, float* lse, void* stream) {
  const kvq_status st = kvq_validate(desc);
  if (st != KVQ_OK) return st;
  if (kvq_decode_workspace_bytes(desc) > KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const kvq_status sa = scratch_address(&scratch);
  if (sa != KVQ_OK) return sa;
  return kvq_decode_attention(desc, q, q_dtype, softmax_scale, out, lse, scratch, KVQ_NOALLOC_SCRATCH_BYTES,
                              stream);
}

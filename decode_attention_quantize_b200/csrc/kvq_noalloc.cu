// Allocation-free decode attention: the existing decode path with its workspace taken
// from a static device array instead of caller memory.
#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace {

// Split partials and the paged plan of kvq_decode_attention, for callers that cannot
// allocate. Held by every GPU that loads the library until the process exits.
static __device__ __align__(256) uint8_t g_decode_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];  // device address of g_decode_scratch, per device ordinal

// Device address of the array on the current device, looked up once per device. In host
// code g_decode_scratch names a host-side stand-in, never the device memory itself.
kvq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
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

// C-ABI entry points of libkvq: argument validation (host only, before any launch),
// workspace queries, footprint arithmetic and kernel launches.
#include <atomic>
#include <cstring>

#include "kvq_device.cuh"
#include "kvq_internal.h"

using namespace kvq;

namespace kvq {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// One warp waits on a barrier whose phase never completes (nothing arrives), through the
// library's bounded wait: it gives up after the wait limit and flags KVQ_DEV_TIMEOUT.
__global__ void bounded_wait_check_kernel(uint32_t* status) {
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = smem_addr(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  mbar_wait(bar, 0, status);
}
}  // namespace kvq

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxQHeads = 8192;  // query heads per sequence the decode accepts
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_scheme(int s) { return s >= KVQ_FP8_E4M3_PER_TENSOR && s <= KVQ_KIVI_INT2_F16; }

bool needs_scale(int s) { return true; }
bool needs_zp(int s) { return s == KVQ_UINT8_ASYM_PER_CHANNEL; }

// Per-side metadata element counts (floats) for the layouts in kvq.h.
uint64_t scale_elems(const kvq_cache_desc* d, int side) {
  const int s = side ? d->v_scheme : d->k_scheme;
  const uint64_t B = d->batch, H = d->num_kv_heads, D = d->head_dim;
  const bool paged = d->layout == KVQ_PAGED;
  switch (s) {
    case KVQ_FP8_E4M3_PER_TENSOR:
    case KVQ_FP8_E5M2_PER_TENSOR:
    case KVQ_INT8_SYM_PER_TENSOR: return 1;
    case KVQ_INT8_SYM_PER_TOKEN:
      return paged ? (uint64_t)d->num_pages * H * d->page_size : B * H * (uint64_t)d->capacity;
    case KVQ_INT8_SYM_PER_CHANNEL:
    case KVQ_UINT8_ASYM_PER_CHANNEL: return H * D;
    case KVQ_INT4_SYM_PER_GROUP:
      return (paged ? (uint64_t)d->num_pages * H * d->page_size : B * H * (uint64_t)d->capacity) *
             (D / (uint64_t)d->group_size);
    default:
      return side == 0 ? B * H * (uint64_t)(d->capacity / 32) * D : B * H * (uint64_t)d->capacity * (D / 32);
  }
}

kvq_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return KVQ_OK;
  if (e == cudaErrorNotSupported) return KVQ_ERR_UNSUPPORTED;
  return KVQ_ERR_CUDA;
}

int seq_capacity(const kvq_cache_desc* d) {
  return d->layout == KVQ_PAGED ? d->max_pages_per_seq * d->page_size : d->capacity;
}

}  // namespace

extern "C" {

int kvq_abi_version(void) { return KVQ_ABI_VERSION; }

uint64_t kvq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

kvq_status kvq_validate(const kvq_cache_desc* d) {
  if (!d) return KVQ_ERR_INVALID_ARG;
  if (d->batch < 1 || d->num_kv_heads < 1 || d->num_q_heads < d->num_kv_heads ||
      d->num_q_heads % d->num_kv_heads != 0 || d->batch > 65535 || d->num_kv_heads > 1024)
    return KVQ_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return d->head_dim > 0 ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_INVALID_ARG;
  if (!valid_scheme(d->k_scheme) || !valid_scheme(d->v_scheme)) return KVQ_ERR_INVALID_ARG;
  if (d->layout != KVQ_DENSE && d->layout != KVQ_PAGED) return KVQ_ERR_INVALID_ARG;
  const bool kivi_k = is_kivi(d->k_scheme), kivi_v = is_kivi(d->v_scheme);
  if (d->rotation != KVQ_ROTATE_NONE && d->rotation != KVQ_ROTATE_HADAMARD) return KVQ_ERR_INVALID_ARG;
  if (d->rotation != KVQ_ROTATE_NONE && (kivi_k || kivi_v)) return KVQ_ERR_UNSUPPORTED;
  // pre-RoPE keys: a finite base >= 0; with 8-bit key codes, without the Hadamard rotation
  if (!(d->rope_theta >= 0.0f) || d->rope_theta > 3.0e38f) return KVQ_ERR_INVALID_ARG;
  if (d->rope_theta > 0.0f && (d->rotation != KVQ_ROTATE_NONE || code_bits(d->k_scheme) != 8))
    return KVQ_ERR_UNSUPPORTED;
  if (kivi_k || kivi_v) {
    if (d->k_scheme != d->v_scheme) return KVQ_ERR_UNSUPPORTED;
    if (d->layout == KVQ_PAGED) return KVQ_ERR_UNSUPPORTED;
    if (d->group_size != 32 || d->residual_cap != 128) return KVQ_ERR_UNSUPPORTED;
    if (!d->k_zero || !d->v_zero || !d->k_res || !d->v_res) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(d->k_zero) || !aligned16(d->v_zero) || !aligned16(d->k_res) || !aligned16(d->v_res))
      return KVQ_ERR_INVALID_ARG;
    if (d->num_residual < 0 || d->num_residual > d->residual_cap) return KVQ_ERR_INVALID_ARG;
  }
  if ((d->k_scheme == KVQ_INT4_SYM_PER_GROUP || d->v_scheme == KVQ_INT4_SYM_PER_GROUP) &&
      d->group_size != 32 && d->group_size != 64 && d->group_size != 128)
    return KVQ_ERR_UNSUPPORTED;
  // The decode's split plan counts (sequence, kv head, head group) pairs and their tiles in
  // 32-bit integers: bound the pair count, and below the tile count of a full cache.
  if (d->num_q_heads > kMaxQHeads) return KVQ_ERR_UNSUPPORTED;
  const uint64_t pairs = (uint64_t)d->batch * d->num_kv_heads * (uint64_t)((d->num_q_heads / d->num_kv_heads + 7) / 8);
  if (pairs >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
  if (d->layout == KVQ_DENSE) {
    if (d->capacity < 128 || d->capacity % 128 != 0) return KVQ_ERR_INVALID_ARG;
    if ((uint64_t)d->batch * d->num_kv_heads * (uint64_t)d->capacity >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
    // quantized tiles of 128 tokens plus at most four residual tiles of 32 per pair
    if (pairs * (uint64_t)(d->capacity / 128 + 4) >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
    if (d->num_quantized < 0 || d->num_quantized > d->capacity) return KVQ_ERR_INVALID_ARG;
    if ((kivi_k) && d->num_quantized % 128 != 0) return KVQ_ERR_INVALID_ARG;
  } else {
    if (d->page_size != 16 && d->page_size != 32 && d->page_size != 64) return KVQ_ERR_UNSUPPORTED;
    if (d->max_pages_per_seq < 1 || d->num_pages < 1) return KVQ_ERR_INVALID_ARG;
    if ((uint64_t)d->num_pages * d->num_kv_heads * (uint64_t)d->page_size >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
    // a sequence's longest length, and every sequence at that length in 128-token tiles
    const uint64_t maxlen = (uint64_t)d->max_pages_per_seq * (uint64_t)d->page_size;
    if (maxlen >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
    if (pairs * ((maxlen + 127) / 128) >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
    if (!d->page_table || !d->seq_lens) return KVQ_ERR_INVALID_ARG;
  }
  if (!d->k_codes || !d->v_codes || !d->k_scale || !d->v_scale || !d->dev_status) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(d->k_codes) || !aligned16(d->v_codes) || !aligned16(d->k_scale) || !aligned16(d->v_scale))
    return KVQ_ERR_INVALID_ARG;
  if ((needs_zp(d->k_scheme) && !d->k_zp) || (needs_zp(d->v_scheme) && !d->v_zp)) return KVQ_ERR_INVALID_ARG;
  (void)needs_scale;
  return KVQ_OK;
}

kvq_status kvq_cache_bytes(const kvq_cache_desc* d, kvq_footprint* out) {
  const kvq_status st = kvq_validate(d);
  if (st != KVQ_OK) return st;
  if (!out) return KVQ_ERR_INVALID_ARG;
  const bool paged = d->layout == KVQ_PAGED;
  const uint64_t rows = paged ? (uint64_t)d->num_pages * d->num_kv_heads * d->page_size
                              : (uint64_t)d->batch * d->num_kv_heads * d->capacity;
  kvq_footprint f;
  std::memset(&f, 0, sizeof(f));
  f.code_bytes = rows * (uint64_t)(row_bytes(d->k_scheme) + row_bytes(d->v_scheme));
  uint64_t meta = 0;
  double per_token_meta = 0.0;
  for (int side = 0; side < 2; ++side) {
    const int s = side ? d->v_scheme : d->k_scheme;
    const uint64_t n = scale_elems(d, side);
    uint64_t bytes = n * (kivi_f16(s) ? 2 : 4);     // fp16 or fp32 elements
    if (is_kivi(s)) bytes *= 2;                       // scale + minimum
    if (needs_zp(s)) bytes += (uint64_t)d->num_kv_heads * d->head_dim;  // uint8 zero points
    meta += bytes;
    if (s == KVQ_INT8_SYM_PER_TOKEN) per_token_meta += 4.0;
    if (s == KVQ_INT4_SYM_PER_GROUP) per_token_meta += 4.0 * d->head_dim / d->group_size;  // fp32 per group
    if (is_kivi(s)) per_token_meta += (kivi_f16(s) ? 4.0 : 8.0) * d->head_dim / 32.0;  // (scale, min) per 32 elements
  }
  f.meta_bytes = meta;
  f.residual_bytes = is_kivi(d->k_scheme)
                         ? 2ull * d->batch * d->num_kv_heads * (uint64_t)d->residual_cap * d->head_dim * 2
                         : 0;
  f.total_bytes = f.code_bytes + f.meta_bytes + f.residual_bytes;
  f.bytes_per_token = (double)(row_bytes(d->k_scheme) + row_bytes(d->v_scheme)) + per_token_meta;
  *out = f;
  return KVQ_OK;
}

size_t kvq_append_workspace_bytes(const kvq_cache_desc* d, uint32_t flags) {
  if (!d || d->num_kv_heads <= 0) return 0;
  const size_t hd = (size_t)d->num_kv_heads * kHeadDim;
  if (flags & KVQ_APPEND_RESCALE) return round_up(rescale_ws_offset(d->num_kv_heads) + 2 * hd * 5 + 16);
  if (flags & KVQ_APPEND_CALIBRATE) return round_up((2 + 4 * hd) * sizeof(uint32_t));
  return 0;
}

kvq_status kvq_quantize_append(kvq_cache_desc* d, const void* k_new, const void* v_new, int32_t in_dtype,
                               int32_t n_new, const int32_t* new_lens, uint32_t flags, void* workspace,
                               size_t workspace_bytes, void* stream) {
  kvq_status st = kvq_validate(d);
  if (st != KVQ_OK) return st;
  if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (n_new < 0 || (flags & ~(KVQ_APPEND_CALIBRATE | KVQ_APPEND_RESCALE))) return KVQ_ERR_INVALID_ARG;
  if ((flags & KVQ_APPEND_CALIBRATE) && (flags & KVQ_APPEND_RESCALE)) return KVQ_ERR_INVALID_ARG;
  if (n_new == 0) return KVQ_OK;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_INVALID_ARG;
  const bool paged = d->layout == KVQ_PAGED;
  if (new_lens && !paged) return KVQ_ERR_INVALID_ARG;
  const bool kivi = is_kivi(d->k_scheme);
  if (kivi && in_dtype != KVQ_BF16) return KVQ_ERR_UNSUPPORTED;
  if (!append_pair_supported(d->k_scheme, d->v_scheme)) return KVQ_ERR_UNSUPPORTED;
  if ((uint64_t)d->batch * d->num_kv_heads * (uint64_t)n_new >= (1ull << 31)) return KVQ_ERR_UNSUPPORTED;
  if (paged && n_new > seq_capacity(d)) return KVQ_ERR_CAPACITY;
  const int mode = kivi                             ? kAppendPlain
                   : (flags & KVQ_APPEND_CALIBRATE) ? kAppendCalibrate
                   : (flags & KVQ_APPEND_RESCALE)   ? kAppendRescale
                                                    : kAppendPlain;
  // the statistics and KIVI flush grids take one block row per (sequence, kv head)
  if ((kivi || mode != kAppendPlain) && (int64_t)d->batch * d->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
  if (mode != kAppendPlain) {
    if (!workspace || workspace_bytes < kvq_append_workspace_bytes(d, flags) || !aligned16(workspace))
      return KVQ_ERR_WORKSPACE;
  }
  int r_old = 0, flushed = 0, r_new = 0;
  if (!paged) {
    if (kivi) {
      r_old = d->num_residual;
      const int total = r_old + n_new;
      r_new = (total - 1) % d->residual_cap + 1;
      flushed = total - r_new;
      if ((int64_t)d->num_quantized + flushed > d->capacity) return KVQ_ERR_CAPACITY;
    } else if ((int64_t)d->num_quantized + n_new > d->capacity) {
      return KVQ_ERR_CAPACITY;
    }
  }
  AppendParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = d->batch;
  p.H = d->num_kv_heads;
  p.n_new = n_new;
  p.k_scheme = d->k_scheme;
  p.v_scheme = d->v_scheme;
  p.in_bf16 = in_dtype == KVQ_BF16;
  p.paged = paged;
  p.cap = d->capacity;
  p.page_size = d->page_size;
  p.max_pages = d->max_pages_per_seq;
  p.num_pages = d->num_pages;
  p.pos0 = d->num_quantized;
  p.rcap = d->residual_cap;
  p.k_new = k_new;
  p.v_new = v_new;
  p.new_lens = new_lens;
  p.k_codes = d->k_codes;
  p.v_codes = d->v_codes;
  p.k_scale = d->k_scale;
  p.k_zero = d->k_zero;
  p.v_scale = d->v_scale;
  p.v_zero = d->v_zero;
  p.k_zp = d->k_zp;
  p.v_zp = d->v_zp;
  p.k_res = d->k_res;
  p.v_res = d->v_res;
  p.page_table = d->page_table;
  p.seq_lens = d->seq_lens;
  p.status = d->dev_status;
  p.rotate = d->rotation == KVQ_ROTATE_HADAMARD;
  p.group = d->group_size;
  const cudaError_t e = launch_append(p, workspace, mode, r_old, flushed, r_new, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return from_cuda(e);
  if (!paged) {
    if (kivi) {
      d->num_quantized += flushed;
      d->num_residual = r_new;
    } else {
      d->num_quantized += n_new;
    }
  }
  return KVQ_OK;
}

kvq_status kvq_dequantize(const kvq_cache_desc* d, int32_t which, float* out, int32_t out_tokens, void* stream) {
  kvq_status st = kvq_validate(d);
  if (st != KVQ_OK) return st;
  if ((which != 0 && which != 1) || !out || out_tokens < 0 || !aligned16(out)) return KVQ_ERR_INVALID_ARG;
  const bool paged = d->layout == KVQ_PAGED;
  if (!paged) {
    const int len = d->num_quantized + (is_kivi(d->k_scheme) ? d->num_residual : 0);
    if (out_tokens < len) return KVQ_ERR_INVALID_ARG;
  }
  DequantParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = d->batch;
  p.H = d->num_kv_heads;
  p.T_out = out_tokens;
  p.which = which;
  p.scheme = which ? d->v_scheme : d->k_scheme;
  p.paged = paged;
  p.cap = d->capacity;
  p.page_size = d->page_size;
  p.max_pages = d->max_pages_per_seq;
  p.num_pages = d->num_pages;
  p.len_q = d->num_quantized;
  p.len_res = d->num_residual;
  p.rcap = d->residual_cap;
  p.codes = static_cast<const uint8_t*>(which ? d->v_codes : d->k_codes);
  p.scale = which ? d->v_scale : d->k_scale;
  p.zero = which ? d->v_zero : d->k_zero;
  p.zp = which ? d->v_zp : d->k_zp;
  p.res = which ? d->v_res : d->k_res;
  p.page_table = d->page_table;
  p.seq_lens = d->seq_lens;
  p.status = d->dev_status;
  p.rotate = d->rotation == KVQ_ROTATE_HADAMARD;
  p.group = d->group_size;
  p.out = out;
  return from_cuda(launch_dequantize(p, static_cast<cudaStream_t>(stream)));
}


size_t kvq_decode_workspace_bytes(const kvq_cache_desc* d) {
  if (!d || d->num_kv_heads < 1 || d->batch < 1 || d->num_q_heads < d->num_kv_heads) return 0;
  const int G = d->num_q_heads / d->num_kv_heads;
  const size_t pairs = (size_t)d->batch * d->num_kv_heads * ((G + 7) / 8);
  const size_t slots = pairs + kMaxCtas;
  return round_up(slots * 8 * kHeadDim * sizeof(float)) + round_up(slots * 8 * 2 * sizeof(float)) +
         round_up((2 * (size_t)d->batch + 2) * sizeof(int32_t));
}

namespace {

// The decode call; early_from >= 0 when the previous launch on the stream is this library's
// plain append writing positions from early_from on (see DecodeParams::early_from); with
// check_only, the argument checks alone.
kvq_status decode_impl(const kvq_cache_desc* d, const void* q, int32_t q_dtype, float softmax_scale, float* out,
                       float* lse, void* workspace, size_t workspace_bytes, void* stream, int early_from,
                       bool check_only) {
  kvq_status st = kvq_validate(d);
  if (st != KVQ_OK) return st;
  if (!q || !out || !aligned16(out) || (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16)) return KVQ_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || softmax_scale <= 0.0f) return KVQ_ERR_INVALID_ARG;
  const size_t need = kvq_decode_workspace_bytes(d);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return KVQ_ERR_WORKSPACE;
  const bool paged = d->layout == KVQ_PAGED;
  const bool rope = d->rope_theta > 0.0f;
  if (!decode_supported(d->k_scheme, d->v_scheme, paged, d->group_size, rope)) return KVQ_ERR_UNSUPPORTED;
  if (check_only) return KVQ_OK;
  const int G = d->num_q_heads / d->num_kv_heads;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = d->batch;
  p.Hq = d->num_q_heads;
  p.Hkv = d->num_kv_heads;
  p.G = G;
  p.HG = (G + 7) / 8;
  p.k_scheme = d->k_scheme;
  p.v_scheme = d->v_scheme;
  p.paged = paged;
  p.cap = d->capacity;
  p.page_size = d->page_size;
  p.max_pages = d->max_pages_per_seq;
  p.num_pages = d->num_pages;
  p.len_q = d->num_quantized;
  p.len_res = is_kivi(d->k_scheme) ? d->num_residual : 0;
  p.rcap = d->residual_cap;
  p.k_codes = static_cast<const uint8_t*>(d->k_codes);
  p.v_codes = static_cast<const uint8_t*>(d->v_codes);
  p.k_scale = d->k_scale;
  p.k_zero = d->k_zero;
  p.v_scale = d->v_scale;
  p.v_zero = d->v_zero;
  p.k_zp = d->k_zp;
  p.v_zp = d->v_zp;
  p.k_res = d->k_res;
  p.v_res = d->v_res;
  p.page_table = d->page_table;
  p.seq_lens = d->seq_lens;
  p.status = d->dev_status;
  p.rotate = d->rotation == KVQ_ROTATE_HADAMARD;
  p.group = d->group_size;
  p.rope_theta = d->rope_theta;
  p.q = q;
  p.q_bf16 = q_dtype == KVQ_BF16;
  p.softmax_scale = softmax_scale;
  p.out = out;
  p.lse = lse;
  p.n_pairs = d->batch * d->num_kv_heads * p.HG;
  const size_t slots = (size_t)p.n_pairs + kMaxCtas;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.part_o = reinterpret_cast<float*>(ws);
  ws += round_up(slots * 8 * kHeadDim * sizeof(float));
  p.part_ml = reinterpret_cast<float*>(ws);
  ws += round_up(slots * 8 * 2 * sizeof(float));
  p.plan = reinterpret_cast<int32_t*>(ws);
  p.early_from = early_from;
  return from_cuda(launch_decode(p, static_cast<cudaStream_t>(stream)));
}

}  // namespace

kvq_status kvq_decode_attention(const kvq_cache_desc* d, const void* q, int32_t q_dtype, float softmax_scale,
                                float* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(d, q, q_dtype, softmax_scale, out, lse, workspace, workspace_bytes, stream, -1, false);
}

kvq_status kvq_append_decode(kvq_cache_desc* d, const void* k_new, const void* v_new, int32_t in_dtype,
                             int32_t n_new, const void* q, int32_t q_dtype, float softmax_scale, float* out,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  // every check of both calls before anything is launched
  kvq_status st = decode_impl(d, q, q_dtype, softmax_scale, out, lse, workspace, workspace_bytes, stream, -1, true);
  if (st != KVQ_OK) return st;
  if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (n_new < 0) return KVQ_ERR_INVALID_ARG;
  const bool kivi = is_kivi(d->k_scheme);
  if (n_new > 0) {
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_INVALID_ARG;
    if (!append_pair_supported(d->k_scheme, d->v_scheme) || (kivi && in_dtype != KVQ_BF16)) return KVQ_ERR_UNSUPPORTED;
    if (d->layout == KVQ_PAGED) {
      if (n_new > seq_capacity(d)) return KVQ_ERR_CAPACITY;
    } else if (kivi) {
      const int total = d->num_residual + n_new;
      const int flushed = total - ((total - 1) % d->residual_cap + 1);
      if ((int64_t)d->num_quantized + flushed > d->capacity) return KVQ_ERR_CAPACITY;
    } else if ((int64_t)d->num_quantized + n_new > d->capacity) {
      return KVQ_ERR_CAPACITY;
    }
  }
  // the decode overlaps the append when the append is one launch of the 8-bit / INT4 rows kernel
  // on a dense cache (it then writes the new positions and nothing else the decode reads)
  const bool overlap = n_new > 0 && d->layout == KVQ_DENSE && !kivi;
  const int pos0 = d->num_quantized;
  st = kvq_quantize_append(d, k_new, v_new, in_dtype, n_new, nullptr, 0u, nullptr, 0, stream);
  if (st != KVQ_OK) return st;
  return decode_impl(d, q, q_dtype, softmax_scale, out, lse, workspace, workspace_bytes, stream,
                     overlap ? pos0 : -1, false);
}

kvq_status kvq_check_bounded_wait(uint32_t* dev_status, void* stream) {
  if (!dev_status || (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0) return KVQ_ERR_INVALID_ARG;
  bounded_wait_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status);
  count_launches(1);
  return from_cuda(cudaGetLastError());
}

kvq_status kvq_get_device_status(const kvq_cache_desc* d, uint32_t* out, int32_t clear, void* stream) {
  if (!d || !d->dev_status || !out) return KVQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(out, d->dev_status, 2 * sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(d->dev_status, 0, 2 * sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  return from_cuda(e);
}

}  // extern "C"

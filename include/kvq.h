/*
 * libkvq: KV-cache quantize-on-append and decode attention over the quantized cache,
 * for NVIDIA B200 (sm_100a). C ABI; every pointer named "device" is CUDA device memory
 * owned by the caller. The library allocates nothing.
 *
 * Problem statement ("How KV cache quantization reduces GPU memory", n4n.ai, Step 1):
 * the cache holds K and V per layer, each [batch, num_heads, seq_len, head_dim]; here
 * num_heads are the KV heads and one descriptor describes one layer.
 *
 * Conventions for every entry point:
 *  - Asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy default).
 *  - Argument errors return synchronously, before any launch, and change nothing.
 *  - A launch failure returns KVQ_ERR_CUDA.
 *  - Faults the device detects (a page id outside the pool, a length outside the page
 *    table, a wait that ran out of time) set bits in the device status word
 *    (desc->dev_status[0]); the kernel skips the affected work and never traps. Read the
 *    word with kvq_get_device_status.
 *  - Codes, scales and zero points are bit-exact functions of the inputs (IEEE fp32
 *    division, round-half-to-even); attention outputs are fp32.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_ABI_VERSION 3

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, bad enum value */
  KVQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (scheme pair, dtype, head_dim) */
  KVQ_ERR_CAPACITY = 3,      /* the append does not fit the dense capacity */
  KVQ_ERR_WORKSPACE = 4,     /* workspace null or smaller than the query says */
  KVQ_ERR_CUDA = 5           /* a CUDA call or launch failed */
} kvq_status;

/* Quantization schemes, chosen separately for K and for V.
 *  FP8_E4M3_PER_TENSOR  OCP E4M3 codes of x/s, s = absmax/448 over the calibrating append
 *                       ("KV Cache Quantization", infra.bea.ai, §4; llms.blog §1).
 *  INT8_SYM_PER_TENSOR  clamp(rne(x/s), -127, 127), s = absmax/127 over the calibrating
 *                       append (n4n.ai Step 2-3; llms.blog §2).
 *  INT8_SYM_PER_TOKEN   same, one s per (batch, kv_head, token) row (llms.blog §2).
 *  INT8_SYM_PER_CHANNEL same, one s per (kv_head, channel) (infra.bea.ai §3 Key example).
 *  UINT8_ASYM_PER_CHANNEL  clamp(rne(x/s) + zp, 0, 255), s = (max(mx,0) - min(mn,0))/255,
 *                       zp = clamp(rne(-min(mn,0)/s), 0, 255) per (kv_head, channel)
 *                       (n4n.ai Step 2 "per-channel asymmetric INT8").
 *  KIVI_INT4 / KIVI_INT2  KIVI (infra.bea.ai §3, llms.blog §3): keys per channel over
 *                       groups of 32 tokens, values per token over groups of 32 channels,
 *                       s = (max - min)/(2^bits - 1), q = clamp(rne((x - min)/s)), fp32
 *                       scale and minimum, codes packed along head_dim (lower channel in
 *                       lower bits), recent tokens in a bf16 residual of 128 tokens.
 *  FP8_E5M2_PER_TENSOR  OCP E5M2 codes of x/s, s = absmax/57344 over the calibrating append,
 *                       saturating at +-57344 (llms.blog §1 compares E4M3 with E5M2; a format
 *                       variant beyond the configurations the pages measure).
 *  INT4_SYM_PER_GROUP   clamp(rne(x/s), -8, 7) with s = absmax/7 per group of group_size (32,
 *                       64 or 128) consecutive channels of one token (llms.blog §2 "INT4
 *                       Group-Wise"; n4n.ai Step 2 "Per-group INT4"); two's-complement nibbles
 *                       packed along head_dim, lower channel in the low bits (64-byte rows);
 *                       fp32 scales [rows][head_dim / group_size]. K and V both.
 *  KIVI_INT4_F16 / KIVI_INT2_F16  KIVI with the scale and minimum of every group stored as IEEE
 *                       fp16 (the precision of the tensors n4n.ai Step 3's cache code works
 *                       in; half the metadata bytes, so INT2 takes 3 bits per element): the fp32
 *                       s and min of a group rounded to nearest-even fp16, saturating at +-65504,
 *                       and the codes taken from the stored values, q = clamp(rne((x - min16) /
 *                       s16), 0, 2^bits - 1); s16 == 0 gives code 0. The scale and minimum
 *                       arrays (k_scale, k_zero, v_scale, v_zero) then hold fp16 elements.
 * A zero range gives s = 0 and code 0. */
typedef enum kvq_scheme {
  KVQ_FP8_E4M3_PER_TENSOR = 0,
  KVQ_INT8_SYM_PER_TENSOR = 1,
  KVQ_INT8_SYM_PER_TOKEN = 2,
  KVQ_INT8_SYM_PER_CHANNEL = 3,
  KVQ_UINT8_ASYM_PER_CHANNEL = 4,
  KVQ_KIVI_INT4 = 5,
  KVQ_KIVI_INT2 = 6,
  KVQ_FP8_E5M2_PER_TENSOR = 7,
  KVQ_INT4_SYM_PER_GROUP = 8,
  KVQ_KIVI_INT4_F16 = 9,
  KVQ_KIVI_INT2_F16 = 10
} kvq_scheme;

typedef enum kvq_dtype { KVQ_F32 = 0, KVQ_BF16 = 1 } kvq_dtype;
typedef enum kvq_layout { KVQ_DENSE = 0, KVQ_PAGED = 1 } kvq_layout;

/* Online rotation of K, V and Q ("KV Cache Quantization in Production LLM Serving",
 * llms.blog §5, QuaRot / RotateKV): the normalised Walsh-Hadamard transform H/sqrt(128) over
 * head_dim, orthogonal and symmetric, so (H q).(H k) = q.k and H (sum p H v) = sum p v. Rows
 * are transformed in fp32 by butterflies of span 1, 2, ..., 64 and a final multiply by the
 * fp32 value of 1/sqrt(128). */
typedef enum kvq_rotation { KVQ_ROTATE_NONE = 0, KVQ_ROTATE_HADAMARD = 1 } kvq_rotation;

/* kvq_quantize_append flags */
#define KVQ_APPEND_CALIBRATE 0x1u  /* recompute per-tensor / per-channel scales from this block */
#define KVQ_APPEND_RESCALE 0x2u    /* merge this block's scales into the cached ones, requantize */

/* device status word bits (dev_status[0]); dev_status[1] counts saturated codes */
#define KVQ_DEV_BAD_PAGE 0x1u
#define KVQ_DEV_BAD_LENGTH 0x2u
#define KVQ_DEV_TIMEOUT 0x4u

/*
 * One layer's cache. Shapes (all device memory, contiguous, caller-owned):
 *   row_bytes(scheme) = head_dim (8-bit), head_dim/2 (KIVI_INT4), head_dim/4 (KIVI_INT2)
 *   dense codes  [batch, kv_heads, capacity, row_bytes]
 *   paged codes  [num_pages, kv_heads, page_size, row_bytes]
 *   per-tensor scale            float [1]
 *   per-token scale             float [batch, kv_heads, capacity]  (paged: [num_pages, kv_heads, page_size])
 *   INT4 per-group scale        float [batch, kv_heads, capacity, head_dim/group_size] (paged:
 *                               [num_pages, kv_heads, page_size, head_dim/group_size])
 *   per-channel scale           float [kv_heads, head_dim]; uint8 zero point (k_zp/v_zp) same shape
 *   KIVI key scale and minimum  float [batch, kv_heads, capacity/32, head_dim] (k_scale, k_zero)
 *   KIVI value scale and minimum float [batch, kv_heads, capacity, head_dim/32] (v_scale, v_zero)
 *                               (fp16 elements, same shapes, for KIVI_INT4_F16 / KIVI_INT2_F16)
 *   KIVI residual               bf16  [batch, kv_heads, residual_cap, head_dim] (k_res, v_res)
 *   paged page_table            int32 [batch, max_pages_per_seq]; seq_lens int32 [batch]
 *   dev_status                  uint32 [2]
 * Unused pointers may be NULL.
 */
typedef struct kvq_cache_desc {
  int32_t batch, num_q_heads, num_kv_heads, head_dim;  /* head_dim must be 128 */
  int32_t k_scheme, v_scheme;                          /* kvq_scheme */
  int32_t layout;                                      /* kvq_layout */
  int32_t capacity;          /* dense: tokens per (batch, kv_head); multiple of 128 */
  int32_t page_size;         /* paged: 16, 32 or 64 tokens */
  int32_t max_pages_per_seq, num_pages;
  int32_t group_size;        /* KIVI: 32; INT4 per group: 32, 64 or 128 */
  int32_t residual_cap;      /* KIVI: 128 */
  int32_t num_quantized;     /* dense: quantized tokens per row (library-maintained) */
  int32_t num_residual;      /* KIVI: tokens in the bf16 residual (library-maintained) */
  void* k_codes;
  void* v_codes;
  float* k_scale;
  float* k_zero;
  float* v_scale;
  float* v_zero;
  uint8_t* k_zp;
  uint8_t* v_zp;
  uint16_t* k_res;
  uint16_t* v_res;
  int32_t* page_table;
  int32_t* seq_lens;
  uint32_t* dev_status;
  int32_t rotation;          /* kvq_rotation: KVQ_ROTATE_HADAMARD rotates every K/V row before it
                                is quantized, each query before attention and each output and
                                dequantized row back (not with KIVI schemes) */
  float rope_theta;          /* 0: keys are cached as given (after RoPE). > 0: keys are cached
                                before RoPE (KVQuant's pre-RoPE key quantization, "KV Cache
                                Quantization in Production LLM Serving", llms.blog §4) and decode
                                rotates each dequantized key at its position t in the sequence
                                (0-based): pairs (i, i + 64), angle t * rope_theta^(-2i/128),
                                (a, b) -> (a cos - b sin, b cos + a sin); queries arrive rotated.
                                8-bit key schemes, not with KVQ_ROTATE_HADAMARD. Dequantize returns
                                the stored (pre-RoPE) keys. */
} kvq_cache_desc;

typedef struct kvq_footprint {
  uint64_t code_bytes;       /* K and V codes at capacity */
  uint64_t meta_bytes;       /* scales, minima and zero points */
  uint64_t residual_bytes;   /* KIVI bf16 residual */
  uint64_t total_bytes;
  double bytes_per_token;    /* codes + per-token share of metadata + residual, per kv_head row pair */
} kvq_footprint;

KVQ_API int kvq_abi_version(void);
KVQ_API const char* kvq_status_string(kvq_status s);

/* Check a descriptor's fields (shapes, enums, pointer presence). No device access. */
KVQ_API kvq_status kvq_validate(const kvq_cache_desc* desc);

/* Bytes the cache arrays take (n4n.ai Step 6 "peak memory"; llms.blog memory-per-token). */
KVQ_API kvq_status kvq_cache_bytes(const kvq_cache_desc* desc, kvq_footprint* out);

/* Workspace kvq_quantize_append needs for `flags` (0 unless KVQ_APPEND_CALIBRATE or
 * KVQ_APPEND_RESCALE). */
KVQ_API size_t kvq_append_workspace_bytes(const kvq_cache_desc* desc, uint32_t flags);

/*
 * Quantize n_new tokens per sequence and append them ("QuantizedKVCache.append",
 * n4n.ai Step 3; KIVI residual policy, infra.bea.ai §3 "Residual Cache for Streaming").
 *   k_new, v_new  device [batch, kv_heads, n_new, head_dim], in_dtype (KIVI: bf16 only)
 *   new_lens      paged only, device int32 [batch] or NULL: per-sequence counts <= n_new
 *   flags         KVQ_APPEND_CALIBRATE: per-tensor / per-channel scales from this block
 *                 (otherwise the scales already in the descriptor are used; values beyond
 *                 them saturate and are counted in dev_status[1]).
 *                 KVQ_APPEND_RESCALE (not with CALIBRATE): the scales grow to cover this
 *                 block and the cached codes whose scale changed are requantized first
 *                 (n4n.ai Step 3 keeps a running maximum of the scales; Step 7 recomputes
 *                 them as the cache grows, e.g. every 1024 tokens). Symmetric schemes take
 *                 max(cached, block) per scale element; uint8 asymmetric takes the union
 *                 of the cached representable range [(0 - zp) s, (255 - zp) s] and the
 *                 block's range. A cached code is requantized from its dequantized value.
 *                 Both flags are ignored for per-token and KIVI schemes.
 *                 Calibrating, rescaling and KIVI appends need batch * kv_heads <= 65535
 *                 (else KVQ_ERR_UNSUPPORTED, before anything is launched).
 * Dense: tokens go to positions num_quantized.. of every row; the library updates
 * num_quantized / num_residual in *desc when the call is accepted. KIVI: tokens enter the
 * residual; when a token arrives at a full residual, its 128 tokens are quantized.
 * Paged: token i of sequence b goes to position seq_lens[b] + i, page
 * page_table[b][pos / page_size], slot pos % page_size; seq_lens is advanced on the device.
 * The caller assigns page_table entries before the call.
 */
KVQ_API kvq_status kvq_quantize_append(kvq_cache_desc* desc, const void* k_new, const void* v_new,
                               int32_t in_dtype, int32_t n_new, const int32_t* new_lens,
                               uint32_t flags, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Dequantize K (which = 0) or V (which = 1) into device fp32 out [batch, kv_heads,
 * out_tokens, head_dim] ("QuantizedKVCache.dequantize / get", n4n.ai Step 3). Token
 * order: quantized tokens, then the KIVI residual. Rows at or past a sequence's length
 * are written as zero. out_tokens must be >= every sequence's length.
 */
KVQ_API kvq_status kvq_dequantize(const kvq_cache_desc* desc, int32_t which, float* out,
                          int32_t out_tokens, void* stream);

/* Workspace kvq_decode_attention needs (split partials and the paged plan). */
KVQ_API size_t kvq_decode_workspace_bytes(const kvq_cache_desc* desc);

/*
 * Decode attention of one query token per sequence over the quantized cache, reading the
 * codes directly (llms.blog, section "Serving Economics and Latency Trade-Offs": decode is bound by
 * memory bandwidth; guide.dupenodi.dev "KV cache quantization": the savings only count
 * when the attention kernel consumes the low-precision cache itself).
 *   q         device [batch, num_q_heads, head_dim], q_dtype (bf16 or fp32)
 *   out       device fp32 [batch, num_q_heads, head_dim], 16-byte aligned (else
 *             KVQ_ERR_INVALID_ARG, returned before anything is launched)
 *   lse       device fp32 [batch, num_q_heads] or NULL: natural-log sum of exp of scores
 * Query head h reads kv head h / (num_q_heads / num_kv_heads). Scores are
 * softmax_scale * q.k over all tokens of the sequence (no mask). A sequence with no
 * tokens gives zeros and lse = -inf.
 */
KVQ_API kvq_status kvq_decode_attention(const kvq_cache_desc* desc, const void* q, int32_t q_dtype,
                                float softmax_scale, float* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * One decode step in one call: kvq_quantize_append(desc, k_new, v_new, in_dtype, n_new,
 * NULL, 0, ...) (a plain append: the cache's scales as they are), then
 * kvq_decode_attention(desc, q, ...) over the updated cache, on `stream`, with the same
 * arguments, layouts, results and errors as those two calls. Every check of both runs before
 * anything is launched. "KV Cache Quantization" (infra.bea.ai), §4 FP8 KV cache: the cache is
 * appended to and read back at every decode step; this call overlaps the two.
 *   workspace  decode workspace (kvq_decode_workspace_bytes; a plain append needs none)
 * On a dense cache with 8-bit or INT4-per-group schemes (not KIVI) the decode kernel is
 * launched as the programmatic dependent of the append and reads the cached tiles that hold
 * no new position while the append runs; it waits for the append before the tiles that do.
 * Otherwise the two run one after the other. Not for a cache whose scales must grow with the
 * block (KVQ_APPEND_RESCALE) or be calibrated from it: call the two entry points.
 */
KVQ_API kvq_status kvq_append_decode(kvq_cache_desc* desc, const void* k_new, const void* v_new, int32_t in_dtype,
                                     int32_t n_new, const void* q, int32_t q_dtype, float softmax_scale,
                                     float* out, float* lse, void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * Test support; the pages have no counterpart. Launches one warp that waits on a
 * shared-memory barrier nothing ever arrives at, through the same bounded wait every kernel
 * of the library uses for its copy barriers. After about one second the wait gives up, sets
 * KVQ_DEV_TIMEOUT in dev_status[0] and the kernel returns, leaving the context usable. This
 * lets a test exercise the timeout path on a GPU without hanging or faulting it.
 *   dev_status  device uint32[2] (caller-owned; only bits are ORed in)
 * Asynchronous on `stream`; KVQ_ERR_INVALID_ARG for a null or misaligned pointer.
 */
KVQ_API kvq_status kvq_check_bounded_wait(uint32_t* dev_status, void* stream);

/* Number of kernels this process has launched through the library (all entry points). */
KVQ_API uint64_t kvq_launch_count(void);

/*
 * Decode attention that allocates nothing and takes no workspace. The paper has no
 * counterpart; this exists for callers that cannot call cudaMalloc: an inference-engine
 * plugin handed only its input and output buffers, code running while a CUDA graph is
 * being captured (a new allocation is not allowed there), or a serving loop that forbids
 * allocation after start-up so it never synchronises the device or fragments its pool.
 *
 * The split partials live in a static device array of KVQ_NOALLOC_SCRATCH_BYTES that
 * every GPU which loads the library holds until the process exits. A cache whose
 * kvq_decode_workspace_bytes exceeds that size is rejected with KVQ_ERR_WORKSPACE
 * before any launch. The first call on a device looks up the array's device address
 * (with that device current), so make the first call on each device before any stream
 * capture. The address is kept per device and CUDA context: a call from another context on
 * the same device (a caller's own driver context, or the new primary context after a device
 * reset) looks it up again. Every call shares the one array: calls that overlap on the GPU (different
 * streams, or devices sharing a context) race, so serialise them. The array keeps the
 * previous call's contents; nothing in it needs to start at zero. Arguments and results
 * are those of kvq_decode_attention.
 */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)
KVQ_API kvq_status kvq_decode_attention_noalloc(const kvq_cache_desc* desc, const void* q, int32_t q_dtype,
                                                float softmax_scale, float* out, float* lse, void* stream);

/* Copy dev_status[0..1] to host out[2] (synchronises `stream`); clear != 0 zeroes them. */
KVQ_API kvq_status kvq_get_device_status(const kvq_cache_desc* desc, uint32_t* out, int32_t clear,
                                 void* stream);

#ifdef __cplusplus
}
#endif
#endif

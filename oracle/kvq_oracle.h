/*
 * KV-cache quantization oracle: TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU statement of what the quantize-on-append and
 * decode-attention path computes. Quantization is strict IEEE fp32 (one correctly
 * rounded operation per step, no FMA contraction, round-half-to-even); attention is
 * fp64. It shares no code, header, table or constant with the CUDA library. Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may call it; the
 * product path never does.
 *
 * Sources (web pages, by title and section):
 *  [P1] "KV Cache Quantization" (infra.bea.ai guide): §1 memory table, §3 KIVI
 *       (Key per-channel, Value per-token, residual cache), §4 FP8 KV cache.
 *  [P3] "KV Cache Quantization in Production LLM Serving: Comparing FP8, INT8, INT4,
 *       KIVI, and KVQuant" (llms.blog): memory-per-token formula, §1 FP8 E4M3 (and
 *       E5M2, the other OCP FP8 format the section compares it with), §2 INT8 symmetric
 *       [-127,127] and INT4 group-wise, §3 KIVI, §4 KVQuant (pre-RoPE keys), §5 QuaRot /
 *       RotateKV (Hadamard rotation).
 *  [P4] "How KV cache quantization reduces GPU memory" (n4n.ai): Step 1 tensor shape,
 *       Step 2 schemes (per-group INT4), Step 3 QuantizedKVCache (quantize / dequantize /
 *       append, running-max scale merge), Step 7 edge cases (scales that grow or are
 *       recomputed as the cache grows).
 *
 * Parity status: every function here is pinned by a CPU test (worked examples,
 * closed forms, invariants, brute force). End-to-end model quality (perplexity,
 * logit parity on a model) is NOT computed here: parity unpinned for that, since it
 * needs model weights and datasets.
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Scheme numbers (same integers as every harness uses). */
enum {
  OQ_FP8_E4M3_PER_TENSOR = 0,
  OQ_INT8_SYM_PER_TENSOR = 1,
  OQ_INT8_SYM_PER_TOKEN = 2,
  OQ_INT8_SYM_PER_CHANNEL = 3,
  OQ_UINT8_ASYM_PER_CHANNEL = 4,
  OQ_KIVI_INT4 = 5,
  OQ_KIVI_INT2 = 6,
  OQ_FP8_E5M2_PER_TENSOR = 7,
  OQ_INT4_SYM_PER_GROUP = 8,
  OQ_KIVI_INT4_F16 = 9,  /* KIVI with fp16 scale and minimum */
  OQ_KIVI_INT2_F16 = 10
};

/* ---- element codecs ---- */
float oq_bf16_to_f32(uint16_t h);
uint16_t oq_f32_to_bf16(float f);
uint8_t oq_e4m3_encode(float x);            /* round-to-nearest-even, saturate finite */
float oq_e4m3_decode(uint8_t code);
uint8_t oq_e5m2_encode(float x);            /* round-to-nearest-even, saturate finite */
float oq_e5m2_decode(uint8_t code);
int oq_sym_code(float x, float s, int qmax); /* clamp(rne(x/s), -qmax, qmax); 0 if s == 0 */
int oq_int4_code(float x, float s);         /* clamp(rne(x/s), -8, 7); 0 if s == 0 */
uint16_t oq_f16_encode(float x);            /* IEEE half, RN-even, saturating at +-65504 */
float oq_f16_decode(uint16_t h);
/* KIVI group with fp16 parameters: s and min in fp32, stored rounded to fp16, codes from
 * the stored values; *s and *mn receive the stored (fp16) values. */
void oq_kivi_group_f16(const float* x, int n, int stride, int bits, int* codes, float* s, float* mn);
void oq_asym_params(float mn, float mx, float* s, uint8_t* zp);
int oq_asym_code(float x, float s, uint8_t zp);
void oq_kivi_group(const float* x, int n, int stride, int bits, int* codes, float* s, float* mn);
float oq_kivi_value(int code, float s, float mn);

/* ---- cache state (mirrors the library's layouts; all arrays caller-owned) ---- */
typedef struct {
  int B, Hq, Hkv, D;
  int k_scheme, v_scheme;
  int paged;                     /* 0: [B,Hkv,cap,bytes]; 1: [P,Hkv,page,bytes] */
  int cap;                       /* dense capacity in tokens */
  int page_size, max_pages, num_pages;
  int group, rcap;               /* KIVI group (32) and residual capacity (128) */
  int len, res;                  /* dense: quantized tokens and residual tokens */
  uint8_t *k_codes, *v_codes;
  float *k_scale, *k_zero, *v_scale, *v_zero;
  uint8_t *k_zp, *v_zp;
  uint16_t *k_res, *v_res;       /* bf16 [B,Hkv,rcap,D] */
  int32_t *page_table, *seq_lens;
  int rotate;                    /* 1: K/V rows and queries rotated by the normalised
                                    Walsh-Hadamard transform over head_dim (not with KIVI) */
  float rope_theta;              /* > 0: keys are cached before RoPE and decode rotates each
                                    dequantized key at its position (KVQuant pre-RoPE keys) */
} oq_cache;

/* Append modes (the `calibrate` argument of oq_append). */
enum { OQ_APPEND_PLAIN = 0, OQ_APPEND_CALIBRATE = 1, OQ_APPEND_RESCALE = 2 };

/* Append n_new tokens per sequence (new_lens: per-sequence counts, paged only).
 * k_new/v_new are [B,Hkv,n_new,D], bf16 bits when in_bf16 else fp32.
 * calibrate: OQ_APPEND_CALIBRATE recomputes per-tensor / per-channel scales from these
 * tokens; OQ_APPEND_RESCALE merges the block's scales into the cached ones (they only
 * grow) and requantizes the cached codes whose scale changed, before the block is
 * quantized. KIVI and per-token schemes ignore both.
 * Returns 0, or -1 on a capacity / argument error. */
int oq_append(oq_cache* c, const void* k_new, const void* v_new, int in_bf16, int n_new,
              const int32_t* new_lens, int calibrate);

/* Only the calibration of oq_append: recompute the per-tensor / per-channel scales of the
 * cache from the block (same arguments), quantize nothing. */
int oq_calibrate(oq_cache* c, const void* k_new, const void* v_new, int in_bf16, int n_new,
                 const int32_t* new_lens);

/* In-place normalised Walsh-Hadamard transform of n (a power of two) values: butterfly
 * stages of span 1, 2, 4, ..., n/2, each (a, b) -> (a + b, a - b) in fp32, then every value
 * times the fp32 constant nearest 1/sqrt(n). The transform is its own inverse. */
void oq_fwht(float* x, int n);

/* Rotate-half RoPE of one row in fp64 at position pos: for i < D/2, with inverse
 * frequency theta^(-2i/D) and angle pos * that, (x_i, x_{i+D/2}) becomes
 * (x_i cos - x_{i+D/2} sin, x_{i+D/2} cos + x_i sin). */
void oq_rope(double* x, int D, int pos, double theta);

/* Tokens visible to decode for sequence b. */
int oq_tokens(const oq_cache* c, int b);

/* Dequantized K (which = 0) or V (which = 1) as fp32 [B,Hkv,T_out,D]; rows past a
 * sequence's length are zero. */
void oq_dequantize(const oq_cache* c, int which, float* out, int T_out);

/* fp64 softmax attention of one query row over T dequantized tokens.
 * q [D] fp32, k,v [T,D] fp32; out [D]; returns lse (natural log) via *lse. */
void oq_attention_row(const float* q, const float* k, const float* v, int T, int D,
                      float scale, double* out, double* lse);

/* Decode attention over the whole cache: q [B,Hq,D] (bf16 bits or fp32),
 * out [B,Hq,D] fp64, lse [B,Hq] fp64 (may be NULL). Head h reads kv head h/(Hq/Hkv). */
void oq_decode(const oq_cache* c, const void* q, int q_bf16, float scale, double* out,
               double* lse);

/* Same, for a subset of (b, kv_head) pairs: pairs [n_pairs][2]; out [n_pairs,G,D]. */
void oq_decode_pairs(const oq_cache* c, const void* q, int q_bf16, float scale,
                     const int32_t* pairs, int n_pairs, double* out, double* lse);

/* Bytes of one token across layers: 2 (K and V) * bytes/elem * layers * kv_heads * d_head. */
double oq_kv_bytes_per_token(int n_layers, int n_kv_heads, int d_head, double bytes_per_elem);

#ifdef __cplusplus
}
#endif
#endif

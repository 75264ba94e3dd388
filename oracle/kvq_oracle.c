/*
 * KV-cache quantization oracle (TEST INFRASTRUCTURE ONLY; see kvq_oracle.h).
 *
 * Build flags: -O2 -ffp-contract=off -fno-fast-math on x86-64 (SSE arithmetic), so
 * every float expression below is one correctly rounded IEEE operation and rintf()
 * rounds half to even.
 *
 * Readings of the pages that this file fixes (each is listed with its reason in the
 * design notes of the repository):
 *  - scale = absmax / qmax by fp32 division; code = clamp(rne(x / scale)).
 *  - symmetric INT8 clamps to [-127, 127] (P3 §2), not the [-128, 127] of P4 Step 3.
 *  - a zero range gives scale 0 and code 0.
 *  - asymmetric uint8 uses the affine form q = rne(x/s) + zp over a range widened to
 *    contain 0; P4 Step 3 quantizes (x - min)/s but dequantizes (q - zp)*s.
 *  - KIVI keeps the fp32 group minimum as its zero point, dequant fl(fl(q*s) + mn).
 *  - per-tensor and per-channel scales are fixed by the calibrating append.
 *  - KIVI residual: 128 tokens, groups of 32, flush when a token arrives at a full
 *    residual.
 *  - INT4 symmetric per group: groups of 32 consecutive channels of a token, s = absmax / 7,
 *    q = clamp(rne(x / s), -8, 7), two's-complement nibbles, lower channel in the low bits.
 *  - rotation (optional): the normalised Walsh-Hadamard transform of each K/V row before it
 *    is quantized, of each query before attention, and of each attention output and
 *    dequantized row after (P3 §5, QuaRot / RotateKV); fp32 butterflies in span order.
 *  - pre-RoPE keys (optional, P3 §4 KVQuant): keys are quantized as given (before RoPE)
 *    and decode applies rotate-half RoPE in fp64 to each dequantized key at its position
 *    in the sequence; queries arrive with RoPE applied.
 */
#include "kvq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* element codecs                                                            */
/* ------------------------------------------------------------------------- */

/* Normalised Walsh-Hadamard transform (Sylvester order): H_n with entries
 * (-1)^popcount(i & j), scaled by 1/sqrt(n) so that it is orthogonal and symmetric, hence
 * its own inverse; rotating q and k alike keeps q.k (P3 §5 "QuaRot / RotateKV"). */
void oq_fwht(float* x, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int i = 0; i < n; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        const float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
  const float c = (float)(1.0 / sqrt((double)n));
  for (int i = 0; i < n; ++i) x[i] = x[i] * c;
}

static void fwht_d(double* x, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int i = 0; i < n; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        const double a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
  const double c = 1.0 / sqrt((double)n);
  for (int i = 0; i < n; ++i) x[i] *= c;
}

float oq_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

uint16_t oq_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* OCP 8-bit floating point E4M3 (P3 §1 names it: sign, 4 exponent and 3 mantissa
 * bits): exponent bias 7, no infinities, S.1111.111 is NaN, largest finite
 * value 1.75 * 2^8 = 448, subnormals M/8 * 2^-6. */
float oq_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  float v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexpf((float)m, -9);            /* (m/8) * 2^-6 */
  else
    v = ldexpf((float)(8 + m), e - 10);  /* (1 + m/8) * 2^(e-7) */
  return s ? -v : v;
}

/* Nearest E4M3 value, ties to even mantissa; finite values above 448 saturate to 448
 * (the "satfinite" behaviour FP8 KV caches use). The sign of zero is kept. */
uint8_t oq_e4m3_encode(float x) {
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const float a = fabsf(x);
  if (isnan(x)) return (uint8_t)(sign | 0x7F);
  if (a > 448.0f) return (uint8_t)(sign | 0x7E);
  if (a < ldexpf(1.0f, -6)) {
    /* subnormal grid: multiples of 2^-9; 8 * 2^-9 is the smallest normal (code 0x08) */
    float m = rintf(ldexpf(a, 9));
    return (uint8_t)(sign | (uint8_t)m);
  }
  int e2;
  frexpf(a, &e2);            /* a in [2^(e2-1), 2^e2) */
  int E = e2 - 1;            /* unbiased exponent, -6..8 */
  float m = rintf(ldexpf(a, 3 - E)); /* significand * 8, in [8, 16] */
  if (m == 16.0f) {
    m = 8.0f;
    E += 1;
  }
  if (E > 8 || (E == 8 && m > 14.0f)) return (uint8_t)(sign | 0x7E);
  return (uint8_t)(sign | (uint8_t)(((E + 7) << 3) | ((int)m - 8)));
}

/* OCP FP8 E5M2: sign, 5 exponent bits (bias 15), 2 mantissa bits; exponent 31 holds infinity
 * and NaN; largest finite value 1.75 * 2^15 = 57344; subnormals M/4 * 2^-14. */
float oq_e5m2_decode(uint8_t code) {
  const int s = code >> 7, E = (code >> 2) & 0x1F, M = code & 3;
  float v;
  if (E == 31)
    v = M == 0 ? INFINITY : NAN;
  else if (E == 0)
    v = ldexpf((float)M, -16);
  else
    v = ldexpf(1.0f + (float)M / 4.0f, E - 15);
  return s ? -v : v;
}

/* Nearest E5M2 value, ties to even mantissa; finite values above 57344 saturate to 57344
 * (as for E4M3). The sign of zero is kept. */
uint8_t oq_e5m2_encode(float x) {
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const float a = fabsf(x);
  if (isnan(x)) return (uint8_t)(sign | 0x7F);
  if (a > 57344.0f) return (uint8_t)(sign | 0x7B);
  if (a < ldexpf(1.0f, -14)) {
    /* subnormal grid: multiples of 2^-16; 4 * 2^-16 is the smallest normal (code 0x04) */
    float m = rintf(ldexpf(a, 16));
    return (uint8_t)(sign | (uint8_t)m);
  }
  int e2;
  frexpf(a, &e2);            /* a in [2^(e2-1), 2^e2) */
  int E = e2 - 1;            /* unbiased exponent, -14..15 */
  float m = rintf(ldexpf(a, 2 - E)); /* significand * 4, in [4, 8] */
  if (m == 8.0f) {
    m = 4.0f;
    E += 1;
  }
  if (E > 15 || (E == 15 && m > 7.0f)) return (uint8_t)(sign | 0x7B);
  return (uint8_t)(sign | (uint8_t)(((E + 15) << 2) | ((int)m - 4)));
}

/* Symmetric code: clamp(rne(x / s), -qmax, qmax) (P4 Step 3 divides by the scale and
 * rounds; P3 §2 gives the symmetric INT8 range as -127..127). */
int oq_sym_code(float x, float s, int qmax) {
  if (s == 0.0f) return 0;
  float y = x / s;
  float r = rintf(y);
  if (r > (float)qmax) r = (float)qmax;
  if (r < (float)-qmax) r = (float)-qmax;
  return (int)r;
}

/* INT4 group code (P3 §2 "INT4 Group-Wise"; the page code of P4 Step 3 divides by
 * max|x| / 7 and clamps to the signed 4-bit range): clamp(rne(x / s), -8, 7); a zero
 * range gives 0. */
int oq_int4_code(float x, float s) {
  if (s == 0.0f) return 0;
  float r = rintf(x / s);
  if (r > 7.0f) r = 7.0f;
  if (r < -8.0f) r = -8.0f;
  return (int)r;
}

/* Asymmetric uint8 parameters over [min(mn,0), max(mx,0)]: s = range / 255,
 * zp = clamp(rne(-lo / s), 0, 255)  (P4 Step 2 "per-channel asymmetric INT8",
 * Step 3 v_scale / v_zp). */
void oq_asym_params(float mn, float mx, float* s, uint8_t* zp) {
  float lo = mn < 0.0f ? mn : 0.0f;
  float hi = mx > 0.0f ? mx : 0.0f;
  float sc = (hi - lo) / 255.0f;
  *s = sc;
  if (sc == 0.0f) {
    *zp = 0;
    return;
  }
  float z = rintf(-lo / sc);
  if (z < 0.0f) z = 0.0f;
  if (z > 255.0f) z = 255.0f;
  *zp = (uint8_t)z;
}

/* q = clamp(rne(x / s) + zp, 0, 255); dequantized as (q - zp) * s (P4 Step 3). */
int oq_asym_code(float x, float s, uint8_t zp) {
  if (s == 0.0f) return 0;
  float r = rintf(x / s) + (float)zp;
  if (r < 0.0f) r = 0.0f;
  if (r > 255.0f) r = 255.0f;
  return (int)r;
}

/* One KIVI group (P1 §3, P3 §3): n values at stride `stride`; asymmetric min-max with
 * 2^bits - 1 steps: s = (max - min) / qmax, q = clamp(rne((x - min) / s), 0, qmax).
 * The minimum is kept in fp32 as the zero point; +-0 extremes are stored as +0. */
void oq_kivi_group(const float* x, int n, int stride, int bits, int* codes, float* s,
                   float* mn) {
  float lo = x[0], hi = x[0];
  for (int i = 1; i < n; ++i) {
    float v = x[(size_t)i * stride];
    if (v < lo) lo = v;
    if (v > hi) hi = v;
  }
  if (lo == 0.0f) lo = 0.0f;
  if (hi == 0.0f) hi = 0.0f;
  const int qmax = (1 << bits) - 1;
  const float sc = (hi - lo) / (float)qmax;
  for (int i = 0; i < n; ++i) {
    if (sc == 0.0f) {
      codes[i] = 0;
      continue;
    }
    float diff = x[(size_t)i * stride] - lo;
    float r = rintf(diff / sc);
    if (r < 0.0f) r = 0.0f;
    if (r > (float)qmax) r = (float)qmax;
    codes[i] = (int)r;
  }
  *s = sc;
  *mn = lo;
}

/* IEEE binary16 (sign, 5 exponent bits with bias 15, 10 mantissa bits; subnormals
 * M * 2^-24): nearest value, ties to even mantissa. Values beyond the largest finite
 * 65504 saturate to it (a scale or minimum must stay finite). NaN stays NaN. */
uint16_t oq_f16_encode(float x) {
  const uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
  const float a = fabsf(x);
  if (isnan(x)) return (uint16_t)(sign | 0x7E00);
  if (a >= 65504.0f) return (uint16_t)(sign | 0x7BFF);
  if (a < ldexpf(1.0f, -14)) {
    /* subnormal grid: multiples of 2^-24; 1024 * 2^-24 is the smallest normal (0x0400) */
    const float m = rintf(ldexpf(a, 24));
    return (uint16_t)(sign | (uint16_t)m);
  }
  int e2;
  frexpf(a, &e2);                        /* a in [2^(e2-1), 2^e2) */
  int E = e2 - 1;                        /* unbiased exponent, -14..15 */
  float m = rintf(ldexpf(a, 10 - E));    /* significand * 1024, in [1024, 2048] */
  if (m == 2048.0f) {
    m = 1024.0f;
    E += 1;
  }
  if (E > 15) return (uint16_t)(sign | 0x7BFF);
  return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | ((int)m - 1024)));
}

float oq_f16_decode(uint16_t h) {
  const int s = h >> 15, E = (h >> 10) & 0x1F, M = h & 0x3FF;
  float v;
  if (E == 31)
    v = M == 0 ? INFINITY : NAN;
  else if (E == 0)
    v = ldexpf((float)M, -24);
  else
    v = ldexpf(1.0f + (float)M / 1024.0f, E - 15);
  return s ? -v : v;
}

/* KIVI group with its scale and minimum stored in fp16 (the precision of the tensors the
 * pages' cache code works in, P4 Step 3; half the metadata bytes, so INT2 takes 3 bits per
 * element): the fp32 scale and minimum of oq_kivi_group rounded to fp16, and the codes of
 * the stored values, q = clamp(rne((x - mn16) / s16), 0, qmax); s16 == 0 gives code 0. */
void oq_kivi_group_f16(const float* x, int n, int stride, int bits, int* codes, float* s, float* mn) {
  float sc, lo;
  oq_kivi_group(x, n, stride, bits, codes, &sc, &lo);
  const float s16 = oq_f16_decode(oq_f16_encode(sc)), mn16 = oq_f16_decode(oq_f16_encode(lo));
  const int qmax = (1 << bits) - 1;
  for (int i = 0; i < n; ++i) {
    if (s16 == 0.0f) {
      codes[i] = 0;
      continue;
    }
    float r = rintf((x[(size_t)i * stride] - mn16) / s16);
    if (r < 0.0f) r = 0.0f;
    if (r > (float)qmax) r = (float)qmax;
    codes[i] = (int)r;
  }
  *s = s16;
  *mn = mn16;
}

/* x_hat = fl(fl(q * s) + min): two roundings, no fused multiply-add. */
float oq_kivi_value(int code, float s, float mn) {
  float a = (float)code * s;
  return a + mn;
}

/* ------------------------------------------------------------------------- */
/* cache layout helpers                                                      */
/* ------------------------------------------------------------------------- */

static int is_kivi(int scheme) {
  return scheme == OQ_KIVI_INT4 || scheme == OQ_KIVI_INT2 || scheme == OQ_KIVI_INT4_F16 || scheme == OQ_KIVI_INT2_F16;
}

static int code_bits(int scheme) {
  if (scheme == OQ_KIVI_INT4 || scheme == OQ_INT4_SYM_PER_GROUP || scheme == OQ_KIVI_INT4_F16) return 4;
  if (scheme == OQ_KIVI_INT2 || scheme == OQ_KIVI_INT2_F16) return 2;
  return 8;
}

static int row_bytes(int scheme, int D) { return D * code_bits(scheme) / 8; }

static float input_at(const void* p, int bf16, size_t i) {
  if (bf16) return oq_bf16_to_f32(((const uint16_t*)p)[i]);
  return ((const float*)p)[i];
}

/* Row of token t of (b, h) in the code array, or in a per-token scale array. Dense:
 * [B,Hkv,cap]; paged: token t lives in page page_table[b][t / page], slot t % page. */
static size_t row_of(const oq_cache* c, int b, int h, int t) {
  if (!c->paged) return ((size_t)b * c->Hkv + h) * (size_t)c->cap + (size_t)t;
  int page = c->page_table[(size_t)b * c->max_pages + t / c->page_size];
  return ((size_t)page * c->Hkv + h) * (size_t)c->page_size + (size_t)(t % c->page_size);
}

static void put_code(uint8_t* codes, int scheme, int D, size_t row, int d, int q) {
  const int bits = code_bits(scheme);
  uint8_t* p = codes + row * (size_t)row_bytes(scheme, D);
  if (bits == 8) {
    p[d] = (uint8_t)(q & 0xFF);
    return;
  }
  const int per = 8 / bits;
  const int byte = d / per, sh = (d % per) * bits;
  const uint8_t mask = (uint8_t)(((1 << bits) - 1) << sh);
  p[byte] = (uint8_t)((p[byte] & ~mask) | ((q << sh) & mask));
}

static int get_code(const uint8_t* codes, int scheme, int D, size_t row, int d) {
  const int bits = code_bits(scheme);
  const uint8_t* p = codes + row * (size_t)row_bytes(scheme, D);
  if (bits == 8) return p[d];
  const int per = 8 / bits;
  return (p[d / per] >> ((d % per) * bits)) & ((1 << bits) - 1);
}

int oq_tokens(const oq_cache* c, int b) {
  if (c->paged) return c->seq_lens[b];
  return c->len + (is_kivi(c->k_scheme) ? c->res : 0);
}

/* ------------------------------------------------------------------------- */
/* append                                                                    */
/* ------------------------------------------------------------------------- */

typedef struct {
  const void* x;
  int bf16, n_new;
  const int32_t* lens;
  int Hkv, D;
} block;

static int block_len(const block* k, int b) { return k->lens ? k->lens[b] : k->n_new; }

static float block_at(const block* k, int b, int h, int t, int d) {
  size_t i = (((size_t)b * k->Hkv + h) * (size_t)k->n_new + (size_t)t) * (size_t)k->D + d;
  return input_at(k->x, k->bf16, i);
}

/* Fixed scales of the per-tensor and per-channel schemes, from the tokens of the
 * calibrating append: the cache is built online, so its scales come from runtime
 * statistics of the data (P1 §2, weights-vs-KV comparison table).
 * Per-tensor: one scale over every batch row, head, token and channel (P4 Step 3
 * `x.abs().max() / 127`). Per-channel: one per (kv_head, channel) over batch and
 * tokens (P4 Step 3 reduces V over batch and sequence per channel). */
static void calibrate(const oq_cache* c, const block* k, int scheme, float* scale, uint8_t* zp) {
  const int B = c->B, H = c->Hkv, D = c->D;
  if (scheme == OQ_FP8_E4M3_PER_TENSOR || scheme == OQ_FP8_E5M2_PER_TENSOR || scheme == OQ_INT8_SYM_PER_TENSOR) {
    float amax = 0.0f;
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h)
        for (int t = 0; t < block_len(k, b); ++t)
          for (int d = 0; d < D; ++d) {
            float a = fabsf(block_at(k, b, h, t, d));
            if (a > amax) amax = a;
          }
    scale[0] = amax / (scheme == OQ_FP8_E4M3_PER_TENSOR ? 448.0f : scheme == OQ_FP8_E5M2_PER_TENSOR ? 57344.0f : 127.0f);
  } else if (scheme == OQ_INT8_SYM_PER_CHANNEL) {
    for (int h = 0; h < H; ++h)
      for (int d = 0; d < D; ++d) {
        float amax = 0.0f;
        for (int b = 0; b < B; ++b)
          for (int t = 0; t < block_len(k, b); ++t) {
            float a = fabsf(block_at(k, b, h, t, d));
            if (a > amax) amax = a;
          }
        scale[h * D + d] = amax / 127.0f;
      }
  } else if (scheme == OQ_UINT8_ASYM_PER_CHANNEL) {
    for (int h = 0; h < H; ++h)
      for (int d = 0; d < D; ++d) {
        float mn = 0.0f, mx = 0.0f;
        int first = 1;
        for (int b = 0; b < B; ++b)
          for (int t = 0; t < block_len(k, b); ++t) {
            float v = block_at(k, b, h, t, d);
            if (first || v < mn) mn = v;
            if (first || v > mx) mx = v;
            first = 0;
          }
        oq_asym_params(mn, mx, &scale[h * D + d], &zp[h * D + d]);
      }
  }
}

/* Code of value x under a fixed scale s (and zero point zp) of an 8-bit scheme with
 * batch-wide scales. */
static int code_for(int scheme, float x, float s, uint8_t zp) {
  switch (scheme) {
    case OQ_FP8_E4M3_PER_TENSOR:
      return s == 0.0f ? 0 : oq_e4m3_encode(x / s);
    case OQ_FP8_E5M2_PER_TENSOR:
      return s == 0.0f ? 0 : oq_e5m2_encode(x / s);
    case OQ_INT8_SYM_PER_TENSOR:
    case OQ_INT8_SYM_PER_CHANNEL:
      return oq_sym_code(x, s, 127);
    case OQ_UINT8_ASYM_PER_CHANNEL:
      return oq_asym_code(x, s, zp);
  }
  return 0;
}

/* Quantize token t of the block (b, h) into cache row `row` (8-bit schemes and INT4
 * per group). */
static void quantize_token(const oq_cache* c, const block* k, int scheme, uint8_t* codes,
                           float* scale, const uint8_t* zp, int b, int h, int t, size_t row) {
  const int D = c->D;
  if (scheme == OQ_INT4_SYM_PER_GROUP) {
    /* one scale per group of g consecutive channels of this token (P3 §2, P4 Step 2) */
    const int g = c->group;
    for (int j = 0; j < D / g; ++j) {
      float amax = 0.0f;
      for (int d = j * g; d < (j + 1) * g; ++d) {
        float a = fabsf(block_at(k, b, h, t, d));
        if (a > amax) amax = a;
      }
      const float s = amax / 7.0f;
      scale[row * (size_t)(D / g) + (size_t)j] = s;
      for (int d = j * g; d < (j + 1) * g; ++d)
        put_code(codes, scheme, D, row, d, oq_int4_code(block_at(k, b, h, t, d), s) & 0xF);
    }
    return;
  }
  float tok_scale = 0.0f;
  if (scheme == OQ_INT8_SYM_PER_TOKEN) {
    /* one scale per token row over head_dim (P3 §2 "INT8 Per-Token") */
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) {
      float a = fabsf(block_at(k, b, h, t, d));
      if (a > amax) amax = a;
    }
    tok_scale = amax / 127.0f;
    scale[row] = tok_scale;
  }
  for (int d = 0; d < D; ++d) {
    const float x = block_at(k, b, h, t, d);
    int q = 0;
    if (scheme == OQ_INT8_SYM_PER_TOKEN)
      q = oq_sym_code(x, tok_scale, 127);
    else if (scheme == OQ_INT8_SYM_PER_CHANNEL || scheme == OQ_UINT8_ASYM_PER_CHANNEL)
      q = code_for(scheme, x, scale[h * D + d], zp ? zp[h * D + d] : 0);
    else
      q = code_for(scheme, x, scale[0], 0);
    put_code(codes, scheme, D, row, d, q);
  }
}

/* KIVI flush of R consecutive tokens (b, h) starting at cache position pos0 (a multiple
 * of R). x is [R, D] fp32. Keys: per channel over each group of g tokens (P1 §3 "Key:
 * Per-Channel Quantization"). Values: per token over each group of g channels (P1 §3
 * "Value: Per-Token Quantization"). Scales and minima stored as fp32. */
static void kivi_flush(oq_cache* c, int b, int h, int pos0, const float* xk, const float* xv,
                       int R) {
  const int D = c->D, g = c->group, H = c->Hkv;
  const int kb = code_bits(c->k_scheme), vb = code_bits(c->v_scheme);
  const int kh = c->k_scheme == OQ_KIVI_INT4_F16 || c->k_scheme == OQ_KIVI_INT2_F16;
  const int vh = c->v_scheme == OQ_KIVI_INT4_F16 || c->v_scheme == OQ_KIVI_INT2_F16;
  int* codes = (int*)malloc(sizeof(int) * (size_t)(g > D ? g : D));
  for (int gi = 0; gi < R / g; ++gi) {
    const size_t meta = (((size_t)b * H + h) * (size_t)(c->cap / g) + (size_t)(pos0 / g + gi)) * D;
    for (int d = 0; d < D; ++d) {
      float s, mn;
      (kh ? oq_kivi_group_f16 : oq_kivi_group)(xk + (size_t)gi * g * D + d, g, D, kb, codes, &s, &mn);
      c->k_scale[meta + d] = s;
      c->k_zero[meta + d] = mn;
      for (int j = 0; j < g; ++j)
        put_code(c->k_codes, c->k_scheme, D, row_of(c, b, h, pos0 + gi * g + j), d, codes[j]);
    }
  }
  for (int t = 0; t < R; ++t) {
    const size_t row = row_of(c, b, h, pos0 + t);
    for (int j = 0; j < D / g; ++j) {
      float s, mn;
      (vh ? oq_kivi_group_f16 : oq_kivi_group)(xv + (size_t)t * D + (size_t)j * g, g, 1, vb, codes, &s, &mn);
      c->v_scale[row * (size_t)(D / g) + j] = s;
      c->v_zero[row * (size_t)(D / g) + j] = mn;
      for (int i = 0; i < g; ++i) put_code(c->v_codes, c->v_scheme, D, row, j * g + i, codes[i]);
    }
  }
  free(codes);
}

/* KIVI append (P1 §3 "Residual Cache for Streaming", P3 §3 "Residual FP16 Buffer"):
 * tokens enter a bf16 residual of rcap tokens; when a token arrives and the residual
 * is full, its rcap tokens are quantized (rcap/g key groups) and it is emptied. For a
 * block of n tokens onto a residual of r tokens this flushes r + n - r' tokens, with
 * r' = ((r + n - 1) mod rcap) + 1 tokens left in the residual. */
static int append_kivi(oq_cache* c, const block* kb, const block* vb) {
  const int B = c->B, H = c->Hkv, D = c->D, R = c->rcap;
  const int n = kb->n_new, r = c->res, total = r + n;
  if (n == 0) return 0;
  if (!kb->bf16) return -1;
  const int r_new = ((total - 1) % R) + 1;
  const int flushed = total - r_new;
  if (c->len + flushed > c->cap) return -1;
  float* xk = (float*)malloc(sizeof(float) * (size_t)R * D);
  float* xv = (float*)malloc(sizeof(float) * (size_t)R * D);
  uint16_t* keep_k = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)R * D);
  uint16_t* keep_v = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)R * D);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t res_base = ((size_t)b * H + h) * (size_t)R * D;
      const size_t in_base = ((size_t)b * H + h) * (size_t)n * D;
      /* combined stream: residual tokens 0..r-1 then new tokens */
#define STREAM_BITS(arr_res, arr_in, i, d) \
  ((i) < r ? (arr_res)[res_base + (size_t)(i) * D + (d)] \
           : ((const uint16_t*)(arr_in))[in_base + (size_t)((i) - r) * D + (d)])
      for (int ch = 0; ch < flushed / R; ++ch) {
        for (int t = 0; t < R; ++t)
          for (int d = 0; d < D; ++d) {
            xk[(size_t)t * D + d] = oq_bf16_to_f32(STREAM_BITS(c->k_res, kb->x, ch * R + t, d));
            xv[(size_t)t * D + d] = oq_bf16_to_f32(STREAM_BITS(c->v_res, vb->x, ch * R + t, d));
          }
        kivi_flush(c, b, h, c->len + ch * R, xk, xv, R);
      }
      for (int t = 0; t < r_new; ++t)
        for (int d = 0; d < D; ++d) {
          keep_k[(size_t)t * D + d] = STREAM_BITS(c->k_res, kb->x, flushed + t, d);
          keep_v[(size_t)t * D + d] = STREAM_BITS(c->v_res, vb->x, flushed + t, d);
        }
#undef STREAM_BITS
      memcpy(c->k_res + res_base, keep_k, sizeof(uint16_t) * (size_t)r_new * D);
      memcpy(c->v_res + res_base, keep_v, sizeof(uint16_t) * (size_t)r_new * D);
    }
  free(xk);
  free(xv);
  free(keep_k);
  free(keep_v);
  c->len += flushed;
  c->res = r_new;
  return 0;
}

/* Dequantized value of an 8-bit code with batch-wide scale s (and zero point zp). */
static float fixed_value(int scheme, int q, float s, uint8_t zp) {
  switch (scheme) {
    case OQ_FP8_E4M3_PER_TENSOR:
      return oq_e4m3_decode((uint8_t)q) * s;
    case OQ_FP8_E5M2_PER_TENSOR:
      return oq_e5m2_decode((uint8_t)q) * s;
    case OQ_INT8_SYM_PER_TENSOR:
    case OQ_INT8_SYM_PER_CHANNEL:
      return (float)(int8_t)q * s;
    case OQ_UINT8_ASYM_PER_CHANNEL:
      return (float)(q - (int)zp) * s;
  }
  return 0.0f;
}

/* Rescaling append, one side (P4 Step 3 merges the scale of every new block into the
 * cached one with a running maximum; P4 Step 7 wants scales that only grow, or are
 * recomputed as the cache grows). Symmetric schemes: s' = max(s, s_block) per scale
 * element, s_block as in calibration. Asymmetric: (s', zp') of the union of the range the
 * cached (s, zp) represent, [(0 - zp) s, (255 - zp) s], and the block's range widened to
 * hold 0; unchanged when the block's range lies inside. Each cached code whose scale
 * element changed is requantized from its dequantized value (the page's snippet keeps the
 * old codes, which then decode with the wrong scale). */
static void rescale(oq_cache* c, const block* k, int which) {
  const int scheme = which ? c->v_scheme : c->k_scheme;
  float* scale = which ? c->v_scale : c->k_scale;
  uint8_t* zp = which ? c->v_zp : c->k_zp;
  uint8_t* codes = which ? c->v_codes : c->k_codes;
  const int B = c->B, H = c->Hkv, D = c->D;
  const int per_tensor = scheme == OQ_FP8_E4M3_PER_TENSOR || scheme == OQ_FP8_E5M2_PER_TENSOR ||
                         scheme == OQ_INT8_SYM_PER_TENSOR;
  const int per_channel = scheme == OQ_INT8_SYM_PER_CHANNEL || scheme == OQ_UINT8_ASYM_PER_CHANNEL;
  if (!per_tensor && !per_channel) return;
  const int n = per_tensor ? 1 : H * D;
  float* s_old = (float*)malloc(sizeof(float) * n);
  uint8_t* zp_old = (uint8_t*)calloc(n, 1);
  float* s_blk = (float*)calloc(n, sizeof(float));
  uint8_t* zp_blk = (uint8_t*)calloc(n, 1);
  memcpy(s_old, scale, sizeof(float) * n);
  if (zp) memcpy(zp_old, zp, n);
  if (scheme != OQ_UINT8_ASYM_PER_CHANNEL) {
    calibrate(c, k, scheme, s_blk, zp_blk);
    for (int i = 0; i < n; ++i)
      if (s_blk[i] > scale[i]) scale[i] = s_blk[i];
  } else {
    for (int h = 0; h < H; ++h)
      for (int d = 0; d < D; ++d) {
        float mn = 0.0f, mx = 0.0f;
        int first = 1;
        for (int b = 0; b < B; ++b)
          for (int t = 0; t < block_len(k, b); ++t) {
            float v = block_at(k, b, h, t, d);
            if (first || v < mn) mn = v;
            if (first || v > mx) mx = v;
            first = 0;
          }
        const int i = h * D + d;
        const float lo_b = mn < 0.0f ? mn : 0.0f, hi_b = mx > 0.0f ? mx : 0.0f;
        const float lo_o = (float)(0 - (int)zp_old[i]) * s_old[i];
        const float hi_o = (float)(255 - (int)zp_old[i]) * s_old[i];
        if (lo_b < lo_o || hi_b > hi_o)
          oq_asym_params(lo_b < lo_o ? lo_b : lo_o, hi_b > hi_o ? hi_b : hi_o, &scale[i], &zp[i]);
      }
  }
  for (int b = 0; b < B; ++b) {
    const int len = c->paged ? c->seq_lens[b] : c->len;
    for (int h = 0; h < H; ++h)
      for (int t = 0; t < len; ++t) {
        const size_t row = row_of(c, b, h, t);
        for (int d = 0; d < D; ++d) {
          const int i = per_tensor ? 0 : h * D + d;
          const uint8_t z_new = zp ? zp[i] : 0;
          if (scale[i] == s_old[i] && z_new == zp_old[i]) continue;
          const float x = fixed_value(scheme, get_code(codes, scheme, D, row, d), s_old[i], zp_old[i]);
          put_code(codes, scheme, D, row, d, code_for(scheme, x, scale[i], z_new));
        }
      }
  }
  free(s_old);
  free(zp_old);
  free(s_blk);
  free(zp_blk);
}

static int append_rows(oq_cache* c, const block* kbp, const block* vbp, int calibrate_flag);

/* fp32 copy of a [B, Hkv, n_new, D] block with every row rotated. */
static float* rotated_rows(const oq_cache* c, const void* x, int in_bf16, int n_new) {
  const size_t n = (size_t)c->B * (size_t)c->Hkv * (size_t)n_new * (size_t)c->D;
  float* r = (float*)malloc(sizeof(float) * (n ? n : 1));
  for (size_t i = 0; i < n; ++i) r[i] = input_at(x, in_bf16, i);
  for (size_t row = 0; row < n / (size_t)c->D; ++row) oq_fwht(r + row * c->D, c->D);
  return r;
}

int oq_append(oq_cache* c, const void* k_new, const void* v_new, int in_bf16, int n_new,
              const int32_t* new_lens, int calibrate_flag) {
  block kb = {k_new, in_bf16, n_new, new_lens, c->Hkv, c->D};
  block vb = {v_new, in_bf16, n_new, new_lens, c->Hkv, c->D};
  if (new_lens && !c->paged) return -1;
  if (c->rotate && c->rope_theta > 0.0f) return -1;  /* one of the two rotations at a time */
  if (is_kivi(c->k_scheme) || is_kivi(c->v_scheme)) {
    if (!(is_kivi(c->k_scheme) && is_kivi(c->v_scheme)) || c->paged || c->rotate) return -1;
    return append_kivi(c, &kb, &vb);
  }
  if (!c->rotate) return append_rows(c, &kb, &vb, calibrate_flag);
  /* rotate every row of the block first: statistics and codes are those of H x */
  float* kr = rotated_rows(c, k_new, in_bf16, n_new);
  float* vr = rotated_rows(c, v_new, in_bf16, n_new);
  block kq = {kr, 0, n_new, new_lens, c->Hkv, c->D};
  block vq = {vr, 0, n_new, new_lens, c->Hkv, c->D};
  const int rc = append_rows(c, &kq, &vq, calibrate_flag);
  free(kr);
  free(vr);
  return rc;
}

static int append_rows(oq_cache* c, const block* kbp, const block* vbp, int calibrate_flag) {
  const block kb = *kbp, vb = *vbp;
  const int n_new = kb.n_new;
  /* capacity */
  for (int b = 0; b < c->B; ++b) {
    const int start = c->paged ? c->seq_lens[b] : c->len;
    const int end = start + block_len(&kb, b);
    if (c->paged) {
      if (end > c->max_pages * c->page_size) return -1;
      for (int t = start; t < end; ++t) {
        int page = c->page_table[(size_t)b * c->max_pages + t / c->page_size];
        if (page < 0 || page >= c->num_pages) return -1;
      }
    } else if (end > c->cap) {
      return -1;
    }
  }
  if (calibrate_flag == OQ_APPEND_CALIBRATE) {
    calibrate(c, &kb, c->k_scheme, c->k_scale, c->k_zp);
    calibrate(c, &vb, c->v_scheme, c->v_scale, c->v_zp);
  } else if (calibrate_flag == OQ_APPEND_RESCALE) {
    rescale(c, &kb, 0);
    rescale(c, &vb, 1);
  } else if (calibrate_flag != 0) {
    return -1;
  }
  for (int b = 0; b < c->B; ++b) {
    const int start = c->paged ? c->seq_lens[b] : c->len;
    for (int h = 0; h < c->Hkv; ++h)
      for (int t = 0; t < block_len(&kb, b); ++t) {
        const size_t row = row_of(c, b, h, start + t);
        quantize_token(c, &kb, c->k_scheme, c->k_codes, c->k_scale, c->k_zp, b, h, t, row);
        quantize_token(c, &vb, c->v_scheme, c->v_codes, c->v_scale, c->v_zp, b, h, t, row);
      }
  }
  if (c->paged)
    for (int b = 0; b < c->B; ++b) c->seq_lens[b] += block_len(&kb, b);
  else
    c->len += n_new;
  return 0;
}

int oq_calibrate(oq_cache* c, const void* k_new, const void* v_new, int in_bf16, int n_new,
                 const int32_t* new_lens) {
  if (is_kivi(c->k_scheme) || is_kivi(c->v_scheme)) return -1;
  float* kr = c->rotate ? rotated_rows(c, k_new, in_bf16, n_new) : NULL;
  float* vr = c->rotate ? rotated_rows(c, v_new, in_bf16, n_new) : NULL;
  block kb = {kr ? (const void*)kr : k_new, kr ? 0 : in_bf16, n_new, new_lens, c->Hkv, c->D};
  block vb = {vr ? (const void*)vr : v_new, vr ? 0 : in_bf16, n_new, new_lens, c->Hkv, c->D};
  calibrate(c, &kb, c->k_scheme, c->k_scale, c->k_zp);
  calibrate(c, &vb, c->v_scheme, c->v_scale, c->v_zp);
  free(kr);
  free(vr);
  return 0;
}

/* ------------------------------------------------------------------------- */
/* dequantize                                                                */
/* ------------------------------------------------------------------------- */

/* Dequantized value of channel d of token t of (b, h): P4 Step 3 `dequantize`
 * (q * scale, or (q - zp) * scale), the E4M3 decode times the scale, the KIVI
 * fl(fl(q*s)+min), or the bf16 residual token itself. */
static float value_at(const oq_cache* c, int which, int b, int h, int t, int d) {
  const int scheme = which ? c->v_scheme : c->k_scheme;
  const uint8_t* codes = which ? c->v_codes : c->k_codes;
  const float* scale = which ? c->v_scale : c->k_scale;
  const float* zero = which ? c->v_zero : c->k_zero;
  const uint8_t* zp = which ? c->v_zp : c->k_zp;
  const int D = c->D, H = c->Hkv;
  if (is_kivi(scheme)) {
    if (t >= c->len) {
      const uint16_t* res = which ? c->v_res : c->k_res;
      return oq_bf16_to_f32(res[(((size_t)b * H + h) * (size_t)c->rcap + (size_t)(t - c->len)) * D + d]);
    }
    const size_t row = row_of(c, b, h, t);
    const int q = get_code(codes, scheme, D, row, d);
    size_t m;
    if (which == 0)
      m = (((size_t)b * H + h) * (size_t)(c->cap / c->group) + (size_t)(t / c->group)) * D + d;
    else
      m = row * (size_t)(D / c->group) + (size_t)(d / c->group);
    return oq_kivi_value(q, scale[m], zero[m]);
  }
  const size_t row = row_of(c, b, h, t);
  const int q = get_code(codes, scheme, D, row, d);
  switch (scheme) {
    case OQ_FP8_E4M3_PER_TENSOR:
      return oq_e4m3_decode((uint8_t)q) * scale[0];
    case OQ_FP8_E5M2_PER_TENSOR:
      return oq_e5m2_decode((uint8_t)q) * scale[0];
    case OQ_INT8_SYM_PER_TENSOR:
      return (float)(int8_t)q * scale[0];
    case OQ_INT8_SYM_PER_TOKEN:
      return (float)(int8_t)q * scale[row];
    case OQ_INT8_SYM_PER_CHANNEL:
      return (float)(int8_t)q * scale[h * D + d];
    case OQ_UINT8_ASYM_PER_CHANNEL:
      return (float)(q - (int)zp[h * D + d]) * scale[h * D + d];
    case OQ_INT4_SYM_PER_GROUP:
      return (float)(q >= 8 ? q - 16 : q) * scale[row * (size_t)(D / c->group) + (size_t)(d / c->group)];
  }
  return 0.0f;
}

void oq_dequantize(const oq_cache* c, int which, float* out, int T_out) {
  const int D = c->D;
  for (int b = 0; b < c->B; ++b)
    for (int h = 0; h < c->Hkv; ++h) {
      const int T = oq_tokens(c, b);
      for (int t = 0; t < T_out; ++t) {
        float* row = out + (((size_t)b * c->Hkv + h) * (size_t)T_out + t) * D;
        for (int d = 0; d < D; ++d) row[d] = t < T ? value_at(c, which, b, h, t, d) : 0.0f;
        if (c->rotate && t < T) oq_fwht(row, D);  /* back from the rotated domain */
      }
    }
}

/* ------------------------------------------------------------------------- */
/* attention (fp64)                                                          */
/* ------------------------------------------------------------------------- */

/* softmax(scale * q.k_t) over t, then the probability-weighted sum of v_t; scores
 * and the sums are fp64, t ascending. T == 0 gives zeros and lse = -inf. */
/* Scores against fp64 keys (kd) when given, else the fp32 keys k. */
static void attention_row(const float* q, const float* k, const double* kd, const float* v, int T, int D,
                          float scale, double* out, double* lse) {
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (T == 0) {
    *lse = -INFINITY;
    return;
  }
  double* s = (double*)malloc(sizeof(double) * (size_t)T);
  double m = -INFINITY;
  for (int t = 0; t < T; ++t) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d)
      acc += (double)q[d] * (kd ? kd[(size_t)t * D + d] : (double)k[(size_t)t * D + d]);
    s[t] = acc * (double)scale;
    if (s[t] > m) m = s[t];
  }
  double l = 0.0;
  for (int t = 0; t < T; ++t) {
    const double p = exp(s[t] - m);
    l += p;
    for (int d = 0; d < D; ++d) out[d] += p * (double)v[(size_t)t * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
  *lse = m + log(l);
  free(s);
}

void oq_attention_row(const float* q, const float* k, const float* v, int T, int D,
                      float scale, double* out, double* lse) {
  attention_row(q, k, NULL, v, T, D, scale, out, lse);
}

void oq_rope(double* x, int D, int pos, double theta) {
  const int half = D / 2;
  for (int i = 0; i < half; ++i) {
    const double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
    const double ang = (double)pos * inv_freq;
    const double c = cos(ang), s = sin(ang);
    const double a = x[i], b = x[i + half];
    x[i] = a * c - b * s;
    x[i + half] = b * c + a * s;
  }
}

static void decode_pair(const oq_cache* c, const void* q, int q_bf16, float scale, int b,
                        int hk, double* out, double* lse) {
  const int D = c->D, G = c->Hq / c->Hkv, T = oq_tokens(c, b);
  float* k = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * D);
  float* v = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * D);
  float* qr = (float*)malloc(sizeof(float) * (size_t)D);
  for (int t = 0; t < T; ++t)
    for (int d = 0; d < D; ++d) {
      k[(size_t)t * D + d] = value_at(c, 0, b, hk, t, d);
      v[(size_t)t * D + d] = value_at(c, 1, b, hk, t, d);
    }
  double* kd = NULL;
  if (c->rope_theta > 0.0f) {  /* pre-RoPE keys: token t sits at position t of the sequence */
    kd = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * D);
    for (int t = 0; t < T; ++t) {
      for (int d = 0; d < D; ++d) kd[(size_t)t * D + d] = (double)k[(size_t)t * D + d];
      oq_rope(kd + (size_t)t * D, D, t, (double)c->rope_theta);
    }
  }
  for (int j = 0; j < G; ++j) {
    const int hq = hk * G + j; /* query head h reads kv head h / G */
    for (int d = 0; d < D; ++d) qr[d] = input_at(q, q_bf16, ((size_t)b * c->Hq + hq) * D + d);
    if (c->rotate) oq_fwht(qr, D);  /* the cache holds H k and H v: attend with H q */
    double l;
    attention_row(qr, k, kd, v, T, D, scale, out + (size_t)j * D, &l);
    if (c->rotate) fwht_d(out + (size_t)j * D, D);  /* sum p (H v) = H (sum p v) */
    if (lse) lse[j] = l;
  }
  free(k);
  free(kd);
  free(v);
  free(qr);
}

void oq_decode(const oq_cache* c, const void* q, int q_bf16, float scale, double* out,
               double* lse) {
  const int G = c->Hq / c->Hkv;
  for (int b = 0; b < c->B; ++b)
    for (int hk = 0; hk < c->Hkv; ++hk) {
      const size_t base = (size_t)b * c->Hq + (size_t)hk * G;
      decode_pair(c, q, q_bf16, scale, b, hk, out + base * c->D, lse ? lse + base : NULL);
    }
}

void oq_decode_pairs(const oq_cache* c, const void* q, int q_bf16, float scale,
                     const int32_t* pairs, int n_pairs, double* out, double* lse) {
  const int G = c->Hq / c->Hkv;
  for (int i = 0; i < n_pairs; ++i)
    decode_pair(c, q, q_bf16, scale, pairs[2 * i], pairs[2 * i + 1],
                out + (size_t)i * G * c->D, lse ? lse + (size_t)i * G : NULL);
}

/* P3 introduction: per-token KV bytes are K and V (2) times the element width times
 * layers, KV heads and head dimension; the page states it for 2-byte elements. */
double oq_kv_bytes_per_token(int n_layers, int n_kv_heads, int d_head, double bytes_per_elem) {
  return 2.0 * bytes_per_elem * (double)n_layers * (double)n_kv_heads * (double)d_head;
}

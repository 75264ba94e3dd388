// Quantize-on-append, calibration and dequantize kernels (sm_100a).
//
// Every code, scale and zero point is computed with one correctly rounded fp32 operation
// per step (IEEE division, round-half-to-even), so results are bit-identical to a plain
// sequential statement of the schemes:
//  - symmetric INT8: s = absmax/127, q = clamp(rne(x/s), -127, 127)
//    ("KV Cache Quantization in Production LLM Serving", llms.blog, §2);
//  - FP8 E4M3: s = absmax/448, q = e4m3_rn_satfinite(x/s) (infra.bea.ai §4, llms.blog §1);
//  - FP8 E5M2: s = absmax/57344, q = e5m2_rn_satfinite(x/s) (the other OCP format llms.blog §1
//    compares);
//  - asymmetric uint8 per channel: affine form over a range widened to contain 0
//    ("How KV cache quantization reduces GPU memory", n4n.ai, Steps 2-3);
//  - KIVI: keys per channel over 32-token groups, values per token over 32-channel
//    groups, min-max with 2^bits - 1 steps, bf16 residual of 128 tokens
//    (infra.bea.ai §3; llms.blog §3);
//  - INT4 symmetric per group: s = absmax/7 over 32 consecutive channels of a token,
//    q = clamp(rne(x/s), -8, 7) as two's-complement nibbles (llms.blog §2; n4n.ai Step 2).
#include <cuda_fp8.h>

#include <algorithm>
#include <atomic>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

// ------------------------------------------------------------------ element helpers
template <bool kBf16>
__device__ __forceinline__ void load8(const void* base, size_t elem, float (&x)[8]) {
  if constexpr (kBf16) {
    const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
      x[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    const float4 a = p[0], b = p[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

// Two E5M2 codes, RN-even with saturation to +-57344: lo -> low byte, hi -> high byte.
__device__ __forceinline__ uint32_t e5m2x2_rn(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes, RN-even with saturation: lo -> low byte, hi -> high byte.
__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Row of token `pos` of (b, h): dense [B,H,cap]; paged via the page table. Returns false
// (and flags the status word) when the page slot is outside the table or the pool.
__device__ __forceinline__ bool cache_row(const AppendParams& p, int b, int h, int pos, size_t& row) {
  if (!p.paged) {
    row = ((size_t)b * p.H + h) * (size_t)p.cap + (size_t)pos;
    return true;
  }
  const int pi = pos / p.page_size;
  if (pos < 0 || pi >= p.max_pages) {
    flag(p.status, KVQ_DEV_BAD_LENGTH);
    return false;
  }
  const int page = p.page_table[(size_t)b * p.max_pages + pi];
  if (page < 0 || page >= p.num_pages) {
    flag(p.status, KVQ_DEV_BAD_PAGE);
    return false;
  }
  row = ((size_t)page * p.H + h) * (size_t)p.page_size + (size_t)(pos % p.page_size);
  return true;
}

__device__ __forceinline__ int new_count(const AppendParams& p, int b) {
  if (!p.new_lens) return p.n_new;
  int n = p.new_lens[b];
  return n < 0 ? 0 : (n > p.n_new ? p.n_new : n);
}

// ------------------------------------------------------------------ calibration
// Workspace keys (uint32): [0] K absmax, [1] V absmax, then per side two arrays of H*D
// (absmax or order-key min, and order-key max).
__global__ void calib_init_kernel(uint32_t* keys, int hd) {
  const int n = 2 + 4 * hd;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    uint32_t v = 0u;
    if (i >= 2) {
      const int j = (i - 2) % (2 * hd);
      v = j < hd ? 0xFFFFFFFFu : 0u;  // first array: min keys start high; absmax uses max
    }
    keys[i] = v;
  }
}

// One block per (token chunk, b*H + h, side). 256 threads: 16 row lanes x 16 lanes of
// 8 channels. Reduces absmax (per-tensor), absmax per channel, or min/max per channel.
template <bool kBf16>
__global__ void __launch_bounds__(256) calib_reduce_kernel(AppendParams p, uint32_t* keys) {
  constexpr int kChunk = 256;
  const int side = blockIdx.z;
  const int scheme = side ? p.v_scheme : p.k_scheme;
  const bool per_tensor = scheme == KVQ_FP8_E4M3_PER_TENSOR || scheme == KVQ_FP8_E5M2_PER_TENSOR ||
                          scheme == KVQ_INT8_SYM_PER_TENSOR;
  const bool per_channel = scheme == KVQ_INT8_SYM_PER_CHANNEL || scheme == KVQ_UINT8_ASYM_PER_CHANNEL;
  if (!per_tensor && !per_channel) return;
  const bool asym = scheme == KVQ_UINT8_ASYM_PER_CHANNEL;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int n_b = new_count(p, b);
  const int t_begin = blockIdx.x * kChunk;
  if (t_begin >= n_b) return;
  const int t_end = min(n_b, t_begin + kChunk);
  const void* x = side ? p.v_new : p.k_new;
  const int lane8 = threadIdx.x & 15, rl = threadIdx.x >> 4;
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i] = INFINITY;
    hi[i] = asym ? -INFINITY : 0.0f;
  }
  for (int t = t_begin + rl; t < t_end; t += 16) {
    float v[8];
    load8<kBf16>(x, (((size_t)b * p.H + h) * (size_t)p.n_new + t) * kHeadDim + lane8 * 8, v);
    if (p.rotate) fwht_row16(v, 0xFFFFu << (threadIdx.x & 16), lane8);  // the half warp shares t
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (asym) {
        lo[i] = fminf(lo[i], v[i]);
        hi[i] = fmaxf(hi[i], v[i]);
      } else {
        hi[i] = fmaxf(hi[i], fabsf(v[i]));
      }
    }
  }
  __shared__ float s_lo[16][kHeadDim], s_hi[16][kHeadDim];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_lo[rl][lane8 * 8 + i] = lo[i];
    s_hi[rl][lane8 * 8 + i] = hi[i];
  }
  __syncthreads();
  const int hd = p.H * kHeadDim;
  uint32_t* base = keys + 2 + side * 2 * hd;
  if (threadIdx.x < kHeadDim) {
    const int d = threadIdx.x;
    float a = s_lo[0][d], m = s_hi[0][d];
    for (int r = 1; r < 16; ++r) {
      a = fminf(a, s_lo[r][d]);
      m = fmaxf(m, s_hi[r][d]);
    }
    if (per_channel) {
      if (asym) {
        atomicMin(base + h * kHeadDim + d, order_key(a));
        atomicMax(base + hd + h * kHeadDim + d, order_key(m));
      } else {
        atomicMax(base + hd + h * kHeadDim + d, __float_as_uint(m));  // m >= +0
      }
    } else {
      s_hi[0][d] = m;
    }
  }
  if (per_tensor) {
    __syncthreads();
    if (threadIdx.x < 32) {
      float m = 0.0f;
      for (int d = threadIdx.x; d < kHeadDim; d += 32) m = fmaxf(m, s_hi[0][d]);
      m = warp_max(m);
      if (threadIdx.x == 0) atomicMax(keys + side, __float_as_uint(m));
    }
  }
}

// Asymmetric parameters of the range [lo, hi] (lo <= 0 <= hi): s = (hi - lo) / 255,
// zp = clamp(rne(-lo / s), 0, 255); a zero range gives s = 0 and zp = 0.
__device__ __forceinline__ void asym_params(float lo, float hi, float& s, uint8_t& zp) {
  s = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
  int z = 0;
  if (s != 0.0f) {
    float zf = rintf(__fdiv_rn(-lo, s));
    zf = fminf(fmaxf(zf, 0.0f), 255.0f);
    z = (int)zf;
  }
  zp = (uint8_t)z;
}

__device__ __forceinline__ float calib_scale(int scheme, float amax) {
  return __fdiv_rn(amax, scheme == KVQ_FP8_E4M3_PER_TENSOR   ? 448.0f
                         : scheme == KVQ_FP8_E5M2_PER_TENSOR ? 57344.0f
                                                             : 127.0f);
}

// Turn the reduced statistics into scales (and zero points): one block.
__global__ void calib_finalize_kernel(AppendParams p, const uint32_t* keys) {
  const int hd = p.H * kHeadDim;
  for (int side = 0; side < 2; ++side) {
    const int scheme = side ? p.v_scheme : p.k_scheme;
    float* scale = side ? p.v_scale : p.k_scale;
    uint8_t* zp = side ? p.v_zp : p.k_zp;
    const uint32_t* base = keys + 2 + side * 2 * hd;
    if (scheme == KVQ_FP8_E4M3_PER_TENSOR || scheme == KVQ_FP8_E5M2_PER_TENSOR || scheme == KVQ_INT8_SYM_PER_TENSOR) {
      if (threadIdx.x == 0) scale[0] = calib_scale(scheme, __uint_as_float(keys[side]));
    } else if (scheme == KVQ_INT8_SYM_PER_CHANNEL) {
      for (int i = threadIdx.x; i < hd; i += blockDim.x)
        scale[i] = __fdiv_rn(__uint_as_float(base[hd + i]), 127.0f);
    } else if (scheme == KVQ_UINT8_ASYM_PER_CHANNEL) {
      for (int i = threadIdx.x; i < hd; i += blockDim.x) {
        const float mn = key_to_float(base[i]), mx = key_to_float(base[hd + i]);
        asym_params(mn < 0.0f ? mn : 0.0f, mx > 0.0f ? mx : 0.0f, scale[i], zp[i]);
      }
    }
  }
}

// ------------------------------------------------------------------ 8-bit quantize-store
// Eight input elements, kept as loaded until they are quantized.
template <bool kBf16>
struct Raw8;
template <>
struct Raw8<true> {
  uint4 v;
  __device__ __forceinline__ void load(const void* base, size_t elem) {
    v = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem);
  }
  __device__ __forceinline__ void clear() { v = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct Raw8<false> {
  float4 a, b;
  __device__ __forceinline__ void load(const void* base, size_t elem) {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    a = q[0];
    b = q[1];
  }
  __device__ __forceinline__ void clear() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// Low bytes of four words -> one word (byte i from word i).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  return prmt(prmt(w0, w1, 0x0040u), prmt(w2, w3, 0x0040u), 0x5410u);
}

// Scales of one row's eight channels (one value repeated for per-tensor and per-token).
struct Scales8 {
  float s[8], y[8];
  int zp[8];  // asymmetric only
};

// The code of one element from its exact quotient z (|z| < 2^22), counting saturation.
__device__ __forceinline__ uint32_t code_of(float z, int zp, int scheme, int& sat) {
  if (scheme == KVQ_FP8_E4M3_PER_TENSOR) {
    sat += fabsf(z) > 448.0f;
    return e4m3x2_rn(z, 0.0f) & 0xFFu;
  }
  if (scheme == KVQ_FP8_E5M2_PER_TENSOR) {
    sat += fabsf(z) > 57344.0f;
    return e5m2x2_rn(z, 0.0f) & 0xFFu;
  }
  if (scheme == KVQ_UINT8_ASYM_PER_CHANNEL) {
    const float c = __fadd_rn(rintf(z), (float)zp);
    sat += c < 0.0f || c > 255.0f;
    return (uint32_t)(int)fminf(fmaxf(c, 0.0f), 255.0f);
  }
  float c = rintf(z);
  if (fabsf(c) > 127.0f) {
    ++sat;
    c = c > 0.0f ? 127.0f : -127.0f;
  }
  return (uint32_t)(int)c & 0xFFu;
}

// The slow form of a row: element by element, dividing where the quotient may be out of the
// correction's range; counts saturation.
__device__ __forceinline__ uint2 careful_row(const float (&x)[8], const Scales8& sc, bool fast, int scheme, int& sat) {
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t code = 0u;
    if (sc.s[k] != 0.0f) {
      float q, z;
      if (fast) {
        z = quot(x[k], sc.s[k], sc.y[k], q);
        if (!(fabsf(q) < 4194304.0f)) z = __fdiv_rn(x[k], sc.s[k]);  // huge or not finite
      } else {
        z = __fdiv_rn(x[k], sc.s[k]);
      }
      code = code_of(z, sc.zp[k], scheme, sat);
    }
    w[k >> 2] |= code << (8 * (k & 3));
  }
  return make_uint2(w[0], w[1]);
}

// Fast rows (s in range): false when a value may saturate or is out of range.
template <bool kE5M2>
__device__ __forceinline__ bool fp8_row(const float (&x)[8], const Scales8& sc, uint2& out) {
  uint32_t c[4];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float q0, q1;
    const float z0 = quot(x[2 * k], sc.s[0], sc.y[0], q0), z1 = quot(x[2 * k + 1], sc.s[0], sc.y[0], q1);
    c[k] = kE5M2 ? e5m2x2_rn(z0, z1) : e4m3x2_rn(z0, z1);
    amax = fmaxf(amax, fmaxf(fabsf(q0), fabsf(q1)));
  }
  out = make_uint2(prmt(c[0], c[1], 0x5410u), prmt(c[2], c[3], 0x5410u));
  return amax < (kE5M2 ? 57340.0f : 447.9f);  // |z| below the largest finite: nothing saturates
                                              // (q is within a few ulps of z)
}

// symmetric: clamp(rne(z), -127, 127); z + 1.5 * 2^23 holds rne(z) (ties to even) in its low bits
__device__ __forceinline__ bool sym_row(const float (&x)[8], const Scales8& sc, uint2& out) {
  uint32_t c[8];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float q;
    const float z = quot(x[k], sc.s[k], sc.y[k], q);
    c[k] = __float_as_uint(__fadd_rn(z, kRoundMagic));
    amax = fmaxf(amax, fabsf(q));
  }
  out = make_uint2(pack_low_bytes(c[0], c[1], c[2], c[3]), pack_low_bytes(c[4], c[5], c[6], c[7]));
  return amax < 127.25f;  // |z| < 127.5: no clamp, no saturation
}

// asymmetric uint8: rne(z) + zp must lie in [0, 255]
__device__ __forceinline__ bool asym_row(const float (&x)[8], const Scales8& sc, uint2& out) {
  uint32_t c[8], range = 0u;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float q;
    const float z = quot(x[k], sc.s[k], sc.y[k], q);
    c[k] = __float_as_uint(__fadd_rn(z, kRoundMagic)) - (uint32_t)(kRoundMagicBits - sc.zp[k]);
    range |= c[k];
  }
  out = make_uint2(pack_low_bytes(c[0], c[1], c[2], c[3]), pack_low_bytes(c[4], c[5], c[6], c[7]));
  return (range & 0xFFFFFF00u) == 0u;  // also fails for huge or non-finite quotients
}

constexpr bool is_per_channel(int s) { return s == KVQ_INT8_SYM_PER_CHANNEL || s == KVQ_UINT8_ASYM_PER_CHANNEL; }

// Two fp32 lanes in one 64-bit register for the packed f32x2 arithmetic of sm_100 (each lane is
// the same correctly rounded IEEE operation as its scalar form).
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float& a, float& b) { asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v)); }
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Eight INT4 codes of a thread's slice of one group: clamp(rne(x / s), -8, 7) as two's-
// complement nibbles, lower channel in the low bits; a zero group gives zero codes. Since
// s = absmax / 7 rounded, |x / s| <= 7 (1 + 2^-23), so rne never leaves [-7, 7] and the clamp
// never acts; RN(z + 1.5 * 2^23) holds rne(z) in its low bits, whose low four bits are the
// two's-complement nibble. The quotients are the fma-corrected ones, two per packed op.
__device__ __forceinline__ uint32_t int4_codes(const float (&x)[8], float s) {
  if (s == 0.0f) return 0u;
  uint32_t w = 0u;
  if (quot_range(s)) {
    const float y = __frcp_rn(s);
    const f32x2 y2 = pk2(y, y), ns2 = pk2(-s, -s), m2 = pk2(kRoundMagic, kRoundMagic);
    uint32_t t[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const f32x2 x2 = pk2(x[2 * k], x[2 * k + 1]);
      const f32x2 q = mul2(x2, y2);
      const f32x2 r = add2(fma2(fma2(q, ns2, x2), y2, q), m2);  // RN(q - e y) + magic
      float t0, t1;
      upk2(r, t0, t1);
      t[2 * k] = __float_as_uint(t0);
      t[2 * k + 1] = __float_as_uint(t1);
    }
    // byte k = (nibble of channel 2k, nibble of channel 2k + 1): the low bytes of the even and
    // of the odd channels gathered by byte permutes, then one shift and one masked merge
    const uint32_t ev = pack_low_bytes(t[0], t[2], t[4], t[6]), od = pack_low_bytes(t[1], t[3], t[5], t[7]);
    return (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float z = __fdiv_rn(x[k], s);
    w |= (__float_as_uint(__fadd_rn(z, kRoundMagic)) & 0xFu) << (4 * k);
  }
  return w;
}

// Rows (b, h, i) of the new block; 16 threads per row, 8 channels each; blockIdx.z = side.
// Bulk form (kR > 1): blockIdx.y = b * H + h and blockIdx.x a run of 16 * kR tokens of that
// row, so no thread divides and every row of the block belongs to one head; each thread loads
// its kR rows before quantizing any. Small form (kR == 1): blockIdx.x covers 16 consecutive
// flattened rows.
template <bool kBf16, int kR, int KS, int VS>
__global__ void __launch_bounds__(256, (is_per_channel(KS) || is_per_channel(VS)) ? 3 : 4)
    quantize_rows_kernel(AppendParams p) {
  // Launched as a programmatic dependent: wait for the previous kernel (its writes of the
  // inputs, its reads of the cache) before touching memory, then let the next kernel (the
  // decode of this step) be scheduled; it waits for this grid to finish before it reads.
  grid_dependency_wait();
  grid_launch_dependents();
  const int side = blockIdx.z;
  const int scheme = side ? VS : KS;  // compile-time per side
  const int lane8 = threadIdx.x & 15;
  const bool per_channel = side ? is_per_channel(VS) : is_per_channel(KS);
  const bool per_tensor = scheme == KVQ_FP8_E4M3_PER_TENSOR || scheme == KVQ_FP8_E5M2_PER_TENSOR ||
                          scheme == KVQ_INT8_SYM_PER_TENSOR;
  float* scale = side ? p.v_scale : p.k_scale;
  const uint8_t* zp = side ? p.v_zp : p.k_zp;
  const void* src_base = side ? p.v_new : p.k_new;
  Scales8 sc;
  bool fixed_fast = true;  // the per-tensor or per-channel scales are all in the correction's range
#pragma unroll
  for (int k = 0; k < 8; ++k) sc.zp[k] = 0;
  if (per_tensor) {
    const float s0 = scale[0], y0 = __frcp_rn(s0);
    fixed_fast = quot_range(s0);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      sc.s[k] = s0;
      sc.y[k] = y0;
    }
  }
  int chan_head = -1;
  int sat = 0;
  // Bulk form: a grid-stride walk over (chunk of 16 * kR tokens, sequence x head) items, so
  // chunks past a sequence's new tokens (a padded paged prefill) cost only a compare, and the
  // per-tensor scale is read once per block. Small form: one item.
  const int nx = kR > 1 ? (p.n_new + 16 * kR - 1) / (16 * kR) : 1;
  const int n_items = kR > 1 ? nx * p.B * p.H : 1;
  for (int item = kR > 1 ? (int)blockIdx.x : 0; item < n_items; item += kR > 1 ? (int)gridDim.x : n_items) {
    Raw8<kBf16> in[kR];
    int rb[kR], rh[kR], ri[kR];
    bool act[kR];
    int rows_at[kR];  // bulk form: cache row of each of the thread's rows (< 2^31, checked at the API)
    int pos_base = 0;  // bulk form: the sequence's first new position, read once (stores may alias it)
    if constexpr (kR > 1) {
      const int bh = item / nx, chunk = item - bh * nx;
      const int b = bh / p.H, h = bh - b * p.H;
      const int n_b = new_count(p, b);
      if (chunk * 16 * kR >= n_b) continue;  // a padded chunk with no token of this sequence
      pos_base = p.paged ? p.seq_lens[b] : p.pos0;
#pragma unroll
      for (int it = 0; it < kR; ++it) {
        const int i = chunk * 16 * kR + 16 * it + (threadIdx.x >> 4);
        rb[it] = b;
        rh[it] = h;
        ri[it] = i;
        act[it] = i < n_b;
        in[it].clear();
        if (act[it]) in[it].load(src_base, ((size_t)bh * p.n_new + i) * kHeadDim + lane8 * 8);
      }
      // every row's cache slot (page-table reads) before any code store: the stores may alias
      // the table, so a lookup left inside the row loop would wait for the previous row's store
#pragma unroll
      for (int it = 0; it < kR; ++it) {
        size_t r64 = 0;
        if (act[it] && !cache_row(p, b, h, pos_base + ri[it], r64)) act[it] = false;
        rows_at[it] = (int)r64;
      }
    } else {
      const int r = blockIdx.x * 16 + (threadIdx.x >> 4);
      const int rows = p.B * p.H * p.n_new;
      const int i = r % p.n_new, bh = r / p.n_new;
      rb[0] = bh / p.H;
      rh[0] = bh - rb[0] * p.H;
      ri[0] = i;
      act[0] = r < rows && i < new_count(p, rb[0]);
      in[0].clear();
      if (act[0]) in[0].load(src_base, (size_t)r * kHeadDim + lane8 * 8);
    }
#pragma unroll
    for (int it = 0; it < kR; ++it) {
      float x[8];
      in[it].unpack(x);
      if (p.rotate) fwht_row16(x, 0xFFFFu << (threadIdx.x & 16), lane8);
      // per-token scale: absmax over the 16 lanes of this row (a half warp)
      float tok_s = 0.0f;
      if (scheme == KVQ_INT8_SYM_PER_TOKEN) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(x[k]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        tok_s = __fdiv_rn(m, 127.0f);
      }
      // INT4 per group: absmax over the group / 8 lanes (4, 8 or 16) of the group
      if (scheme == KVQ_INT4_SYM_PER_GROUP) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(x[k]));
        for (int o = 1; o < p.group / 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        tok_s = __fdiv_rn(m, 7.0f);
      }
      if (!act[it]) continue;
      const int b = rb[it], h = rh[it];
      size_t row;
      if constexpr (kR > 1) {
        row = (size_t)rows_at[it];
      } else {
        if (!cache_row(p, b, h, (p.paged ? p.seq_lens[b] : p.pos0) + ri[it], row)) continue;
      }
      if (scheme == KVQ_INT4_SYM_PER_GROUP) {
        uint8_t* dst = static_cast<uint8_t*>(side ? p.v_codes : p.k_codes) + row * (kHeadDim / 2);
        *reinterpret_cast<uint32_t*>(dst + lane8 * 4) = int4_codes(x, tok_s);
        const int lanes = p.group / 8;  // lanes per group
        if ((lane8 & (lanes - 1)) == 0) scale[row * (kHeadDim / p.group) + lane8 / lanes] = tok_s;
        continue;
      }
      if (per_channel && h != chan_head) {
        fixed_fast = true;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int c = h * kHeadDim + lane8 * 8 + k;
          sc.s[k] = scale[c];
          sc.y[k] = __frcp_rn(sc.s[k]);
          fixed_fast &= quot_range(sc.s[k]);
          if (scheme == KVQ_UINT8_ASYM_PER_CHANNEL) sc.zp[k] = zp[c];
        }
        chan_head = h;
      }
      bool row_fast = fixed_fast;
      if (scheme == KVQ_INT8_SYM_PER_TOKEN) {
        const float y = __frcp_rn(tok_s);
        row_fast = quot_range(tok_s);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          sc.s[k] = tok_s;
          sc.y[k] = y;
        }
      }
      uint2 codes;
      bool ok = false;
      if (row_fast) {
        if (scheme == KVQ_FP8_E4M3_PER_TENSOR)
          ok = fp8_row<false>(x, sc, codes);
        else if (scheme == KVQ_FP8_E5M2_PER_TENSOR)
          ok = fp8_row<true>(x, sc, codes);
        else if (scheme == KVQ_UINT8_ASYM_PER_CHANNEL)
          ok = asym_row(x, sc, codes);
        else
          ok = sym_row(x, sc, codes);
      }
      if (!ok) codes = careful_row(x, sc, row_fast, scheme, sat);  // may saturate, or out of range
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(side ? p.v_codes : p.k_codes) + row * kHeadDim + lane8 * 8) = codes;
      if (scheme == KVQ_INT8_SYM_PER_TOKEN && lane8 == 0) scale[row] = tok_s;
    }
  }
  if (sat && p.status) atomicAdd(p.status + 1, (uint32_t)sat);
}

// ------------------------------------------------------------------ rescaling append
// Merge each block's scales into the cached ones (n4n.ai Step 3 keeps a running maximum;
// Step 7 wants scales that only grow, or are recomputed as the cache grows) and requantize
// the cached codes whose scale element changed. Symmetric schemes: s' = max(s, s_block).
// uint8 asymmetric: the parameters of the union of the range the cached (s, zp) represent,
// [(0 - zp) s, (255 - zp) s], and the block's range (with 0), unchanged when it lies inside.
// Workspace after the calibration keys: old scales [2][H*D] fp32, old zero points
// [2][H*D] uint8, and one changed flag per side.
struct RescaleWs {
  float* s_old;
  uint8_t* zp_old;
  uint32_t* changed;
};

__global__ void rescale_finalize_kernel(AppendParams p, const uint32_t* keys, RescaleWs ws) {
  const int hd = p.H * kHeadDim;
  __shared__ uint32_t grew[2];
  if (threadIdx.x < 2) grew[threadIdx.x] = 0u;
  __syncthreads();
  for (int side = 0; side < 2; ++side) {
    const int scheme = side ? p.v_scheme : p.k_scheme;
    float* scale = side ? p.v_scale : p.k_scale;
    uint8_t* zp = side ? p.v_zp : p.k_zp;
    const uint32_t* base = keys + 2 + side * 2 * hd;
    float* s_old = ws.s_old + side * hd;
    uint8_t* z_old = ws.zp_old + side * hd;
    if (scheme == KVQ_FP8_E4M3_PER_TENSOR || scheme == KVQ_FP8_E5M2_PER_TENSOR || scheme == KVQ_INT8_SYM_PER_TENSOR) {
      if (threadIdx.x == 0) {
        const float so = scale[0], sb = calib_scale(scheme, __uint_as_float(keys[side]));
        s_old[0] = so;
        z_old[0] = 0;
        if (sb > so) {
          scale[0] = sb;
          grew[side] = 1u;
        }
      }
    } else if (scheme == KVQ_INT8_SYM_PER_CHANNEL) {
      for (int i = threadIdx.x; i < hd; i += blockDim.x) {
        const float so = scale[i], sb = __fdiv_rn(__uint_as_float(base[hd + i]), 127.0f);
        s_old[i] = so;
        z_old[i] = 0;
        if (sb > so) {
          scale[i] = sb;
          grew[side] = 1u;
        }
      }
    } else if (scheme == KVQ_UINT8_ASYM_PER_CHANNEL) {
      for (int i = threadIdx.x; i < hd; i += blockDim.x) {
        const float so = scale[i];
        const uint8_t zo = zp[i];
        s_old[i] = so;
        z_old[i] = zo;
        const float mn = key_to_float(base[i]), mx = key_to_float(base[hd + i]);
        const float lo_b = mn < 0.0f ? mn : 0.0f, hi_b = mx > 0.0f ? mx : 0.0f;
        const float lo_o = __fmul_rn((float)(0 - (int)zo), so), hi_o = __fmul_rn((float)(255 - (int)zo), so);
        if (lo_b < lo_o || hi_b > hi_o) {
          asym_params(lo_b < lo_o ? lo_b : lo_o, hi_b > hi_o ? hi_b : hi_o, scale[i], zp[i]);
          grew[side] = 1u;
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < 2) ws.changed[threadIdx.x] = grew[threadIdx.x];
}

// Value of an 8-bit code of a batch-wide scheme under (s, zp).
template <int SCHEME>
__device__ __forceinline__ float fixed_value(uint32_t q, float s, int zp) {
  if constexpr (SCHEME == KVQ_FP8_E4M3_PER_TENSOR) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
    return __fmul_rn(__half2float(__half(hr)), s);
  } else if constexpr (SCHEME == KVQ_FP8_E5M2_PER_TENSOR) {
    __half_raw hr;
    hr.x = (unsigned short)(q << 8);
    return __fmul_rn(__half2float(__half(hr)), s);
  } else if constexpr (SCHEME == KVQ_UINT8_ASYM_PER_CHANNEL) {
    return __fmul_rn((float)((int)q - zp), s);
  } else {
    return __fmul_rn((float)(int8_t)q, s);
  }
}

// Requantize the cached rows of one side (blockIdx.y = kv head) when its scales changed:
// 8 threads per 128-code row, 16 codes each; the thread's 16 channels keep their old and
// new parameters in registers across the rows it visits.
template <int SCHEME>
__global__ void __launch_bounds__(256) requant_kernel(AppendParams p, RescaleWs ws, int side) {
  if (ws.changed[side] == 0u) return;
  constexpr bool kPerChannel = SCHEME == KVQ_INT8_SYM_PER_CHANNEL || SCHEME == KVQ_UINT8_ASYM_PER_CHANNEL;
  const int h = blockIdx.y, lane8 = threadIdx.x & 7;
  const int hd = p.H * kHeadDim;
  const float* scale = side ? p.v_scale : p.k_scale;
  const uint8_t* zp = side ? p.v_zp : p.k_zp;
  uint8_t* codes = static_cast<uint8_t*>(side ? p.v_codes : p.k_codes);
  float so[16], sn[16], yn[16];
  int zo[16], zn[16];
  uint32_t keep = 0u, fast = 0u;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int i = kPerChannel ? h * kHeadDim + lane8 * 16 + k : 0;
    so[k] = ws.s_old[side * hd + i];
    sn[k] = scale[i];
    yn[k] = __frcp_rn(sn[k]);
    zo[k] = SCHEME == KVQ_UINT8_ASYM_PER_CHANNEL ? (int)ws.zp_old[side * hd + i] : 0;
    zn[k] = SCHEME == KVQ_UINT8_ASYM_PER_CHANNEL ? (int)zp[i] : 0;
    if (sn[k] == so[k] && zn[k] == zo[k]) keep |= 1u << k;
    if (quot_range(sn[k]) && quot_range(so[k])) fast |= 1u << k;
  }
  // FP8 per-tensor with both scales in the quotient's range: two codes per packed operation
  constexpr bool kFp8 = SCHEME == KVQ_FP8_E4M3_PER_TENSOR || SCHEME == KVQ_FP8_E5M2_PER_TENSOR;
  const bool packed = kFp8 && keep == 0u && fast == 0xFFFFu;
  // (the residual is formed as q s - x and subtracted, as in quot, so a zero keeps its sign)
  const f32x2 so2 = pk2(so[0], so[0]), nso2 = pk2(-so[0], -so[0]), sn2 = pk2(sn[0], sn[0]);
  const f32x2 y2 = pk2(yn[0], yn[0]), ny2 = pk2(-yn[0], -yn[0]);
  const int span = p.paged ? p.max_pages * p.page_size : p.pos0;
  const long long rows = (long long)p.B * span;
  const bool rows32 = rows < (1LL << 31);  // row index and its (sequence, position) in 32 bits
  for (long long r = (long long)blockIdx.x * 32 + (threadIdx.x >> 3); r < rows; r += (long long)gridDim.x * 32) {
    int b, pos;
    if (rows32) {
      b = (int)((unsigned)r / (unsigned)span);
      pos = (int)r - b * span;
    } else {
      b = (int)(r / span);
      pos = (int)(r % span);
    }
    if (p.paged && pos >= p.seq_lens[b]) continue;
    size_t row;
    if (!cache_row(p, b, h, pos, row)) continue;
    uint4* ptr = reinterpret_cast<uint4*>(codes + row * kHeadDim + lane8 * 16);
    const uint4 in = *ptr;
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    if constexpr (kFp8) {
      if (packed) {  // per code the same operations as below: x = v * s_old, z = x / s_new, RN code
        uint32_t o2[4];
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          uint32_t half_codes[2];
#pragma unroll
          for (int hp = 0; hp < 2; ++hp) {
            uint32_t h2;  // the two codes' values as f16x2 (exact), lower code in the low half
            if constexpr (SCHEME == KVQ_FP8_E4M3_PER_TENSOR) {
              asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(w[wi] >> (16 * hp))));
            } else {
              h2 = prmt(w[wi], 0u, hp ? 0x3424u : 0x1404u);
            }
            float v0, v1;
            asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n cvt.f32.f16 %0, l;\n cvt.f32.f16 %1, h;\n}\n"
                : "=f"(v0), "=f"(v1)
                : "r"(h2));
            const f32x2 v2 = pk2(v0, v1);
            const f32x2 x2 = mul2(v2, so2), nx2 = mul2(v2, nso2);  // x and -x, both exact negations
            const f32x2 q2 = mul2(x2, y2);
            const f32x2 z2 = fma2(fma2(q2, sn2, nx2), ny2, q2);  // q - RN(q s - x) y
            float z0, z1;
            upk2(z2, z0, z1);
            half_codes[hp] = SCHEME == KVQ_FP8_E4M3_PER_TENSOR ? e4m3x2_rn(z0, z1) : e5m2x2_rn(z0, z1);
          }
          o2[wi] = half_codes[0] | (half_codes[1] << 16);
        }
        *ptr = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        continue;
      }
    }
    uint32_t o[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t q = (w[k >> 2] >> (8 * (k & 3))) & 0xFFu;
      uint32_t c = q;
      if (!((keep >> k) & 1u)) {
        c = 0u;
        if (sn[k] != 0.0f) {
          const float x = fixed_value<SCHEME>(q, so[k], zo[k]);
          float qq;
          const float z = ((fast >> k) & 1u) ? quot(x, sn[k], yn[k], qq) : __fdiv_rn(x, sn[k]);
          int sat = 0;
          c = code_of(z, zn[k], SCHEME, sat);
        }
      }
      o[k >> 2] |= c << (8 * (k & 3));
    }
    *ptr = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

template <int SCHEME>
void launch_requant(const AppendParams& p, const RescaleWs& ws, int side, cudaStream_t st) {
  const long long span = p.paged ? (long long)p.max_pages * p.page_size : p.pos0;
  const long long chunks = ((long long)p.B * span + 31) / 32;
  if (chunks == 0) return;
  const long long cap = std::max(1LL, 16LL * sm_count() / p.H);
  dim3 grid((unsigned)std::min(chunks, cap), p.H);
  requant_kernel<SCHEME><<<grid, 256, 0, st>>>(p, ws, side);
  count_launches(1);
}

void launch_requant_side(const AppendParams& p, const RescaleWs& ws, int side, cudaStream_t st) {
  switch (side ? p.v_scheme : p.k_scheme) {
    case KVQ_FP8_E4M3_PER_TENSOR: launch_requant<KVQ_FP8_E4M3_PER_TENSOR>(p, ws, side, st); break;
    case KVQ_FP8_E5M2_PER_TENSOR: launch_requant<KVQ_FP8_E5M2_PER_TENSOR>(p, ws, side, st); break;
    case KVQ_INT8_SYM_PER_TENSOR: launch_requant<KVQ_INT8_SYM_PER_TENSOR>(p, ws, side, st); break;
    case KVQ_INT8_SYM_PER_CHANNEL: launch_requant<KVQ_INT8_SYM_PER_CHANNEL>(p, ws, side, st); break;
    case KVQ_UINT8_ASYM_PER_CHANNEL: launch_requant<KVQ_UINT8_ASYM_PER_CHANNEL>(p, ws, side, st); break;
    default: break;  // per-token scales: nothing to merge
  }
}


// A sequence's length grows by its new tokens only when every page they land on is a page of
// the pool: an append that met a bad page or ran past the page table (flagged by the store) is
// refused for that sequence, which keeps its length and so never shows rows that were not
// written. The rows the store did write past the kept length stay invisible to decode.
__global__ void seq_lens_advance_kernel(AppendParams p) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= p.B) return;
  const int n = new_count(p, b);
  if (n == 0) return;
  const int L = p.seq_lens[b];
  const long long last = (long long)L + n - 1;
  bool ok = L >= 0 && last / p.page_size < p.max_pages;
  for (int pi = L / p.page_size; ok && pi <= (int)(last / p.page_size); ++pi) {
    const int page = p.page_table[(size_t)b * p.max_pages + pi];
    ok = page >= 0 && page < p.num_pages;
  }
  if (ok)
    p.seq_lens[b] = L + n;
  else
    flag(p.status, L < 0 || last / p.page_size >= p.max_pages ? KVQ_DEV_BAD_LENGTH : KVQ_DEV_BAD_PAGE);
}

// ------------------------------------------------------------------ KIVI
// Lane-wise minimum / maximum of two bf16 pairs (exact: a selection; a NaN lane yields the
// other operand, as fminf / fmaxf do).
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}


// clamp(rne(z), 0, qmax) for any finite quotient z (the stored fp16 minimum may lie above a
// value, and a saturated or underflowing fp16 scale may make z large): z is first bounded to
// [-1, qmax + 1], where RN(z + 1.5 * 2^23) holds rne(z) in its low bits, then the code clamped.
template <int kQmax>
__device__ __forceinline__ uint32_t signed_code(float z) {
  z = fminf(fmaxf(z, -1.0f), (float)kQmax + 1.0f);
  const int c = (int)(__float_as_uint(__fadd_rn(z, kRoundMagic)) - (uint32_t)kRoundMagicBits);
  return (uint32_t)(c < 0 ? 0 : (c > kQmax ? kQmax : c));
}

// Two KIVI codes at once: d = RN(v - min), then the division-free quotient of `quot` in its
// residual form r = RN(d - q * s) (the same values; zero signs do not reach integer codes),
// then rne. v2 holds the two values; lo2, s2, ns2 (= -s), y2 (= RN(1/s)) the lanes' group terms.
// kSigned: the minimum is the stored fp16 one, so d may be negative (or the quotient large).
template <int kQmax, bool kSigned = false>
__device__ __forceinline__ void kivi_code2(f32x2 v2, f32x2 lo2, f32x2 s2n, f32x2 y2, uint32_t& c0, uint32_t& c1) {
  const f32x2 d = sub2(v2, lo2);
  const f32x2 q = mul2(d, y2);
  const f32x2 r = fma2(q, s2n, d);
  if constexpr (kSigned) {
    float z0, z1;
    upk2(fma2(r, y2, q), z0, z1);
    c0 = signed_code<kQmax>(z0);
    c1 = signed_code<kQmax>(z1);
    return;
  }
  const f32x2 t = add2(fma2(r, y2, q), pk2(kRoundMagic, kRoundMagic));
  float t0, t1;
  upk2(t, t0, t1);
  c0 = __float_as_uint(t0) - (uint32_t)kRoundMagicBits;
  c1 = __float_as_uint(t1) - (uint32_t)kRoundMagicBits;
  c0 = c0 < (uint32_t)kQmax ? c0 : (uint32_t)kQmax;
  c1 = c1 < (uint32_t)kQmax ? c1 : (uint32_t)kQmax;
}

// Code of d = RN(x - min) with step s: rne(RN(d / s)); with the exact fp32 minimum d >= 0 and
// d <= max - min keeps it in [0, qmax]; with the stored fp16 minimum it is clamped (kSigned).
template <int kQmax, bool kSigned = false>
__device__ __forceinline__ uint32_t kivi_code(float d, float s, float y, bool fast) {
  float q;
  const float z = fast ? quot(d, s, y, q) : __fdiv_rn(d, s);
  if constexpr (kSigned) return signed_code<kQmax>(z);
  const uint32_t c = __float_as_uint(__fadd_rn(z, kRoundMagic)) - (uint32_t)kRoundMagicBits;
  return c < (uint32_t)kQmax ? c : (uint32_t)kQmax;
}

// fp16 storage of a KIVI scale or minimum: nearest-even, saturating at +-65504 (the value must
// stay finite); returns the stored bits and the stored value as fp32 (exact).
__device__ __forceinline__ uint32_t f16_store(float x, float& stored) {
  const __half h = __float2half_rn(fminf(fmaxf(x, -65504.0f), 65504.0f));
  stored = __half2float(h);
  return (uint32_t)__half_as_ushort(h);
}

// One block per (R-token chunk, b*H + h): quantize R consecutive tokens of the combined
// stream (old residual tokens, then the new block) into the cache at pos0 + chunk*R.
// kF16: scales and minima stored as fp16 (KIVI_INT4_F16 / KIVI_INT2_F16), codes from the stored
// values.
template <int kBits, bool kF16>
__global__ void __launch_bounds__(256, 3) kivi_flush_kernel(AppendParams p, int r_old) {
  constexpr int R = 128, G = 32, kQmax = (1 << kBits) - 1, kPer = 8 / kBits;
  constexpr int kRowBytes = kHeadDim * kBits / 8;
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* xk = reinterpret_cast<uint16_t*>(smem);           // [R][D] bf16
  uint16_t* xv = xk + R * kHeadDim;                            // [R][D] bf16
  uint8_t* kcodes = reinterpret_cast<uint8_t*>(xv + R * kHeadDim);  // [R][row bytes]
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int pos0 = p.pos0 + chunk * R;
  // gather the combined stream (old residual rows, then new rows: at most two contiguous runs
  // of 256-byte rows per side) with the bulk copy engine; completion on one mbarrier
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = smem_addr(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int s0 = chunk * R;
    const int nres = min(max(r_old - s0, 0), R);  // rows taken from the residual
    const size_t bhs = (size_t)b * p.H + h;
    mbar_arrive_expect_tx(bar, 2u * R * kHeadDim * 2u);
    if (nres > 0) {
      const size_t o = (bhs * p.rcap + s0) * kHeadDim;
      bulk_g2s(smem_addr(xk), p.k_res + o, (uint32_t)nres * kHeadDim * 2u, bar);
      bulk_g2s(smem_addr(xv), p.v_res + o, (uint32_t)nres * kHeadDim * 2u, bar);
    }
    if (nres < R) {
      const size_t o = (bhs * (size_t)p.n_new + (size_t)(s0 + nres - r_old)) * kHeadDim;
      bulk_g2s(smem_addr(xk + nres * kHeadDim), static_cast<const uint16_t*>(p.k_new) + o,
               (uint32_t)(R - nres) * kHeadDim * 2u, bar);
      bulk_g2s(smem_addr(xv + nres * kHeadDim), static_cast<const uint16_t*>(p.v_new) + o,
               (uint32_t)(R - nres) * kHeadDim * 2u, bar);
    }
  }
  if (!mbar_wait(bar, 0, p.status)) {
    mbar_wait(bar, 0, p.status);  // give copies still in flight a second bounded wait, then leave
    return;
  }
  // keys: task = (group gi, 2 adjacent channels); the thread keeps the 32 tokens' 4-byte
  // words (both channels as bf16) in registers and widens a channel when it needs it. The
  // codes of token j sit in byte j % 4 of word j / 4; with 2-bit codes a byte holds 4
  // channels and the two threads of neighbouring tasks combine their halves.
  constexpr int kKTasks = (R / G) * (kHeadDim / 2);  // 256
  static_assert(kKTasks == 256, "one key task per thread");
  {
    const int task = threadIdx.x;
    const int gi = task / (kHeadDim / 2), c0 = (task % (kHeadDim / 2)) * 2;
    uint32_t raw[G];
#pragma unroll
    for (int j = 0; j < G; ++j) raw[j] = *reinterpret_cast<const uint32_t*>(xk + (gi * G + j) * kHeadDim + c0);
    uint32_t bits[G / 4];
#pragma unroll
    for (int j = 0; j < G / 4; ++j) bits[j] = 0u;
    const size_t meta = (((size_t)b * p.H + h) * (size_t)(p.cap / G) + (size_t)(pos0 / G + gi)) * kHeadDim;
    const int shift0 = (c0 % kPer) * kBits;  // position of channel c0 inside its byte
    uint32_t mn2 = raw[0], mx2 = raw[0];  // both channels at once
#pragma unroll
    for (int j = 1; j < G; ++j) {
      mn2 = bmin2(mn2, raw[j]);
      mx2 = bmax2(mx2, raw[j]);
    }
    float lo[2], sc[2], yr[2];
    bool fast[2];
    uint32_t s16[2], m16[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      lo[k] = __uint_as_float(k ? (mn2 & 0xFFFF0000u) : (mn2 << 16));
      float hi = __uint_as_float(k ? (mx2 & 0xFFFF0000u) : (mx2 << 16));
      if (lo[k] == 0.0f) lo[k] = 0.0f;
      if (hi == 0.0f) hi = 0.0f;
      sc[k] = __fdiv_rn(__fsub_rn(hi, lo[k]), (float)kQmax);
      if constexpr (kF16) {  // the stored values take over
        s16[k] = f16_store(sc[k], sc[k]);
        m16[k] = f16_store(lo[k], lo[k]);
      } else {
        p.k_scale[meta + c0 + k] = sc[k];
        p.k_zero[meta + c0 + k] = lo[k];
      }
      yr[k] = __frcp_rn(sc[k]);
      fast[k] = sc[k] != 0.0f && quot_range(sc[k]);
    }
    if constexpr (kF16) {  // channels c0, c0 + 1: one 32-bit word of halves per array
      *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.k_scale) + meta + c0) = s16[0] | (s16[1] << 16);
      *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.k_zero) + meta + c0) = m16[0] | (m16[1] << 16);
    }
    if (fast[0] && fast[1]) {
      // both channels of a token in one packed operation
      const f32x2 lo2 = pk2(lo[0], lo[1]), s2n = pk2(-sc[0], -sc[1]), y2 = pk2(yr[0], yr[1]);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        uint32_t a, bb;
        kivi_code2<kQmax, kF16>(pk2(__uint_as_float(raw[j] << 16), __uint_as_float(raw[j] & 0xFFFF0000u)), lo2, s2n,
                                y2, a, bb);
        bits[j / 4] |= (a << (8 * (j % 4) + shift0)) | (bb << (8 * (j % 4) + shift0 + kBits));
      }
    } else {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (sc[k] == 0.0f) continue;
        auto val = [&](int j) { return __uint_as_float(k ? (raw[j] & 0xFFFF0000u) : (raw[j] << 16)); };
#pragma unroll
        for (int j = 0; j < G; ++j)
          bits[j / 4] |= kivi_code<kQmax, kF16>(__fsub_rn(val(j), lo[k]), sc[k], yr[k], fast[k])
                         << (8 * (j % 4) + shift0 + k * kBits);
      }
    }
#pragma unroll
    for (int w = 0; w < G / 4; ++w) {
      uint32_t word = bits[w];
      if constexpr (kBits == 2) word |= __shfl_xor_sync(0xffffffffu, word, 1);
      if (kBits == 4 || (c0 % kPer) == 0) {
#pragma unroll
        for (int t = 0; t < 4; ++t) kcodes[(gi * G + 4 * w + t) * kRowBytes + c0 / kPer] = (uint8_t)(word >> (8 * t));
      }
    }
  }
  // values: task = (token, channel group); 32 channels = four 16-byte shared loads
  for (int task = threadIdx.x; task < R * (kHeadDim / G); task += blockDim.x) {
    const int tok = task / (kHeadDim / G), j = task % (kHeadDim / G);
    const uint4* row = reinterpret_cast<const uint4*>(xv + tok * kHeadDim + j * G);
    uint32_t raw[G / 2];
#pragma unroll
    for (int q4 = 0; q4 < G / 8; ++q4) {
      const uint4 w = row[q4];
      raw[4 * q4] = w.x;
      raw[4 * q4 + 1] = w.y;
      raw[4 * q4 + 2] = w.z;
      raw[4 * q4 + 3] = w.w;
    }
    auto val = [&](int i) { return __uint_as_float((i & 1) ? (raw[i >> 1] & 0xFFFF0000u) : (raw[i >> 1] << 16)); };
    uint32_t mn2 = raw[0], mx2 = raw[0];
#pragma unroll
    for (int i = 1; i < G / 2; ++i) {
      mn2 = bmin2(mn2, raw[i]);
      mx2 = bmax2(mx2, raw[i]);
    }
    float lo = fminf(__uint_as_float(mn2 << 16), __uint_as_float(mn2 & 0xFFFF0000u));
    float hi = fmaxf(__uint_as_float(mx2 << 16), __uint_as_float(mx2 & 0xFFFF0000u));
    if (lo == 0.0f) lo = 0.0f;
    if (hi == 0.0f) hi = 0.0f;
    float sc = __fdiv_rn(__fsub_rn(hi, lo), (float)kQmax);
    uint32_t s16 = 0u, m16 = 0u;
    if constexpr (kF16) {  // the stored values take over
      s16 = f16_store(sc, sc);
      m16 = f16_store(lo, lo);
    }
    uint32_t words[G * kBits / 32];
#pragma unroll
    for (int w = 0; w < G * kBits / 32; ++w) words[w] = 0u;
    if (sc != 0.0f) {
      const float y = __frcp_rn(sc);
      if (quot_range(sc)) {
        // channel pairs (2i, 2i + 1) in one packed operation
        const f32x2 lo2 = pk2(lo, lo), s2n = pk2(-sc, -sc), y2 = pk2(y, y);
#pragma unroll
        for (int i = 0; i < G / 2; ++i) {
          uint32_t a, bb;
          kivi_code2<kQmax, kF16>(pk2(__uint_as_float(raw[i] << 16), __uint_as_float(raw[i] & 0xFFFF0000u)), lo2, s2n,
                                  y2, a, bb);
          words[(2 * i * kBits) / 32] |= (a << ((2 * i * kBits) % 32)) | (bb << ((2 * i * kBits) % 32 + kBits));
        }
      } else {
#pragma unroll
        for (int i = 0; i < G; ++i)
          words[(i * kBits) / 32] |= kivi_code<kQmax, kF16>(__fsub_rn(val(i), lo), sc, y, false) << ((i * kBits) % 32);
      }
    }
    const size_t crow = ((size_t)b * p.H + h) * (size_t)p.cap + (size_t)(pos0 + tok);
    uint8_t* dst = static_cast<uint8_t*>(p.v_codes) + crow * kRowBytes + j * (G * kBits / 8);
    if constexpr (kBits == 4) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
    } else {
      *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
    }
    if constexpr (kF16) {
      reinterpret_cast<uint16_t*>(p.v_scale)[crow * (kHeadDim / G) + j] = (uint16_t)s16;
      reinterpret_cast<uint16_t*>(p.v_zero)[crow * (kHeadDim / G) + j] = (uint16_t)m16;
    } else {
      p.v_scale[crow * (kHeadDim / G) + j] = sc;
      p.v_zero[crow * (kHeadDim / G) + j] = lo;
    }
  }
  __syncthreads();
  // key codes: R rows x kRowBytes, contiguous in the cache
  uint8_t* kdst = static_cast<uint8_t*>(p.k_codes) + (((size_t)b * p.H + h) * (size_t)p.cap + pos0) * kRowBytes;
  for (int e = threadIdx.x; e < R * kRowBytes / 16; e += blockDim.x)
    reinterpret_cast<uint4*>(kdst)[e] = reinterpret_cast<const uint4*>(kcodes)[e];
}

// Copy `count` new tokens (input rows src0..) into residual slots dst0.. for every (b, h).
__global__ void kivi_residual_kernel(AppendParams p, int src0, int dst0, int count) {
  const long long total = (long long)p.B * p.H * count * 16;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int piece = (int)(e & 15);
    const long long rr = e >> 4;
    const int i = (int)(rr % count);
    const long long bh = rr / count;
    const size_t src = ((size_t)bh * p.n_new + src0 + i) * kHeadDim;
    const size_t dst = ((size_t)bh * p.rcap + dst0 + i) * kHeadDim;
    reinterpret_cast<uint4*>(p.k_res + dst)[piece] =
        reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.k_new) + src)[piece];
    reinterpret_cast<uint4*>(p.v_res + dst)[piece] =
        reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.v_new) + src)[piece];
  }
}

// ------------------------------------------------------------------ dequantize
// out [B, H, T_out, D]; one thread per 8 channels of one row.
__global__ void __launch_bounds__(256) dequantize_kernel(DequantParams p) {
  const long long rows = (long long)p.B * p.H * p.T_out;
  const long long r = (long long)blockIdx.x * 16 + (threadIdx.x >> 4);
  if (r >= rows) return;
  const int lane8 = threadIdx.x & 15;
  const int t = (int)(r % p.T_out);
  const int h = (int)((r / p.T_out) % p.H);
  const int b = (int)(r / ((long long)p.T_out * p.H));
  float y[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const int scheme = p.scheme;
  const int len = p.paged ? p.seq_lens[b] : p.len_q + (is_kivi(scheme) ? p.len_res : 0);
  if (t < len) {
    if (is_kivi(scheme) && t >= p.len_q) {
      const uint16_t* res = p.res + (((size_t)b * p.H + h) * p.rcap + (t - p.len_q)) * kHeadDim + lane8 * 8;
#pragma unroll
      for (int k = 0; k < 8; ++k) y[k] = bf16_bits_to_float(res[k]);
    } else {
      size_t row;
      bool ok = true;
      if (!p.paged) {
        row = ((size_t)b * p.H + h) * (size_t)p.cap + t;
      } else {
        const int pi = t / p.page_size;
        const int page = pi < p.max_pages ? p.page_table[(size_t)b * p.max_pages + pi] : -1;
        ok = page >= 0 && page < p.num_pages;
        if (!ok) flag(p.status, KVQ_DEV_BAD_PAGE);
        row = ((size_t)page * p.H + h) * (size_t)p.page_size + (t % p.page_size);
      }
      if (ok) {
        const int bits = code_bits(scheme);
        const uint8_t* codes = p.codes + row * (size_t)row_bytes(scheme);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int d = lane8 * 8 + k;
          int q;
          if (bits == 8) {
            q = codes[d];
          } else {
            const int per = 8 / bits;
            q = (codes[d / per] >> ((d % per) * bits)) & ((1 << bits) - 1);
          }
          float v = 0.0f;
          switch (scheme) {
            case KVQ_FP8_E4M3_PER_TENSOR: {
              const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
              v = __fmul_rn(__half2float(__half(hr)), p.scale[0]);
              break;
            }
            case KVQ_FP8_E5M2_PER_TENSOR: {  // an E5M2 byte is the high byte of the same-valued f16
              __half_raw hr;
              hr.x = (unsigned short)(q << 8);
              v = __fmul_rn(__half2float(__half(hr)), p.scale[0]);
              break;
            }
            case KVQ_INT8_SYM_PER_TENSOR: v = __fmul_rn((float)(int8_t)q, p.scale[0]); break;
            case KVQ_INT8_SYM_PER_TOKEN: v = __fmul_rn((float)(int8_t)q, p.scale[row]); break;
            case KVQ_INT8_SYM_PER_CHANNEL: v = __fmul_rn((float)(int8_t)q, p.scale[h * kHeadDim + d]); break;
            case KVQ_UINT8_ASYM_PER_CHANNEL:
              v = __fmul_rn((float)(q - (int)p.zp[h * kHeadDim + d]), p.scale[h * kHeadDim + d]);
              break;
            case KVQ_INT4_SYM_PER_GROUP:
              v = __fmul_rn((float)(q >= 8 ? q - 16 : q), p.scale[row * (kHeadDim / p.group) + d / p.group]);
              break;
            default: {  // KIVI: fl(fl(q * s) + min), s and min as stored (fp32 or fp16)
              size_t m;
              if (p.which == 0)
                m = (((size_t)b * p.H + h) * (size_t)(p.cap / 32) + (size_t)(t / 32)) * kHeadDim + d;
              else
                m = row * (kHeadDim / 32) + d / 32;
              float sm, mn;
              if (kivi_f16(scheme)) {
                sm = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(p.scale)[m]));
                mn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(p.zero)[m]));
              } else {
                sm = p.scale[m];
                mn = p.zero[m];
              }
              v = __fadd_rn(__fmul_rn((float)q, sm), mn);
            }
          }
          y[k] = v;
        }
      }
    }
  }
  if (p.rotate) fwht_row16(y, 0xFFFFu << (threadIdx.x & 16), lane8);  // back from the rotated domain
  float4* o = reinterpret_cast<float4*>(p.out + (size_t)r * kHeadDim + lane8 * 8);
  o[0] = make_float4(y[0], y[1], y[2], y[3]);
  o[1] = make_float4(y[4], y[5], y[6], y[7]);
}

// ------------------------------------------------------------------ launchers
// Streaming multiprocessors of the current device, queried once per device ordinal (devices
// past the cache are queried on every call).
int sm_count() {
  constexpr int kCached = 64;
  static std::atomic<int> cached[kCached];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = (dev >= 0 && dev < kCached) ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    if (dev >= 0 && dev < kCached) cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int KS, int VS>
cudaError_t launch_quantize_rows_pair(const AppendParams& p, long long rows, cudaStream_t st) {
  // several rows per thread once every (batch, kv head) row has enough new tokens: four of
  // bf16, two of fp32 (the same bytes in flight per thread); a grid of a few waves of the SMs
  // walks the (chunk, sequence x head) items
  if (p.n_new >= 64 && rows >= 16LL * 4 * 148 * 8 && p.B * p.H <= 65535) {
    const int per_item = p.in_bf16 ? 64 : 32;
    const long long items = (long long)((p.n_new + per_item - 1) / per_item) * p.B * p.H;
    const long long cap = 16LL * sm_count();
    dim3 grid((unsigned)(items < cap ? items : cap), 1, 2);
    if (p.in_bf16) return launch_pdl(quantize_rows_kernel<true, 4, KS, VS>, grid, dim3(256), 0, st, p);
    return launch_pdl(quantize_rows_kernel<false, 2, KS, VS>, grid, dim3(256), 0, st, p);
  }
  dim3 grid((unsigned)((rows + 15) / 16), 1, 2);
  if (p.in_bf16) return launch_pdl(quantize_rows_kernel<true, 1, KS, VS>, grid, dim3(256), 0, st, p);
  return launch_pdl(quantize_rows_kernel<false, 1, KS, VS>, grid, dim3(256), 0, st, p);
}

bool append_pair_supported(int ks, int vs) {
  if (is_kivi(ks) || is_kivi(vs)) return ks == vs;
  constexpr int F = KVQ_FP8_E4M3_PER_TENSOR, T = KVQ_INT8_SYM_PER_TENSOR, K = KVQ_INT8_SYM_PER_TOKEN,
                C = KVQ_INT8_SYM_PER_CHANNEL, U = KVQ_UINT8_ASYM_PER_CHANNEL;
  constexpr int E = KVQ_FP8_E5M2_PER_TENSOR, G = KVQ_INT4_SYM_PER_GROUP;
  const int pairs[][2] = {{F, F}, {T, T}, {K, K}, {C, C}, {U, U}, {T, U}, {C, U}, {K, U}, {T, K}, {F, T}, {T, F},
                          {E, E}, {G, G}};
  for (const auto& pr : pairs)
    if (pr[0] == ks && pr[1] == vs) return true;
  return false;
}

cudaError_t launch_quantize_rows(const AppendParams& p, long long rows, cudaStream_t st) {
  constexpr int F = KVQ_FP8_E4M3_PER_TENSOR, T = KVQ_INT8_SYM_PER_TENSOR, K = KVQ_INT8_SYM_PER_TOKEN,
                C = KVQ_INT8_SYM_PER_CHANNEL, U = KVQ_UINT8_ASYM_PER_CHANNEL;
  const int ks = p.k_scheme, vs = p.v_scheme;
#define KVQ_PAIR(A, B) \
  if (ks == A && vs == B) return launch_quantize_rows_pair<A, B>(p, rows, st);
  KVQ_PAIR(F, F) KVQ_PAIR(T, T) KVQ_PAIR(K, K) KVQ_PAIR(C, C) KVQ_PAIR(U, U)
  KVQ_PAIR(T, U) KVQ_PAIR(C, U) KVQ_PAIR(K, U) KVQ_PAIR(T, K) KVQ_PAIR(F, T) KVQ_PAIR(T, F)
  constexpr int E = KVQ_FP8_E5M2_PER_TENSOR, G = KVQ_INT4_SYM_PER_GROUP;
  KVQ_PAIR(E, E) KVQ_PAIR(G, G)
#undef KVQ_PAIR
  return cudaErrorNotSupported;
}

size_t rescale_ws_offset(int H) { return ((2 + 4 * (size_t)H * kHeadDim) * sizeof(uint32_t) + 255) & ~(size_t)255; }

cudaError_t launch_append(const AppendParams& p, void* workspace, int mode, int r_old, int flushed, int r_new,
                          cudaStream_t st) {
  uint32_t* calib_keys = static_cast<uint32_t*>(workspace);
  const bool kivi = is_kivi(p.k_scheme);
  if (kivi) {
    if (flushed > 0) {
      const int bits = code_bits(p.k_scheme);
      const size_t smem = 2 * 128 * kHeadDim * 2 + 128 * (kHeadDim * bits / 8);
      dim3 grid(flushed / 128, p.B * p.H);
      void (*kern)(AppendParams, int) =
          kivi_f16(p.k_scheme) ? (bits == 4 ? kivi_flush_kernel<4, true> : kivi_flush_kernel<2, true>)
                               : (bits == 4 ? kivi_flush_kernel<4, false> : kivi_flush_kernel<2, false>);
      const cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (ea != cudaSuccess) return ea;
      kern<<<grid, 256, smem, st>>>(p, r_old);
      count_launches(1);
    }
    // residual update: only new tokens ever move into it
    const int count = flushed > 0 ? r_new : p.n_new;
    const int src0 = flushed > 0 ? p.n_new - r_new : 0;
    const int dst0 = flushed > 0 ? 0 : r_old;
    if (count > 0) {
      const long long pieces = (long long)p.B * p.H * count * 16;
      const long long want = (pieces + 255) / 256;
      const int blocks = (int)(want < 65535 ? want : 65535);
      kivi_residual_kernel<<<blocks, 256, 0, st>>>(p, src0, dst0, count);
      count_launches(1);
    }
    return cudaGetLastError();
  }
  if (mode != kAppendPlain) {
    const int hd = p.H * kHeadDim;
    calib_init_kernel<<<(2 + 4 * hd + 255) / 256, 256, 0, st>>>(calib_keys, hd);
    dim3 grid((p.n_new + 255) / 256, p.B * p.H, 2);
    if (p.in_bf16)
      calib_reduce_kernel<true><<<grid, 256, 0, st>>>(p, calib_keys);
    else
      calib_reduce_kernel<false><<<grid, 256, 0, st>>>(p, calib_keys);
    count_launches(2);
    if (mode == kAppendCalibrate) {
      calib_finalize_kernel<<<1, 256, 0, st>>>(p, calib_keys);
      count_launches(1);
    } else {
      uint8_t* w = static_cast<uint8_t*>(workspace) + rescale_ws_offset(p.H);
      RescaleWs ws;
      ws.s_old = reinterpret_cast<float*>(w);
      ws.zp_old = w + 2 * (size_t)hd * sizeof(float);
      ws.changed = reinterpret_cast<uint32_t*>(w + 2 * (size_t)hd * (sizeof(float) + 1));
      rescale_finalize_kernel<<<1, 256, 0, st>>>(p, calib_keys, ws);
      count_launches(1);
      launch_requant_side(p, ws, 0, st);
      launch_requant_side(p, ws, 1, st);
    }
  }
  const long long rows = (long long)p.B * p.H * p.n_new;
  const cudaError_t e = launch_quantize_rows(p, rows, st);
  if (e != cudaSuccess) return e;
  count_launches(1);
  if (p.paged) {
    seq_lens_advance_kernel<<<(p.B + 255) / 256, 256, 0, st>>>(p);
    count_launches(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const DequantParams& p, cudaStream_t st) {
  const long long rows = (long long)p.B * p.H * p.T_out;
  if (rows == 0) return cudaSuccess;
  dequantize_kernel<<<(unsigned)((rows + 15) / 16), 256, 0, st>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq

// Device helpers for libkvq (sm_100a): shared-memory barriers, bulk async copies,
// warp-level tensor-core MMA, exact code -> f16 conversions and order-preserving keys.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // a barrier wait gives up after ~1 s

// ------------------------------------------------------------------ status
__device__ __forceinline__ void flag(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// ------------------------------------------------------------------ mbarrier + bulk copy
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with `parity` to complete; gives up after kWaitLimitNs, sets
// KVQ_DEV_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) {
      flag(status, KVQ_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// One-dimensional bulk copy global -> shared through the async copy engine; completion
// is signalled on `bar` as transaction bytes. dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Named barrier among `threads` threads (id 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------------------ programmatic dependent launch
// Wait until the grids this one depends on have completed and their writes are visible (a
// no-op when the kernel was launched without a programmatic dependency).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel in the stream to be scheduled while this grid is still running.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ------------------------------------------------------------------ tensor core
// D += A(16x16 f16, row) * B(16x8 f16, col), fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ bit tricks
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// (a & mask) | bits in one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(bits));
  return r;
}

// (a & mask) ^ bits in one LOP3
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(a), "r"(mask), "r"(bits));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// f16 bit pattern 0x6400 is 1024; OR-ing an integer n < 1024 into the mantissa gives
// exactly 1024 + n.
constexpr uint32_t kF16Magic1024x2 = 0x64006400u;

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h) {
  __half2 v = *reinterpret_cast<__half2*>(&h);
  return __half22float2(v);
}

__device__ __forceinline__ uint32_t float2_to_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// x = hi + lo with hi, lo f16: relative error of the pair <= 2^-22 in the normal f16 range.
__device__ __forceinline__ void split_f16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = float2_to_f16x2(x0, x1);
  const float2 h = f16x2_to_float2(hi);
  lo = float2_to_f16x2(x0 - h.x, x1 - h.y);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// 2^e for an integer e in [-126, 127], exact.
__device__ __forceinline__ float pow2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// Exponent shift that brings a positive finite m into [2^14, 2^15): returns e with
// m * 2^e in that range (e clamped to a safe window).
__device__ __forceinline__ int range_shift(float m) {
  if (!(m > 0.0f)) return 0;
  const int ex = static_cast<int>((__float_as_uint(m) >> 23) & 0xFF) - 127;  // floor(log2 m)
  int e = 14 - ex;
  return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// ------------------------------------------------------------------ exact quotients
// Rounding with the 1.5 * 2^23 add-and-subtract identity: RN(v + 1.5 * 2^23) holds rne(v) (ties to
// even) in its low mantissa bits for |v| < 2^22.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;

// The quotient RN(x / s) without a division per element (Markstein's fma correction, "Computation
// of elementary functions on the IBM RISC System/6000 processor", 1990): with y = RN(1/s),
// q = RN(x * y) and the residual e = RN(q * s - x) (exact under fma), RN(q - e * y) is the
// correctly rounded quotient. Every pair of fp32 significands (x, s in [1, 2), 2^46 pairs) has
// been checked against IEEE division with no mismatch (tests/gpu_quotient_check.cu runs that
// check). The operations scale exactly with the exponents while the intermediate results stay
// normal, which the range of s below guarantees for every x that can produce a nonzero code.
// Writing the residual as q * s - x keeps the sign of a zero quotient.
__device__ __forceinline__ float quot(float x, float s, float y, float& q) {
  q = __fmul_rn(x, y);
  return __fmaf_rn(-__fmaf_rn(q, s, -x), y, q);
}

// s with a normal reciprocal and room for the correction's residual: 2^-60 .. 2^60
__device__ __forceinline__ bool quot_range(float s) { return s >= 8.67361738e-19f && s <= 1.15292150e+18f; }

// ------------------------------------------------------------------ Walsh-Hadamard rotation
// Normalised transform H/sqrt(128) of a 128-value row, as butterflies of span 1, 2, ..., 64
// ((a, b) -> (a + b, a - b), a the lower index) and a final multiply by the fp32 value of
// 1/sqrt(128): every output is the same sequence of fp32 operations in any thread layout.
constexpr float kInvSqrt128 = 0.0883883476483184405f;

// Row held by the 16 lanes of a half warp, lane l holding values 8l .. 8l + 7 (mask: the
// half warp's lanes, which must all take part).
__device__ __forceinline__ void fwht_row16(float (&x)[8], unsigned mask, int lane16) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1)
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (!(k & h)) {
        const float a = x[k], b = x[k + h];
        x[k] = a + b;
        x[k + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) {
    // upper lane: partner - own; lower lane: own + partner; one fma with the sign (exact:
    // fma(-1, x, y) rounds y - x and fma(1, x, y) rounds x + y)
    const float sg = (lane16 & m) ? -1.0f : 1.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float y = __shfl_xor_sync(mask, x[k], m);
      x[k] = __fmaf_rn(sg, x[k], y);
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] *= kInvSqrt128;
}

// Row held by a whole warp, lane l holding values 4l .. 4l + 3.
__device__ __forceinline__ void fwht_row32(float (&x)[4], int lane) {
#pragma unroll
  for (int h = 1; h < 4; h <<= 1)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (!(k & h)) {
        const float a = x[k], b = x[k + h];
        x[k] = a + b;
        x[k + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float y = __shfl_xor_sync(0xffffffffu, x[k], m);
      x[k] = upper ? y - x[k] : x[k] + y;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] *= kInvSqrt128;
}

// ------------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Order-preserving map float -> uint32 (for atomicMin/atomicMax on arbitrary signs).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ------------------------------------------------------------------ scheme traits
__host__ __device__ constexpr bool kivi_f16(int s) { return s == KVQ_KIVI_INT4_F16 || s == KVQ_KIVI_INT2_F16; }
__host__ __device__ constexpr bool is_kivi(int s) {
  return s == KVQ_KIVI_INT4 || s == KVQ_KIVI_INT2 || kivi_f16(s);
}
__host__ __device__ constexpr int code_bits(int s) {
  return (s == KVQ_KIVI_INT4 || s == KVQ_KIVI_INT4_F16 || s == KVQ_INT4_SYM_PER_GROUP) ? 4
         : (s == KVQ_KIVI_INT2 || s == KVQ_KIVI_INT2_F16)                              ? 2
                                                                                        : 8;
}
__host__ __device__ constexpr int row_bytes(int s) { return kHeadDim * code_bits(s) / 8; }

}  // namespace kvq

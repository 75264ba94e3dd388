// Checks the library's division-free quotient (kvq::quot, the fma correction) against IEEE
// division, over significand pairs (x, s) in [1, 2) x [1, 2); both signs of x.
//   gpu_quotient_check bf16            every bf16 significand x every fp32 significand of s
//   gpu_quotient_check slice N K       every fp32 significand of x x the K-th of N slices of s
// Prints "pairs P mismatches M" and exits 0 when M == 0.
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <cuda_runtime.h>

#include "kvq_device.cuh"

__device__ unsigned long long g_bad;
__device__ uint32_t g_first[2][4];

__device__ __forceinline__ void check(float x, float s) {
  const float y = __frcp_rn(s);
  float q;
  const float z = kvq::quot(x, s, y, q);
  const float ref = __fdiv_rn(x, s);
  if (__float_as_uint(z) != __float_as_uint(ref)) {
    const unsigned long long k = atomicAdd(&g_bad, 1ull);
    if (k < 4) {
      g_first[0][k] = __float_as_uint(x);
      g_first[1][k] = __float_as_uint(s);
    }
  }
}

// thread = significand of s; loop over the 256 bf16 significands of x
__global__ void bf16_kernel() {
  const uint32_t j = blockIdx.x * blockDim.x + threadIdx.x;  // < 2^23
  const float s = __uint_as_float(0x3F800000u | j);
  for (uint32_t i = 0; i < 256; ++i) {
    const float x = __uint_as_float(0x3F800000u | (i << 16));
    check(x, s);
    check(-x, s);
  }
}

// thread = significand of x; loop over a run of significands of s
__global__ void slice_kernel(uint32_t s0, uint32_t ns) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;  // < 2^23
  const float x = __uint_as_float(0x3F800000u | i);
  for (uint32_t j = s0; j < s0 + ns; ++j) check((j & 1u) ? -x : x, __uint_as_float(0x3F800000u | j));
}

int main(int argc, char** argv) {
  const uint32_t kSig = 1u << 23;
  unsigned long long zero = 0, bad = 0, pairs = 0;
  cudaMemcpyToSymbol(g_bad, &zero, sizeof(zero));
  if (argc >= 2 && argv[1][0] == 'b') {
    bf16_kernel<<<kSig / 256, 256>>>();
    pairs = 2ull * 256 * kSig;
  } else if (argc >= 4) {
    const uint32_t n = (uint32_t)atoi(argv[2]), k = (uint32_t)atoi(argv[3]);
    if (n == 0 || k >= n || kSig % n != 0) {
      fprintf(stderr, "bad slice\n");
      return 2;
    }
    const uint32_t per = kSig / n, step = per < 8192u ? per : 8192u;
    for (uint32_t s0 = k * per; s0 < (k + 1) * per; s0 += step) {
      slice_kernel<<<kSig / 256, 256>>>(s0, step);
      if (cudaDeviceSynchronize() != cudaSuccess) break;
    }
    pairs = (unsigned long long)per * kSig;
  } else {
    fprintf(stderr, "usage: %s bf16 | slice N K\n", argv[0]);
    return 2;
  }
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    printf("cuda error %s\n", cudaGetErrorString(e));
    return 1;
  }
  cudaMemcpyFromSymbol(&bad, g_bad, sizeof(bad));
  printf("pairs %llu mismatches %llu\n", pairs, bad);
  uint32_t f[2][4];
  cudaMemcpyFromSymbol(f, g_first, sizeof(f));
  for (unsigned k = 0; k < 4 && k < bad; ++k) printf("  x=%08x s=%08x\n", f[0][k], f[1][k]);
  return bad == 0 ? 0 : 1;
}

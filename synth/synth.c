/*
 * Seeded synthetic inputs for the KV-cache quantization workloads.
 *
 * This module only draws numbers: it holds no quantization, dequantization or
 * attention arithmetic. Both the CPU oracle and the CUDA library consume its
 * outputs, so every value is a pure function of (seed, stream, coordinates):
 * a counter-based generator (SplitMix64, Steele/Lea/Flood 2014, used as a hash
 * of the counter) feeding Box-Muller normals, evaluated in double precision.
 * Results do not depend on the number of OpenMP threads.
 *
 * Shapes follow the problem statement of "How KV cache quantization reduces GPU
 * memory" (n4n.ai, Step 1): K and V are [batch, kv_heads, seq, head_dim].
 * Key outlier channels follow "KV Cache Quantization in Production LLM Serving"
 * (llms.blog, "The Numerical Dilemma"): a few fixed channels much larger than the
 * rest, rotated by RoPE; Values carry a per-token magnitude instead.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYN_STREAM_Q 1u
#define SYN_STREAM_K 2u
#define SYN_STREAM_V 3u
#define SYN_STREAM_SIGMA 4u
#define SYN_STREAM_OUTLIER 5u
#define SYN_STREAM_LENS 6u
#define SYN_STREAM_PAGES 7u
#define SYN_STREAM_RES 8u

static uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static uint64_t hash3(uint64_t seed, uint64_t stream, uint64_t index) {
  return splitmix64(splitmix64(splitmix64(seed) ^ stream) ^ index);
}

/* Uniform in the open interval (0, 1), 53-bit resolution. */
static double uniform01(uint64_t seed, uint64_t stream, uint64_t index) {
  uint64_t h = hash3(seed, stream, index);
  return ((double)(h >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Standard normal from two uniforms of the doubled counter (Box-Muller). */
static double normal01(uint64_t seed, uint64_t stream, uint64_t index) {
  double u1 = uniform01(seed, stream, 2 * index);
  double u2 = uniform01(seed, stream, 2 * index + 1);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

/* Coordinate packing: b < 2^10, h < 2^10, t < 2^24, d < 2^8. */
static uint64_t coord4(uint64_t b, uint64_t h, uint64_t t, uint64_t d) {
  return (((b << 10 | h) << 24 | t) << 8) | d;
}

static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* out_kind: 0 = fp32 array, 1 = bf16 (uint16) array. */
static void store(void* out, size_t i, int out_kind, double v) {
  float f = (float)v;
  if (out_kind == 0)
    ((float*)out)[i] = f;
  else
    ((uint16_t*)out)[i] = f32_to_bf16_rne(f);
}

/* n_out distinct channels in [0, D) chosen by a seeded partial Fisher-Yates. */
void syn_outlier_channels(uint64_t seed, int D, int n_out, int32_t* out) {
  int perm[1024];
  for (int i = 0; i < D; ++i) perm[i] = i;
  for (int i = 0; i < n_out; ++i) {
    uint64_t h = hash3(seed, SYN_STREAM_OUTLIER, (uint64_t)i);
    int j = i + (int)(h % (uint64_t)(D - i));
    int t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
    out[i] = perm[i];
  }
}

/*
 * Keys for rows b in [b0,b1), heads h in [h0,h1), tokens t in [t0,t1), all D channels.
 * value = N(0,1) * (outlier_scale on outlier channels), then rotate-half RoPE at
 * position t (pairs (i, i + D/2), inverse frequency theta^(-2i/D)) when theta > 0.
 * Output layout [b1-b0, h1-h0, t1-t0, D], contiguous.
 */
void syn_keys(uint64_t seed, int b0, int b1, int h0, int h1, int t0, int t1, int D,
              const int32_t* outliers, int n_out, double outlier_scale, double theta,
              int out_kind, void* out) {
  const int nb = b1 - b0, nh = h1 - h0, nt = t1 - t0;
  const long long rows = (long long)nb * nh * nt;
  double scale_of[256];
  for (int d = 0; d < D; ++d) scale_of[d] = 1.0;
  for (int i = 0; i < n_out; ++i) scale_of[outliers[i]] = outlier_scale;
#pragma omp parallel for schedule(static)
  for (long long r = 0; r < rows; ++r) {
    const int bi = (int)(r / ((long long)nh * nt));
    const int hi = (int)((r / nt) % nh);
    const int ti = (int)(r % nt);
    const int b = b0 + bi, h = h0 + hi, t = t0 + ti;
    double x[256];
    for (int d = 0; d < D; ++d)
      x[d] = normal01(seed, SYN_STREAM_K, coord4(b, h, t, d)) * scale_of[d];
    if (theta > 0.0) {
      const int half = D / 2;
      double y[256];
      for (int i = 0; i < half; ++i) {
        double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
        double ang = (double)t * inv_freq;
        double c = cos(ang), s = sin(ang);
        y[i] = x[i] * c - x[i + half] * s;
        y[i + half] = x[i + half] * c + x[i] * s;
      }
      for (int d = 0; d < D; ++d) x[d] = y[d];
    }
    for (int d = 0; d < D; ++d) store(out, (size_t)r * D + d, out_kind, x[d]);
  }
}

/* Per-token magnitude sigma = 10^U(-1,1) (log-uniform on [0.1, 10]). */
static double value_sigma(uint64_t seed, int b, int h, int t) {
  double u = uniform01(seed, SYN_STREAM_SIGMA, coord4(b, h, t, 0));
  return pow(10.0, 2.0 * u - 1.0);
}

/* Values: N(0,1) * sigma(b,h,t). Output [b1-b0, h1-h0, t1-t0, D]. */
void syn_values(uint64_t seed, int b0, int b1, int h0, int h1, int t0, int t1, int D,
                int out_kind, void* out) {
  const int nb = b1 - b0, nh = h1 - h0, nt = t1 - t0;
  const long long rows = (long long)nb * nh * nt;
#pragma omp parallel for schedule(static)
  for (long long r = 0; r < rows; ++r) {
    const int b = b0 + (int)(r / ((long long)nh * nt));
    const int h = h0 + (int)((r / nt) % nh);
    const int t = t0 + (int)(r % nt);
    const double sig = value_sigma(seed, b, h, t);
    for (int d = 0; d < D; ++d)
      store(out, (size_t)r * D + d, out_kind, normal01(seed, SYN_STREAM_V, coord4(b, h, t, d)) * sig);
  }
}

/* Queries of decode step `step`: N(0,1), output [b1-b0, Hq, D]. */
void syn_queries(uint64_t seed, int step, int b0, int b1, int Hq, int D, int out_kind, void* out) {
  const long long rows = (long long)(b1 - b0) * Hq;
#pragma omp parallel for schedule(static)
  for (long long r = 0; r < rows; ++r) {
    const int b = b0 + (int)(r / Hq);
    const int h = (int)(r % Hq);
    for (int d = 0; d < D; ++d)
      store(out, (size_t)r * D + d, out_kind,
            normal01(seed, SYN_STREAM_Q + ((uint64_t)step << 8), coord4(b, h, 0, d)));
  }
}

/* Sequence lengths uniform on the integers [lo, hi]. */
void syn_lengths(uint64_t seed, int B, int lo, int hi, int32_t* out) {
  for (int b = 0; b < B; ++b) {
    double u = uniform01(seed, SYN_STREAM_LENS, (uint64_t)b);
    int v = lo + (int)(u * (double)(hi - lo + 1));
    out[b] = v > hi ? hi : v;
  }
}

/* One integer uniform on [0, n). */
int syn_uniform_int(uint64_t seed, uint64_t tag, int n) {
  double u = uniform01(seed, SYN_STREAM_RES, tag);
  int v = (int)(u * (double)n);
  return v >= n ? n - 1 : v;
}

/* Seeded permutation of [0, n) (full Fisher-Yates). */
void syn_permutation(uint64_t seed, int n, int32_t* out) {
  for (int i = 0; i < n; ++i) out[i] = i;
  for (int i = n - 1; i > 0; --i) {
    uint64_t h = hash3(seed, SYN_STREAM_PAGES, (uint64_t)i);
    int j = (int)(h % (uint64_t)(i + 1));
    int t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
}

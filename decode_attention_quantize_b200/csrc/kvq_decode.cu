// Split-KV decode attention over the quantized cache (sm_100a).
//
// One CTA = 4 consumer warps + 1 producer warp. The grid is a persistent-style set of
// CTAs; the flattened list of (batch, kv_head, head-group) token tiles is cut into equal
// contiguous ranges, one per CTA, so every SM streams the same number of bytes however
// the sequence lengths vary. Tiles of codes reach shared memory by 2-D TMA with hardware
// swizzle (bank-conflict-free fragment loads); scales and residual tokens by 1-D bulk
// copies; both complete on per-stage mbarriers (bounded waits).
//
// Math per tile (transposed GQA packing: the G <= 8 query heads that share a KV head form
// the N = 8 side of a warp-level m16n8k16 MMA):
//   S^T[tokens x heads] = codes(f16, exact) . Q'^T      (Q' = q * fold, split hi + lo f16)
//   online softmax in the log2 domain, fp32
//   O^T[d x heads]     += codes^T(f16, exact) . P'^T   (P' = p * fold, split hi + lo f16)
// Codes stay exact (every E4M3, int8, uint8 - zp, INT4 and INT2 value is an f16 value);
// scales are folded into the fp32 operand, which is split into two f16 halves (about 22
// significant bits, range-normalised by a power of two) so the result stays well inside
// 2e-4 of an fp64 reference. Each CTA writes one (m, l, O) partial per pair it touches;
// a second kernel merges partials with the log-sum-exp rule.
//
// Sources: decode is bandwidth-bound and the kernel must consume the low-precision cache
// directly (llms.blog, "Serving Economics and Latency Trade-Offs"; n4n.ai Step 5, custom
// engine: a separate dequantize pass wastes the bandwidth saving). Scheme definitions as
// in kvq_append.cu.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kCW = 4;                  // consumer warps
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kRT = 32;                 // residual tile tokens (bf16 rows)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();

enum { FMT_E4M3, FMT_S8, FMT_U8, FMT_U4, FMT_U2 };
enum { FOLD_TENSOR, FOLD_TOKEN, FOLD_CHANNEL, FOLD_KIVI };

__host__ __device__ constexpr int fmt_of(int s) {
  return s == KVQ_FP8_E4M3_PER_TENSOR      ? FMT_E4M3
         : s == KVQ_UINT8_ASYM_PER_CHANNEL ? FMT_U8
         : s == KVQ_KIVI_INT4              ? FMT_U4
         : s == KVQ_KIVI_INT2              ? FMT_U2
                                           : FMT_S8;
}
__host__ __device__ constexpr int fold_of(int s) {
  return (s == KVQ_FP8_E4M3_PER_TENSOR || s == KVQ_INT8_SYM_PER_TENSOR)        ? FOLD_TENSOR
         : s == KVQ_INT8_SYM_PER_TOKEN                                          ? FOLD_TOKEN
         : (s == KVQ_INT8_SYM_PER_CHANNEL || s == KVQ_UINT8_ASYM_PER_CHANNEL) ? FOLD_CHANNEL
                                                                                : FOLD_KIVI;
}
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int rup(int a, int m) { return (a + m - 1) / m * m; }

template <int KS, int VS, bool PAGED>
struct Cfg {
  static constexpr bool kPaged = PAGED;
  static constexpr int kKFmt = fmt_of(KS), kVFmt = fmt_of(VS);
  static constexpr int kKFold = fold_of(KS), kVFold = fold_of(VS);
  static constexpr bool kKivi = kKFold == FOLD_KIVI;
  static constexpr int kTPW = kKivi ? 32 : 16;  // tokens per consumer warp per tile
  static constexpr int kNSub = kTPW / 16;
  static constexpr int kTS = kTPW * kCW;        // tokens per quantized tile
  static constexpr int kKRow = row_bytes(KS), kVRow = row_bytes(VS);
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTS * kKRow;     // multiple of 1024 (swizzle atom)
  static constexpr int kOffKM = kOffV + kTS * kVRow;
  static constexpr int kKMeta = kKivi ? (kTS / 32) * kHeadDim * 4 * 2 : (kKFold == FOLD_TOKEN ? kTS * 4 : 0);
  static constexpr int kOffVM = kOffKM + kKMeta;
  static constexpr int kVMeta = kKivi ? kTS * 4 * 4 * 2 : (kVFold == FOLD_TOKEN ? kTS * 4 : 0);
  static constexpr int kQuantBytes = kOffVM + kVMeta;
  static constexpr int kResBytes = kKivi ? 2 * kRT * kHeadDim * 2 : 0;
  static constexpr int kStageBytes = rup(cmax(kQuantBytes, kResBytes), 1024);
  static constexpr int kStages = kKivi ? 3 : 4;
  static constexpr int kOffDesc = kStages * kStageBytes;
  static constexpr int kOffBar = kOffDesc + kStages * 64;
  static constexpr int kOffRedO = kOffBar + 2 * kStages * 8 + 64;
  static constexpr int kOffRedM = kOffRedO + kCW * 8 * kHeadDim * 4;
  static constexpr int kOffRedL = kOffRedM + kCW * 8 * 4;
  static constexpr int kOffRedZ = kOffRedL + kCW * 8 * 4;
  static constexpr int kOffQ = kOffRedZ + kCW * 8 * 4 * 4;
  static constexpr int kQStride = 132;          // q row stride (floats), conflict-free reads
  static constexpr int kSmemBytes = kOffQ + 8 * kQStride * 4 + 1024;  // + alignment slack
};

struct TileDesc {
  int pair, b, hk, hg;
  int kind;       // 0: quantized codes, 1: bf16 residual (KIVI)
  int t0, n;      // first token (cache position or residual slot), valid tokens
  int first, last;
  uint32_t valid; // paged: bit i set when page i of the tile was loaded
  int pad[6];
};
static_assert(sizeof(TileDesc) == 64, "descriptor slot is 64 bytes");

struct Sched {
  int N, W;       // tiles, tiles per CTA
  int per_seq;    // pairs per sequence (Hkv * HG)
};

__device__ __forceinline__ Sched make_sched(const DecodeParams& p) {
  Sched s;
  s.per_seq = p.Hkv * p.HG;
  s.N = p.paged ? p.plan[p.B] : p.n_pairs * (p.nq + p.nr);
  s.W = (s.N + p.ncta - 1) / p.ncta;
  return s;
}

__device__ __forceinline__ TileDesc locate(const DecodeParams& p, const Sched& s, int t, int tb, int te) {
  TileDesc d;
  int j, npt;
  if (p.paged) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.plan[mid] <= t) lo = mid; else hi = mid - 1;
    }
    d.b = lo;
    npt = (p.plan[lo + 1] - p.plan[lo]) / s.per_seq;
    const int local = t - p.plan[lo];
    const int hh = local / npt;
    j = local % npt;
    d.pair = lo * s.per_seq + hh;
    d.hk = hh / p.HG;
    d.hg = hh % p.HG;
    d.kind = 0;
    d.t0 = j * p.ts;
    d.n = min(p.ts, p.plan[p.B + 1 + lo] - d.t0);
  } else {
    npt = p.nq + p.nr;
    d.pair = t / npt;
    j = t % npt;
    d.b = d.pair / s.per_seq;
    const int hh = d.pair % s.per_seq;
    d.hk = hh / p.HG;
    d.hg = hh % p.HG;
    if (j < p.nq) {
      d.kind = 0;
      d.t0 = j * p.ts;
      d.n = min(p.ts, p.len_q - d.t0);
    } else {
      d.kind = 1;
      d.t0 = (j - p.nq) * kRT;
      d.n = min(kRT, p.len_res - d.t0);
    }
  }
  d.first = (t == tb) || (j == 0);
  d.last = (t == te - 1) || (j == npt - 1);
  d.valid = 0xFFFFFFFFu;
  return d;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile written by TMA with the
// swizzle whose span equals the row width R (128B: 3 bits, 64B: 2 bits, 32B: 1 bit of
// the 16-byte chunk index are XORed with address bits 7..9 of the 1024-byte atom).
template <int R>
__device__ __forceinline__ int swz(int row, int chunk) {
  if constexpr (R == 128) return row * 128 + ((chunk ^ (row & 7)) << 4);
  if constexpr (R == 64) return row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4);
  return row * 32 + ((chunk ^ ((row >> 2) & 1)) << 4);
}

// ------------------------------------------------------------------ producer
template <class C>
__device__ void producer(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                         uint8_t* stages, TileDesc* descs, uint32_t full0, uint32_t empty0,
                         const Sched& s, int tb, int te) {
  for (int t = tb, it = 0; t < te; ++t, ++it) {
    const int st = it % C::kStages;
    if (it >= C::kStages && !mbar_wait(empty0 + 8 * st, ((it / C::kStages) - 1) & 1, p.status)) return;
    TileDesc d = locate(p, s, t, tb, te);
    const uint32_t sb = smem_addr(stages + st * C::kStageBytes);
    const uint32_t bar = full0 + 8 * st;
    const size_t pair_row = (size_t)d.b * p.Hkv + d.hk;
    if (d.kind == 1) {  // KIVI residual: bf16 rows, whole 32-token slab (inside rcap)
      const size_t r0 = (pair_row * p.rcap + d.t0) * kHeadDim;
      descs[st] = d;
      mbar_arrive_expect_tx(bar, 2 * kRT * kHeadDim * 2);
      bulk_g2s(sb, p.k_res + r0, kRT * kHeadDim * 2, bar);
      bulk_g2s(sb + kRT * kHeadDim * 2, p.v_res + r0, kRT * kHeadDim * 2, bar);
      continue;
    }
    if constexpr (!C::kPaged) {
      // whole tile: capacity is a multiple of 128 tokens, so the tile lies inside the row
      const size_t row0 = pair_row * p.cap + d.t0;
      const uint32_t bytes = C::kTS * (C::kKRow + C::kVRow) + C::kKMeta + C::kVMeta;
      descs[st] = d;
      mbar_arrive_expect_tx(bar, bytes);
      tma_2d(sb + C::kOffK, tk, 0, (int)row0, bar);
      tma_2d(sb + C::kOffV, tv, 0, (int)row0, bar);
      if constexpr (C::kKivi) {
        const size_t g0 = (pair_row * (p.cap / 32) + d.t0 / 32) * kHeadDim;
        bulk_g2s(sb + C::kOffKM, p.k_scale + g0, C::kKMeta / 2, bar);
        bulk_g2s(sb + C::kOffKM + C::kKMeta / 2, p.k_zero + g0, C::kKMeta / 2, bar);
        bulk_g2s(sb + C::kOffVM, p.v_scale + row0 * 4, C::kVMeta / 2, bar);
        bulk_g2s(sb + C::kOffVM + C::kVMeta / 2, p.v_zero + row0 * 4, C::kVMeta / 2, bar);
      } else {
        if constexpr (C::kKFold == FOLD_TOKEN) bulk_g2s(sb + C::kOffKM, p.k_scale + row0, C::kKMeta, bar);
        if constexpr (C::kVFold == FOLD_TOKEN) bulk_g2s(sb + C::kOffVM, p.v_scale + row0, C::kVMeta, bar);
      }
    } else {
      // paged: page i of the tile -> rows (page * Hkv + hk) * page_size of the pool
      const int ps = p.page_size;
      const int npg = (d.n + ps - 1) / ps;
      const int pi0 = d.t0 / ps;
      int page[C::kTS / 16];
      uint32_t valid = 0, nvalid = 0;
#pragma unroll
      for (int i = 0; i < C::kTS / 16; ++i) {
        page[i] = -1;
        if (i < npg) {
          const int pi = pi0 + i;
          const int id = pi < p.max_pages ? p.page_table[(size_t)d.b * p.max_pages + pi] : -1;
          page[i] = id;
          if (id >= 0 && id < p.num_pages) {
            valid |= 1u << i;
            ++nvalid;
          } else {
            flag(p.status, KVQ_DEV_BAD_PAGE);
          }
        }
      }
      d.valid = valid;
      descs[st] = d;
      uint32_t per_page = ps * (C::kKRow + C::kVRow);
      if constexpr (C::kKFold == FOLD_TOKEN) per_page += ps * 4;
      if constexpr (C::kVFold == FOLD_TOKEN) per_page += ps * 4;
      mbar_arrive_expect_tx(bar, nvalid * per_page);
#pragma unroll
      for (int i = 0; i < C::kTS / 16; ++i) {
        if (i >= npg || !((valid >> i) & 1u)) continue;
        const size_t prow = ((size_t)page[i] * p.Hkv + d.hk) * ps;
        tma_2d(sb + C::kOffK + i * ps * C::kKRow, tk, 0, (int)prow, bar);
        tma_2d(sb + C::kOffV + i * ps * C::kVRow, tv, 0, (int)prow, bar);
        if constexpr (C::kKFold == FOLD_TOKEN) bulk_g2s(sb + C::kOffKM + i * ps * 4, p.k_scale + prow, ps * 4, bar);
        if constexpr (C::kVFold == FOLD_TOKEN) bulk_g2s(sb + C::kOffVM + i * ps * 4, p.v_scale + prow, ps * 4, bar);
      }
    }
  }
}

// ------------------------------------------------------------------ fragment helpers
// Channel of k-slot pair `h` (0: columns 2c,2c+1; 1: columns 2c+8,2c+9), element e, of
// k-step ks, for the thread with column group c. The mapping follows how each code width
// unpacks into f16 pairs; Q' uses the same mapping so the dot product is unchanged.
template <int FMT>
__device__ __forceinline__ int dmap_k(int c, int ks, int h, int e) {
  if constexpr (FMT == FMT_U4) return 32 * c + 8 * (ks >> 1) + 2 * (ks & 1) + h + 4 * e;
  if constexpr (FMT == FMT_U2) return 32 * c + 16 * (ks >> 2) + 2 * (ks & 3) + h + 8 * e;
  return 32 * c + 4 * ks + 2 * h + e;  // 8-bit codes and bf16 rows
}

// Channel held by V^T fragment row (m-tile mt, row half rh) for row group g.
template <bool kGrouped>
__device__ __forceinline__ int dmap_v(int g, int mt, int rh) {
  if constexpr (kGrouped) return 32 * (mt >> 1) + 4 * g + 2 * (mt & 1) + rh;  // inside 32-channel groups
  return 16 * g + 2 * mt + rh;
}

// 16-bit piece (two 8-bit codes) -> f16x2 of the code values.
template <int FMT>
__device__ __forceinline__ uint32_t cvt8x2(uint32_t piece16, uint32_t zp_bias) {
  if constexpr (FMT == FMT_E4M3) {
    return e4m3x2_to_f16x2(piece16);
  } else if constexpr (FMT == FMT_S8) {  // piece already XORed with 0x80: biased by 128
    return hsub2_u(prmt(piece16, 0x64646464u, 0x5150u), 0x64806480u);  // - 1152
  } else {  // FMT_U8: subtract 1024 + zero point
    return hsub2_u(prmt(piece16, 0x64646464u, 0x5150u), zp_bias);
  }
}

// Nibble pairs of a 32-bit word: k = 0..3 -> (nibble k, nibble k + 4).
__device__ __forceinline__ uint32_t u4_pair(uint32_t w, int k) {
  const uint32_t x = (k & 2) ? (w >> 8) : w;
  if (k & 1) return hfma2_u(and_or(x, 0x00F000F0u, kF16Magic1024x2), 0x2C002C00u, 0xD400D400u);  // /16 - 64
  return hsub2_u(and_or(x, 0x000F000Fu, kF16Magic1024x2), kF16Magic1024x2);
}

// 2-bit field pairs of a 32-bit word: k = 0..7 -> (field k, field k + 8).
__device__ __forceinline__ uint32_t u2_pair(uint32_t w, int k) {
  const uint32_t x = (k & 4) ? (w >> 8) : w;
  switch (k & 3) {
    case 0: return hsub2_u(and_or(x, 0x00030003u, kF16Magic1024x2), kF16Magic1024x2);
    case 1: return hfma2_u(and_or(x, 0x000C000Cu, kF16Magic1024x2), 0x34003400u, 0xDC00DC00u);  // /4 - 256
    case 2: return hfma2_u(and_or(x, 0x00300030u, kF16Magic1024x2), 0x2C002C00u, 0xD400D400u);  // /16 - 64
    default: return hfma2_u(and_or(x, 0x00C000C0u, kF16Magic1024x2), 0x24002400u, 0xCC00CC00u); // /64 - 16
  }
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return float2_to_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

template <class T>
__device__ __forceinline__ T lds(const uint8_t* p) {
  return *reinterpret_cast<const T*>(p);
}

// ------------------------------------------------------------------ consumer state
template <class C>
struct Consumer {
  int w, lane, g, c;
  float o[8][4];
  float m[2], l[2];
  int ev;            // O accumulator holds (true value) * 2^ev
  bool ev_set;
  float zacc[4];     // KIVI: sum p * min per channel group, head g
  uint32_t qh[8][2], ql[8][2];
  bool qsplit;
  float kmul;        // score multiplier (log2 domain)
  float bias[2];     // KIVI group bias (raw units), heads 2c, 2c+1
  int qmode;         // 0: fragments for codes built, 1: for bf16 residual rows
};

// Build Q' fragments (head g, this thread's channels) from q_s, optionally multiplied by
// a per-channel fold; returns the power-of-two shift applied.
template <int FMT>
__device__ __forceinline__ int build_q(const float* q_s, const float* fold, int g, int c,
                                       uint32_t (&qh)[8][2], uint32_t (&ql)[8][2]) {
  float v[8][2][2];
  float mx = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int d = dmap_k<FMT>(c, ks, h, e);
        float x = q_s[g * 132 + d + (d >> 5)];
        if (fold) x *= fold[d];
        v[ks][h][e] = x;
        mx = fmaxf(mx, fabsf(x));
      }
  mx = warp_max(mx);
  const int eq = range_shift(mx);
  const float f = pow2i(eq);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h) split_f16x2(v[ks][h][0] * f, v[ks][h][1] * f, qh[ks][h], ql[ks][h]);
  return eq;
}

// ------------------------------------------------------------------ the kernel
template <int KS, int VS, bool PAGED>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
  using C = Cfg<KS, VS, PAGED>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  const Sched sc = make_sched(p);
  const int tb = blockIdx.x * sc.W;
  const int te = min(sc.N, tb + sc.W);
  if (tb >= te) return;
  TileDesc* descs = reinterpret_cast<TileDesc*>(smem + C::kOffDesc);
  const uint32_t full0 = smem_addr(smem + C::kOffBar);
  const uint32_t empty0 = full0 + 8 * C::kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kCW);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == kCW) {
    if (lane == 0) producer<C>(p, &tmap_k, &tmap_v, smem, descs, full0, empty0, sc, tb, te);
    return;
  }

  // ---------------------------------------------------------------- consumers
  Consumer<C> S;
  S.w = warp;
  S.lane = lane;
  S.g = lane >> 2;
  S.c = lane & 3;
  const int g = S.g, c = S.c, w = S.w;
  float* red_o = reinterpret_cast<float*>(smem + C::kOffRedO);
  float* red_m = reinterpret_cast<float*>(smem + C::kOffRedM);
  float* red_l = reinterpret_cast<float*>(smem + C::kOffRedL);
  float* red_z = reinterpret_cast<float*>(smem + C::kOffRedZ);
  float* q_s = reinterpret_cast<float*>(smem + C::kOffQ);
  const float sc_log2 = p.softmax_scale * kLog2e;
  bool dead = false;
  uint32_t zpk[8][2], zpv[8][2];

  for (int t = tb, it = 0; t < te; ++t, ++it) {
    const int st = it % C::kStages;
    const TileDesc d = locate(p, sc, t, tb, te);
    if (!dead && !mbar_wait(full0 + 8 * st, (it / C::kStages) & 1, p.status)) dead = true;
    const uint8_t* base = smem + st * C::kStageBytes;
    const uint32_t valid = C::kPaged ? descs[st].valid : 0xFFFFFFFFu;

    // ------------------------------------------------ pair start
    if (d.first) {
      const int tid = threadIdx.x;  // 0..127
      for (int idx = tid; idx < 8 * kHeadDim; idx += kCW * 32) {
        const int j = idx >> 7, dd = idx & 127;
        const int hl = d.hg * 8 + j;
        float v = 0.0f;
        if (hl < p.G) {
          const size_t qi = ((size_t)d.b * p.Hq + (size_t)d.hk * p.G + hl) * kHeadDim + dd;
          v = p.q_bf16 ? bf16_bits_to_float(static_cast<const uint16_t*>(p.q)[qi])
                       : static_cast<const float*>(p.q)[qi];
        }
        q_s[j * 132 + dd + (dd >> 5)] = v;
      }
      named_sync(1, kCW * 32);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) S.o[mt][k] = 0.0f;
      S.m[0] = S.m[1] = kNegInf;
      S.l[0] = S.l[1] = 0.0f;
      S.ev = 15;
      S.ev_set = false;
#pragma unroll
      for (int j = 0; j < 4; ++j) S.zacc[j] = 0.0f;
      S.qmode = -1;
      if constexpr (!C::kKivi) {
        const float* fold = nullptr;
        if constexpr (C::kKFold == FOLD_CHANNEL) fold = p.k_scale + (size_t)d.hk * kHeadDim;
        const int eq = build_q<C::kKFmt>(q_s, fold, g, c, S.qh, S.ql);
        S.qsplit = (C::kKFold == FOLD_CHANNEL) || !p.q_bf16;
        float mul = sc_log2 * pow2i(-eq);
        if constexpr (C::kKFold == FOLD_TENSOR) mul *= p.k_scale[0];
        S.kmul = mul;
        S.qmode = 0;
        if constexpr (C::kKFmt == FMT_U8) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int d0 = dmap_k<C::kKFmt>(c, ks, h, 0);
              const float z0 = 1024.0f + p.k_zp[d.hk * kHeadDim + d0];
              const float z1 = 1024.0f + p.k_zp[d.hk * kHeadDim + d0 + 1];
              zpk[ks][h] = float2_to_f16x2(z0, z1);
            }
        }
      }
      if constexpr (C::kVFmt == FMT_U8) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int rh = 0; rh < 2; ++rh) {
            const float z = 1024.0f + p.v_zp[d.hk * kHeadDim + dmap_v<false>(g, mt, rh)];
            zpv[mt][rh] = float2_to_f16x2(z, z);
          }
      }
    }

    // ------------------------------------------------ tile work
    const bool residual = C::kKivi && d.kind == 1;
    const int tok_base = residual ? 0 : w * C::kTPW;
    const bool busy = !dead && (residual ? (w == 0) : true) && (d.n - tok_base > 0);
    if (busy) {
      // (1) query fragments for this tile
      if constexpr (C::kKivi) {
        if (!residual) {
          const float* ksm = reinterpret_cast<const float*>(base + C::kOffKM) + w * kHeadDim;
          const float* kzm = reinterpret_cast<const float*>(base + C::kOffKM + C::kKMeta / 2) + w * kHeadDim;
          const int eq = build_q<C::kKFmt>(q_s, ksm, g, c, S.qh, S.ql);
          float bs = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int dd = 32 * c + i;
            bs = fmaf(q_s[g * 132 + dd + (dd >> 5)], kzm[dd], bs);
          }
          bs += __shfl_xor_sync(0xffffffffu, bs, 1);
          bs += __shfl_xor_sync(0xffffffffu, bs, 2);
          S.bias[0] = __shfl_sync(0xffffffffu, bs, 4 * (2 * c));
          S.bias[1] = __shfl_sync(0xffffffffu, bs, 4 * (2 * c + 1));
          S.kmul = pow2i(-eq);
          S.qsplit = true;
          S.qmode = 0;
        } else if (S.qmode != 1) {
          const int eq = build_q<FMT_S8>(q_s, nullptr, g, c, S.qh, S.ql);
          S.kmul = sc_log2 * pow2i(-eq);
          S.qsplit = !p.q_bf16;
          S.qmode = 1;
        }
      }

      // (2) S^T = K . Q'^T for kNSub blocks of 16 tokens
      float acc[C::kNSub][4];
#pragma unroll
      for (int sb = 0; sb < C::kNSub; ++sb) {
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[sb][k] = 0.0f;
        const int r0 = tok_base + sb * 16 + g, r1 = r0 + 8;
        if (residual) {
          const uint8_t* kr = base;  // bf16 rows of 256 bytes
          uint32_t w0[16], w1[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 a = lds<uint4>(kr + r0 * 256 + c * 64 + i * 16);
            const uint4 b = lds<uint4>(kr + r1 * 256 + c * 64 + i * 16);
            w0[4 * i] = a.x; w0[4 * i + 1] = a.y; w0[4 * i + 2] = a.z; w0[4 * i + 3] = a.w;
            w1[4 * i] = b.x; w1[4 * i + 1] = b.y; w1[4 * i + 2] = b.z; w1[4 * i + 3] = b.w;
          }
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t a0 = bf16x2_to_f16x2(w0[2 * ks]), a1 = bf16x2_to_f16x2(w1[2 * ks]);
            const uint32_t a2 = bf16x2_to_f16x2(w0[2 * ks + 1]), a3 = bf16x2_to_f16x2(w1[2 * ks + 1]);
            mma_16816(acc[sb], a0, a1, a2, a3, S.qh[ks][0], S.qh[ks][1]);
            if (S.qsplit) mma_16816(acc[sb], a0, a1, a2, a3, S.ql[ks][0], S.ql[ks][1]);
          }
        } else if constexpr (C::kKFmt == FMT_U4) {
          const uint4 a = lds<uint4>(base + C::kOffK + swz<64>(r0, c));
          const uint4 b = lds<uint4>(base + C::kOffK + swz<64>(r1, c));
          const uint32_t w0[4] = {a.x, a.y, a.z, a.w}, w1[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const int i = ks >> 1, k0 = 2 * (ks & 1);
            const uint32_t a0 = u4_pair(w0[i], k0), a1 = u4_pair(w1[i], k0);
            const uint32_t a2 = u4_pair(w0[i], k0 + 1), a3 = u4_pair(w1[i], k0 + 1);
            mma_16816(acc[sb], a0, a1, a2, a3, S.qh[ks][0], S.qh[ks][1]);
            mma_16816(acc[sb], a0, a1, a2, a3, S.ql[ks][0], S.ql[ks][1]);
          }
        } else if constexpr (C::kKFmt == FMT_U2) {
          const uint2 a = lds<uint2>(base + C::kOffK + swz<32>(r0, c >> 1) + 8 * (c & 1));
          const uint2 b = lds<uint2>(base + C::kOffK + swz<32>(r1, c >> 1) + 8 * (c & 1));
          const uint32_t w0[2] = {a.x, a.y}, w1[2] = {b.x, b.y};
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const int i = ks >> 2, k0 = 2 * (ks & 3);
            const uint32_t a0 = u2_pair(w0[i], k0), a1 = u2_pair(w1[i], k0);
            const uint32_t a2 = u2_pair(w0[i], k0 + 1), a3 = u2_pair(w1[i], k0 + 1);
            mma_16816(acc[sb], a0, a1, a2, a3, S.qh[ks][0], S.qh[ks][1]);
            mma_16816(acc[sb], a0, a1, a2, a3, S.ql[ks][0], S.ql[ks][1]);
          }
        } else {
          // 8-bit codes, 128-byte rows: chunks 2c, 2c+1 (order swapped on odd rows so the
          // eight lanes of a load phase touch distinct banks)
          const int sw0 = g & 1;
          const uint4 a0v = lds<uint4>(base + C::kOffK + swz<128>(r0, 2 * c + sw0));
          const uint4 a1v = lds<uint4>(base + C::kOffK + swz<128>(r0, 2 * c + (sw0 ^ 1)));
          const uint4 b0v = lds<uint4>(base + C::kOffK + swz<128>(r1, 2 * c + sw0));
          const uint4 b1v = lds<uint4>(base + C::kOffK + swz<128>(r1, 2 * c + (sw0 ^ 1)));
          const uint4 a_lo = sw0 ? a1v : a0v, a_hi = sw0 ? a0v : a1v;
          const uint4 b_lo = sw0 ? b1v : b0v, b_hi = sw0 ? b0v : b1v;
          uint32_t w0[8] = {a_lo.x, a_lo.y, a_lo.z, a_lo.w, a_hi.x, a_hi.y, a_hi.z, a_hi.w};
          uint32_t w1[8] = {b_lo.x, b_lo.y, b_lo.z, b_lo.w, b_hi.x, b_hi.y, b_hi.z, b_hi.w};
          if constexpr (C::kKFmt == FMT_S8) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              w0[i] ^= 0x80808080u;
              w1[i] ^= 0x80808080u;
            }
          }
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t z0 = C::kKFmt == FMT_U8 ? zpk[ks][0] : 0u;
            const uint32_t z1 = C::kKFmt == FMT_U8 ? zpk[ks][1] : 0u;
            const uint32_t a0 = cvt8x2<C::kKFmt>(w0[ks] & 0xFFFFu, z0);
            const uint32_t a1 = cvt8x2<C::kKFmt>(w1[ks] & 0xFFFFu, z0);
            const uint32_t a2 = cvt8x2<C::kKFmt>(w0[ks] >> 16, z1);
            const uint32_t a3 = cvt8x2<C::kKFmt>(w1[ks] >> 16, z1);
            mma_16816(acc[sb], a0, a1, a2, a3, S.qh[ks][0], S.qh[ks][1]);
            if (S.qsplit) mma_16816(acc[sb], a0, a1, a2, a3, S.ql[ks][0], S.ql[ks][1]);
          }
        }
      }

      // (3) scores (log2 domain) with masking
      float sco[C::kNSub][4];
#pragma unroll
      for (int sb = 0; sb < C::kNSub; ++sb)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int tok = tok_base + sb * 16 + g + 8 * r;
          bool ok = tok < d.n;
          if constexpr (C::kPaged) ok = ok && ((valid >> (tok / p.page_size)) & 1u);
          float mul = S.kmul;
          if constexpr (C::kKFold == FOLD_TOKEN) mul *= reinterpret_cast<const float*>(base + C::kOffKM)[tok];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            float s;
            if (C::kKivi && !residual)
              s = fmaf(acc[sb][2 * r + j], S.kmul, S.bias[j]) * sc_log2;
            else
              s = acc[sb][2 * r + j] * mul;
            sco[sb][2 * r + j] = ok ? s : kNegInf;
          }
        }

      // (4) online softmax over this warp's tokens
      float alpha[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float mx = kNegInf;
#pragma unroll
        for (int sb = 0; sb < C::kNSub; ++sb) mx = fmaxf(mx, fmaxf(sco[sb][j], sco[sb][2 + j]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mnew = fmaxf(S.m[j], mx);
        const float ms = mnew == kNegInf ? 0.0f : mnew;
        alpha[j] = fast_exp2(S.m[j] - ms);
        float ls = 0.0f;
#pragma unroll
        for (int sb = 0; sb < C::kNSub; ++sb) {
          sco[sb][j] = fast_exp2(sco[sb][j] - ms);
          sco[sb][2 + j] = fast_exp2(sco[sb][2 + j] - ms);
          ls += sco[sb][j] + sco[sb][2 + j];
        }
        S.l[j] = S.l[j] * alpha[j] + ls;
        S.m[j] = mnew;
      }

      // (5) probabilities to the B-operand layout: head g, tokens 2c, 2c+1, 2c+8, 2c+9
      float pt[C::kNSub][4];
      const int srcA = 4 * (2 * c) + (g >> 1), srcB = srcA + 4;
#pragma unroll
      for (int sb = 0; sb < C::kNSub; ++sb) {
        const float a0 = __shfl_sync(0xffffffffu, sco[sb][0], srcA);
        const float a1 = __shfl_sync(0xffffffffu, sco[sb][1], srcA);
        const float a2 = __shfl_sync(0xffffffffu, sco[sb][2], srcA);
        const float a3 = __shfl_sync(0xffffffffu, sco[sb][3], srcA);
        const float b0 = __shfl_sync(0xffffffffu, sco[sb][0], srcB);
        const float b1 = __shfl_sync(0xffffffffu, sco[sb][1], srcB);
        const float b2 = __shfl_sync(0xffffffffu, sco[sb][2], srcB);
        const float b3 = __shfl_sync(0xffffffffu, sco[sb][3], srcB);
        const bool odd = g & 1;
        pt[sb][0] = odd ? a1 : a0;
        pt[sb][1] = odd ? b1 : b0;
        pt[sb][2] = odd ? a3 : a2;
        pt[sb][3] = odd ? b3 : b2;
      }

      // (6) value-side fold and accumulator exponent
      constexpr bool kVPerToken = C::kVFold == FOLD_TOKEN || C::kKivi;
      float vs[C::kNSub][4][4];  // [sb][token][group] folded scale (token fold: group 0)
      int evn = 15;
      if (kVPerToken && !residual) {
        float smax = 0.0f;
#pragma unroll
        for (int sb = 0; sb < C::kNSub; ++sb)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int tok = tok_base + sb * 16 + 2 * c + (k & 1) + 8 * (k >> 1);
            bool ok = tok < d.n;
            if constexpr (C::kPaged) ok = ok && ((valid >> (tok / p.page_size)) & 1u);
            if constexpr (C::kKivi) {
              const float4 s4 = lds<float4>(base + C::kOffVM + tok * 16);
              vs[sb][k][0] = ok ? s4.x : 0.0f;
              vs[sb][k][1] = ok ? s4.y : 0.0f;
              vs[sb][k][2] = ok ? s4.z : 0.0f;
              vs[sb][k][3] = ok ? s4.w : 0.0f;
              smax = fmaxf(smax, fmaxf(fmaxf(vs[sb][k][0], vs[sb][k][1]), fmaxf(vs[sb][k][2], vs[sb][k][3])));
            } else {
              const float s1 = reinterpret_cast<const float*>(base + C::kOffVM)[tok];
              vs[sb][k][0] = ok ? s1 : 0.0f;
              smax = fmaxf(smax, vs[sb][k][0]);
            }
          }
        smax = warp_max(smax);
        evn = smax > 0.0f ? range_shift(smax) : (S.ev_set ? S.ev : 15);
      }
      float f0 = alpha[0], f1 = alpha[1];
      if (S.ev_set) {
        const float r = fast_exp2((float)(evn - S.ev));
        f0 *= r;
        f1 *= r;
      }
      S.ev = evn;
      S.ev_set = true;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        S.o[mt][0] *= f0;
        S.o[mt][1] *= f1;
        S.o[mt][2] *= f0;
        S.o[mt][3] *= f1;
      }
      const float pscale = pow2i(evn);

      // (7) O^T += V^T . P'^T
      if constexpr (C::kKivi) {
        // alpha for head g rescales the min-term accumulator
        const float ag0 = __shfl_sync(0xffffffffu, alpha[0], g >> 1);
        const float ag1 = __shfl_sync(0xffffffffu, alpha[1], g >> 1);
        const float ag = (g & 1) ? ag1 : ag0;
#pragma unroll
        for (int j = 0; j < 4; ++j) S.zacc[j] *= ag;
      }
#pragma unroll
      for (int sb = 0; sb < C::kNSub; ++sb) {
        const int tb0 = tok_base + sb * 16;
        const int tk[4] = {tb0 + 2 * c, tb0 + 2 * c + 1, tb0 + 2 * c + 8, tb0 + 2 * c + 9};
        bool ok[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ok[k] = tk[k] < d.n;
          if constexpr (C::kPaged) ok[k] = ok[k] && ((valid >> (tk[k] / p.page_size)) & 1u);
        }
        if constexpr (!C::kKivi) {
          float pv[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            pv[k] = (C::kVFold == FOLD_TOKEN ? pt[sb][k] * vs[sb][k][0] : pt[sb][k]) * pscale;
          uint32_t bh0, bl0, bh1, bl1;
          split_f16x2(pv[0], pv[1], bh0, bl0);
          split_f16x2(pv[2], pv[3], bh1, bl1);
          const int vrow = 16 * g;  // chunk g of each 128-byte row
          uint4 W[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            W[k] = lds<uint4>(base + C::kOffV + swz<128>(tk[k], g));
            if (!ok[k]) W[k] = make_uint4(0u, 0u, 0u, 0u);
            if constexpr (C::kVFmt == FMT_S8) {
              W[k].x ^= 0x80808080u; W[k].y ^= 0x80808080u; W[k].z ^= 0x80808080u; W[k].w ^= 0x80808080u;
            }
          }
          (void)vrow;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t x0 = q == 0 ? W[0].x : q == 1 ? W[0].y : q == 2 ? W[0].z : W[0].w;
            const uint32_t x1 = q == 0 ? W[1].x : q == 1 ? W[1].y : q == 2 ? W[1].z : W[1].w;
            const uint32_t x2 = q == 0 ? W[2].x : q == 1 ? W[2].y : q == 2 ? W[2].z : W[2].w;
            const uint32_t x3 = q == 0 ? W[3].x : q == 1 ? W[3].y : q == 2 ? W[3].z : W[3].w;
            const uint32_t t01a = prmt(x0, x1, 0x5140u), t01b = prmt(x0, x1, 0x7362u);
            const uint32_t t23a = prmt(x2, x3, 0x5140u), t23b = prmt(x2, x3, 0x7362u);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int mt = 2 * q + half;
              const uint32_t ta = half ? t01b : t01a, tb2 = half ? t23b : t23a;
              const uint32_t zr0 = C::kVFmt == FMT_U8 ? zpv[mt][0] : 0u;
              const uint32_t zr1 = C::kVFmt == FMT_U8 ? zpv[mt][1] : 0u;
              const uint32_t a0 = cvt8x2<C::kVFmt>(ta & 0xFFFFu, zr0);
              const uint32_t a1 = cvt8x2<C::kVFmt>(ta >> 16, zr1);
              const uint32_t a2 = cvt8x2<C::kVFmt>(tb2 & 0xFFFFu, zr0);
              const uint32_t a3 = cvt8x2<C::kVFmt>(tb2 >> 16, zr1);
              mma_16816(S.o[mt], a0, a1, a2, a3, bh0, bh1);
              mma_16816(S.o[mt], a0, a1, a2, a3, bl0, bl1);
            }
          }
        } else {
          // KIVI: one B operand per 32-channel group; zero-point term on CUDA cores
          uint32_t bh[4][2], bl[4][2];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float pv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) pv[k] = residual ? pt[sb][k] * pscale : pt[sb][k] * vs[sb][k][j] * pscale;
            split_f16x2(pv[0], pv[1], bh[j][0], bl[j][0]);
            split_f16x2(pv[2], pv[3], bh[j][1], bl[j][1]);
          }
          if (!residual) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if (!ok[k]) continue;
              const float4 z4 = lds<float4>(base + C::kOffVM + C::kVMeta / 2 + tk[k] * 16);
              S.zacc[0] = fmaf(pt[sb][k], z4.x, S.zacc[0]);
              S.zacc[1] = fmaf(pt[sb][k], z4.y, S.zacc[1]);
              S.zacc[2] = fmaf(pt[sb][k], z4.z, S.zacc[2]);
              S.zacc[3] = fmaf(pt[sb][k], z4.w, S.zacc[3]);
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t pr[2][4];  // [token pair][channel e]: f16x2 (token even, token odd)
            if (residual) {
#pragma unroll
              for (int pp = 0; pp < 2; ++pp) {
                const uint8_t* vr = base + kRT * kHeadDim * 2;
                uint2 u0 = lds<uint2>(vr + tk[2 * pp] * 256 + (32 * j + 4 * g) * 2);
                uint2 u1 = lds<uint2>(vr + tk[2 * pp + 1] * 256 + (32 * j + 4 * g) * 2);
                if (!ok[2 * pp]) u0 = make_uint2(0u, 0u);
                if (!ok[2 * pp + 1]) u1 = make_uint2(0u, 0u);
                pr[pp][0] = float2_to_f16x2(bf16_bits_to_float(u0.x & 0xFFFFu), bf16_bits_to_float(u1.x & 0xFFFFu));
                pr[pp][1] = float2_to_f16x2(bf16_bits_to_float(u0.x >> 16), bf16_bits_to_float(u1.x >> 16));
                pr[pp][2] = float2_to_f16x2(bf16_bits_to_float(u0.y & 0xFFFFu), bf16_bits_to_float(u1.y & 0xFFFFu));
                pr[pp][3] = float2_to_f16x2(bf16_bits_to_float(u0.y >> 16), bf16_bits_to_float(u1.y >> 16));
              }
            } else if constexpr (C::kVFmt == FMT_U4) {
#pragma unroll
              for (int pp = 0; pp < 2; ++pp) {
                uint32_t u0 = lds<uint16_t>(base + C::kOffV + swz<64>(tk[2 * pp], j) + 2 * g);
                uint32_t u1 = lds<uint16_t>(base + C::kOffV + swz<64>(tk[2 * pp + 1], j) + 2 * g);
                if (!ok[2 * pp]) u0 = 0u;
                if (!ok[2 * pp + 1]) u1 = 0u;
                const uint32_t wv = prmt(u0, u1, 0x5410u);
#pragma unroll
                for (int e = 0; e < 4; ++e) pr[pp][e] = u4_pair(wv, e);
              }
            } else {
#pragma unroll
              for (int pp = 0; pp < 2; ++pp) {
                uint32_t u0 = lds<uint8_t>(base + C::kOffV + swz<32>(tk[2 * pp], j >> 1) + 8 * (j & 1) + g);
                uint32_t u1 = lds<uint8_t>(base + C::kOffV + swz<32>(tk[2 * pp + 1], j >> 1) + 8 * (j & 1) + g);
                if (!ok[2 * pp]) u0 = 0u;
                if (!ok[2 * pp + 1]) u1 = 0u;
                const uint32_t wv = prmt(u0, u1, 0x5410u);
#pragma unroll
                for (int e = 0; e < 4; ++e) pr[pp][e] = u2_pair(wv, e);
              }
            }
            // channel e = 2 * (mt & 1) + rh within the group: mt = 2j + (e >> 1)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int mt = 2 * j + half;
              const uint32_t a0 = pr[0][2 * half], a1 = pr[0][2 * half + 1];
              const uint32_t a2 = pr[1][2 * half], a3 = pr[1][2 * half + 1];
              mma_16816(S.o[mt], a0, a1, a2, a3, bh[j][0], bh[j][1]);
              mma_16816(S.o[mt], a0, a1, a2, a3, bl[j][0], bl[j][1]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * st);

    // ------------------------------------------------ pair end: merge the warps
    if (d.last) {
      float l0 = S.l[0], l1 = S.l[1];
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
      }
      if (g == 0) {
        red_m[w * 8 + 2 * c] = S.m[0];
        red_m[w * 8 + 2 * c + 1] = S.m[1];
        red_l[w * 8 + 2 * c] = l0;
        red_l[w * 8 + 2 * c + 1] = l1;
      }
      const float oscale = S.ev_set ? pow2i(-S.ev) : 0.0f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int rh = 0; rh < 2; ++rh) {
          const int dd = dmap_v<C::kKivi>(g, mt, rh);
          red_o[(w * 8 + 2 * c) * kHeadDim + dd] = S.o[mt][2 * rh] * oscale;
          red_o[(w * 8 + 2 * c + 1) * kHeadDim + dd] = S.o[mt][2 * rh + 1] * oscale;
        }
      if constexpr (C::kKivi) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float z = S.zacc[j];
          z += __shfl_xor_sync(0xffffffffu, z, 1);
          z += __shfl_xor_sync(0xffffffffu, z, 2);
          if (c == 0) red_z[(w * 8 + g) * 4 + j] = z;
        }
      }
      named_sync(1, kCW * 32);
      const int dd = threadIdx.x;  // channel
      const int slot = d.pair + blockIdx.x;
      float vsc = 1.0f;
      if constexpr (C::kVFold == FOLD_TENSOR) vsc = p.v_scale[0];
      if constexpr (C::kVFold == FOLD_CHANNEL) vsc = p.v_scale[(size_t)d.hk * kHeadDim + dd];
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        float M = kNegInf;
#pragma unroll
        for (int ww = 0; ww < kCW; ++ww) M = fmaxf(M, red_m[ww * 8 + j]);
        float ov = 0.0f, L = 0.0f;
        if (M != kNegInf) {
#pragma unroll
          for (int ww = 0; ww < kCW; ++ww) {
            const float a = fast_exp2(red_m[ww * 8 + j] - M);
            float x = red_o[(ww * 8 + j) * kHeadDim + dd];
            if constexpr (C::kKivi) x += red_z[(ww * 8 + j) * 4 + (dd >> 5)];
            ov = fmaf(a, x, ov);
            L = fmaf(a, red_l[ww * 8 + j], L);
          }
        }
        p.part_o[((size_t)slot * 8 + j) * kHeadDim + dd] = ov * vsc;
        if (dd == 0) {
          p.part_ml[((size_t)slot * 8 + j) * 2] = M;
          p.part_ml[((size_t)slot * 8 + j) * 2 + 1] = L;
        }
      }
      named_sync(1, kCW * 32);
    }
  }
}

// ------------------------------------------------------------------ merge
__global__ void __launch_bounds__(128) merge_kernel(const DecodeParams p) {
  const int pair = blockIdx.x, dd = threadIdx.x;
  const int per_seq = p.Hkv * p.HG;
  const int b = pair / per_seq, hh = pair % per_seq, hk = hh / p.HG, hg = hh % p.HG;
  int off, n, N;
  if (p.paged) {
    N = p.plan[p.B];
    n = (p.plan[b + 1] - p.plan[b]) / per_seq;
    off = p.plan[b] + hh * n;
  } else {
    n = p.nq + p.nr;
    N = p.n_pairs * n;
    off = pair * n;
  }
  const int W = (N + p.ncta - 1) / p.ncta;
  for (int j = 0; j < 8; ++j) {
    const int hl = hg * 8 + j;
    if (hl >= p.G) break;
    const int hq = hk * p.G + hl;
    float ov = 0.0f, lse = kNegInf;
    if (n > 0) {
      const int c0 = off / W, c1 = (off + n - 1) / W;
      float M = kNegInf;
      for (int cta = c0; cta <= c1; ++cta) M = fmaxf(M, p.part_ml[((size_t)(pair + cta) * 8 + j) * 2]);
      if (M != kNegInf) {
        float L = 0.0f, acc = 0.0f;
        for (int cta = c0; cta <= c1; ++cta) {
          const size_t sl = (size_t)(pair + cta) * 8 + j;
          const float a = exp2f(p.part_ml[sl * 2] - M);
          L = fmaf(a, p.part_ml[sl * 2 + 1], L);
          acc = fmaf(a, p.part_o[sl * kHeadDim + dd], acc);
        }
        ov = acc / L;
        lse = (M + log2f(L)) * 0.69314718055994531f;
      }
    }
    p.out[((size_t)b * p.Hq + hq) * kHeadDim + dd] = ov;
    if (dd == 0 && p.lse) p.lse[(size_t)b * p.Hq + hq] = lse;
  }
}

// ------------------------------------------------------------------ paged plan
// plan[b] = tiles before sequence b (all its pairs), plan[B] = total, plan[B+1+b] = length.
__global__ void __launch_bounds__(1024) plan_kernel(const DecodeParams p) {
  __shared__ int warp_sum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  const int maxlen = p.max_pages * p.page_size;
  const int per_seq = p.Hkv * p.HG;
  for (int base = 0; base < p.B; base += 1024) {
    const int b = base + tid;
    int n = 0;
    if (b < p.B) {
      int L = p.seq_lens[b];
      if (L < 0 || L > maxlen) {
        flag(p.status, KVQ_DEV_BAD_LENGTH);
        L = L < 0 ? 0 : maxlen;
      }
      p.plan[p.B + 1 + b] = L;
      n = (L + p.ts - 1) / p.ts * per_seq;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sum[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = warp_sum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sum[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int before = (wid ? warp_sum[wid - 1] : 0) + x - n;
    if (b < p.B) p.plan[b] = carry + before;
    __syncthreads();
    if (tid == 0) carry += warp_sum[31];
    __syncthreads();
  }
  if (tid == 0) p.plan[p.B] = carry;
}

// ------------------------------------------------------------------ host side
using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn encoder() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  });
  return fn;
}

bool make_map(CUtensorMap* map, const void* base, int row_bytes_, uint64_t rows, int box_rows) {
  EncodeFn fn = encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes_, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes_};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes_, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes_ == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : row_bytes_ == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_32B;
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Variant {
  int k, v, paged;
  void (*kernel)(const DecodeParams, const CUtensorMap, const CUtensorMap);
  int smem, ts;
};

template <int KS, int VS, bool PG>
Variant variant() {
  using C = Cfg<KS, VS, PG>;
  return Variant{KS, VS, PG ? 1 : 0, decode_kernel<KS, VS, PG>, C::kSmemBytes, C::kTS};
}

const Variant* find_variant(int k, int v, int paged) {
  static const Variant table[] = {
      variant<KVQ_FP8_E4M3_PER_TENSOR, KVQ_FP8_E4M3_PER_TENSOR, false>(),
      variant<KVQ_FP8_E4M3_PER_TENSOR, KVQ_FP8_E4M3_PER_TENSOR, true>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_INT8_SYM_PER_TENSOR, false>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_INT8_SYM_PER_TENSOR, true>(),
      variant<KVQ_INT8_SYM_PER_TOKEN, KVQ_INT8_SYM_PER_TOKEN, false>(),
      variant<KVQ_INT8_SYM_PER_TOKEN, KVQ_INT8_SYM_PER_TOKEN, true>(),
      variant<KVQ_INT8_SYM_PER_CHANNEL, KVQ_INT8_SYM_PER_CHANNEL, false>(),
      variant<KVQ_INT8_SYM_PER_CHANNEL, KVQ_INT8_SYM_PER_CHANNEL, true>(),
      variant<KVQ_UINT8_ASYM_PER_CHANNEL, KVQ_UINT8_ASYM_PER_CHANNEL, false>(),
      variant<KVQ_UINT8_ASYM_PER_CHANNEL, KVQ_UINT8_ASYM_PER_CHANNEL, true>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_UINT8_ASYM_PER_CHANNEL, false>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_UINT8_ASYM_PER_CHANNEL, true>(),
      variant<KVQ_INT8_SYM_PER_CHANNEL, KVQ_UINT8_ASYM_PER_CHANNEL, false>(),
      variant<KVQ_INT8_SYM_PER_CHANNEL, KVQ_UINT8_ASYM_PER_CHANNEL, true>(),
      variant<KVQ_KIVI_INT4, KVQ_KIVI_INT4, false>(),
      variant<KVQ_KIVI_INT2, KVQ_KIVI_INT2, false>(),
  };
  for (const Variant& x : table)
    if (x.k == k && x.v == v && x.paged == paged) return &x;
  return nullptr;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

bool decode_supported(int k_scheme, int v_scheme, int paged) {
  return find_variant(k_scheme, v_scheme, paged) != nullptr;
}

cudaError_t launch_decode(DecodeParams p, cudaStream_t st) {
  const Variant* var = find_variant(p.k_scheme, p.v_scheme, p.paged);
  if (!var) return cudaErrorNotSupported;
  p.ts = var->ts;
  if (!p.paged) {
    p.nq = (p.len_q + var->ts - 1) / var->ts;
    p.nr = is_kivi(p.k_scheme) ? (p.len_res + kRT - 1) / kRT : 0;
  } else {
    p.nq = p.nr = 0;
  }
  cudaError_t e = cudaFuncSetAttribute(var->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, var->smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, var->kernel, kThreads, var->smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  int ncta = sm_count() * occ;
  if (ncta > kMaxCtas) ncta = kMaxCtas;
  if (!p.paged) {
    const long long N = (long long)p.n_pairs * (p.nq + p.nr);
    if (N < ncta) ncta = N > 0 ? (int)N : 1;
  }
  p.ncta = ncta;
  CUtensorMap tk, tv;
  const int kr = row_bytes(p.k_scheme), vr = row_bytes(p.v_scheme);
  const uint64_t rows = p.paged ? (uint64_t)p.num_pages * p.Hkv * p.page_size : (uint64_t)p.B * p.Hkv * p.cap;
  const int box = p.paged ? p.page_size : var->ts;
  if (!make_map(&tk, p.k_codes, kr, rows, box) || !make_map(&tv, p.v_codes, vr, rows, box))
    return cudaErrorInvalidValue;
  if (p.paged) plan_kernel<<<1, 1024, 0, st>>>(p);
  var->kernel<<<ncta, kThreads, var->smem, st>>>(p, tk, tv);
  merge_kernel<<<p.n_pairs, 128, 0, st>>>(p);
  count_launches(p.paged ? 3 : 2);
  return cudaGetLastError();
}

}  // namespace kvq

// Split-KV decode attention over the quantized cache (sm_100a).
//
// One CTA = 4 consumer warps + 1 producer warp (dense KIVI: the consumer warps refill the
// stages themselves, see Cfg::kSelfFed). The grid is a persistent-style set of
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
// Codes stay exact (every E4M3, E5M2, int8, uint8 - zp, INT4 and INT2 value is an f16 value);
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

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kCW = 4;                  // consumer warps
constexpr int kRT = 32;                 // residual tile tokens (bf16 rows)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();

enum { FMT_E4M3, FMT_E5M2, FMT_S8, FMT_U8, FMT_U4, FMT_U2, FMT_S4 };
// FOLD_GROUP: one scale per (token, 32-channel group), for keys and values (INT4 per group)
enum { FOLD_TENSOR, FOLD_TOKEN, FOLD_CHANNEL, FOLD_KIVI, FOLD_GROUP };

__host__ __device__ constexpr int fmt_of(int s) {
  return s == KVQ_FP8_E4M3_PER_TENSOR      ? FMT_E4M3
         : s == KVQ_FP8_E5M2_PER_TENSOR    ? FMT_E5M2
         : s == KVQ_UINT8_ASYM_PER_CHANNEL ? FMT_U8
         : (s == KVQ_KIVI_INT4 || s == KVQ_KIVI_INT4_F16) ? FMT_U4
         : (s == KVQ_KIVI_INT2 || s == KVQ_KIVI_INT2_F16) ? FMT_U2
         : s == KVQ_INT4_SYM_PER_GROUP     ? FMT_S4
                                           : FMT_S8;
}
__host__ __device__ constexpr int fold_of(int s) {
  return (s == KVQ_FP8_E4M3_PER_TENSOR || s == KVQ_FP8_E5M2_PER_TENSOR || s == KVQ_INT8_SYM_PER_TENSOR)
             ? FOLD_TENSOR
         : s == KVQ_INT8_SYM_PER_TOKEN                                          ? FOLD_TOKEN
         : (s == KVQ_INT8_SYM_PER_CHANNEL || s == KVQ_UINT8_ASYM_PER_CHANNEL) ? FOLD_CHANNEL
         : s == KVQ_INT4_SYM_PER_GROUP                                          ? FOLD_GROUP
                                                                                : FOLD_KIVI;
}
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int rup(int a, int m) { return (a + m - 1) / m * m; }

// NG: scales per token row of an INT4 per-group side (4, 2 or 1 for groups of 32, 64, 128)
// ROPE: keys cached before RoPE (8-bit codes), rotated at their positions in the kernel
template <int KS, int VS, bool PAGED, int NG = 4, bool ROPE = false>
struct Cfg {
  static constexpr bool kPaged = PAGED;
  static constexpr int kNG = NG;
  static constexpr bool kRope = ROPE;
  static_assert(!ROPE || (row_bytes(KS) == kHeadDim && fold_of(KS) != FOLD_GROUP), "RoPE keys: 8-bit codes");
  static constexpr int kKFmt = fmt_of(KS), kVFmt = fmt_of(VS);
  static constexpr int kKFold = fold_of(KS), kVFold = fold_of(VS);
  static constexpr bool kKivi = kKFold == FOLD_KIVI;
  // KIVI scale and minimum stored as fp16 (2 bytes per element instead of 4)
  static constexpr bool kHalfMeta = kivi_f16(KS);
  static constexpr int kMetaElem = kHalfMeta ? 2 : 4;
  // values with one scale per (token, 32-channel group): KIVI and INT4 per group
  static constexpr bool kGroupV = kVFold == FOLD_KIVI || kVFold == FOLD_GROUP;
  // 32 tokens per consumer warp per tile: two independent 16-token MMA chains per warp, and
  // the per-tile bookkeeping and softmax reductions shared by twice the tokens
  static constexpr int kTPW = 32;
  static constexpr int kNSub = kTPW / 16;
  static constexpr int kTS = kTPW * kCW;        // tokens per quantized tile
  static constexpr int kKRow = row_bytes(KS), kVRow = row_bytes(VS);
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTS * kKRow;     // multiple of 1024 (swizzle atom)
  static constexpr int kOffKM = kOffV + kTS * kVRow;
  static constexpr int kKMeta = kKivi ? (kTS / 32) * kHeadDim * kMetaElem * 2
                                : (kKFold == FOLD_TOKEN ? kTS * 4 : (kKFold == FOLD_GROUP ? kTS * NG * 4 : 0));
  static constexpr int kOffVM = kOffKM + kKMeta;
  static constexpr int kVMeta = kKivi ? kTS * 4 * kMetaElem * 2
                                : (kVFold == FOLD_TOKEN ? kTS * 4 : (kVFold == FOLD_GROUP ? kTS * NG * 4 : 0));
  static constexpr int kQuantBytes = kOffVM + kVMeta;
  static constexpr int kResBytes = kKivi ? 2 * kRT * kHeadDim * 2 : 0;
  static constexpr int kStageBytes = rup(cmax(kQuantBytes, kResBytes), 1024);
  // RoPE: the inverse frequencies (64 fp64), each warp's (base angle, frequency) pairs (64 float2)
  // and the kv head's per-channel key scales (128 fp32)
  static constexpr int kRopeBytes = ROPE ? 64 * 8 + kCW * 64 * 8 + kHeadDim * 4 : 0;
  // Shared memory of a CTA with `stages` tile stages and `mh` heads staged per pass of the
  // per-pair warp merge (the layout below, plus 1 KB of alignment slack).
  static constexpr int smem_for(int stages, int mh) {
    return stages * kStageBytes + stages * 64 + 2 * stages * 8 + 64 + kCW * mh * kHeadDim * 4 + kCW * 8 * 4 * 2 +
           kCW * mh * 4 * 4 + 8 * 144 * 4 + kRopeBytes + 1024;
  }
  static constexpr int kSmPerSm = 228 * 1024;  // shared memory of an SM (1 KB of it reserved per CTA)
  static constexpr bool fits(int ctas, int stages, int mh) { return ctas * (smem_for(stages, mh) + 1024) <= kSmPerSm; }
  // Dense KIVI: no producer warp. The consumer warps refill the stages themselves (the last
  // warp to release a stage issues its next tile), so three CTAs of four warps fit on an SM at
  // the same 168 registers a thread. The other kernels keep a producer warp and two CTAs per SM
  // (three self-fed CTAs of two stages were slower for FP8 and INT4 per group).
  static constexpr bool kSelfFed = kKivi && !PAGED;
  // 8-bit keys: a pair's query loads are issued before the wait for its first tile (and the
  // queries are prefetched toward L2 when that tile is issued); measured slower for KIVI and
  // INT4 per group, whose pair start is cheaper than the registers the overlap costs them
  static constexpr bool kEarlyPairStart = !kKivi && kKFold != FOLD_GROUP;
  // may start while the one-token append of the same step runs (dense, producer warp, codes and
  // their per-token / per-group scales all reach the consumers through the stages)
  static constexpr bool kOverlapAppend = !PAGED && !kSelfFed;
  static constexpr int kThreadsCta = kSelfFed ? kCW * 32 : (kCW + 1) * 32;
  static constexpr int kMinBlocks = kSelfFed ? 3 : 2;  // resident CTAs per SM the registers are sized for
  static constexpr int kStages = kSelfFed ? (fits(3, 3, 4) ? 3 : 2) : (fits(2, 3, 4) ? 3 : 2);
  static constexpr int kMergeHeads = (kSelfFed && !fits(3, kStages, 4)) ? 2 : 4;
  static constexpr int kOffDesc = kStages * kStageBytes;
  static constexpr int kOffBar = kOffDesc + kStages * 64;
  static constexpr int kOffRedO = kOffBar + 2 * kStages * 8 + 64;
  static constexpr int kOffRedM = kOffRedO + kCW * kMergeHeads * kHeadDim * 4;
  static constexpr int kOffRedL = kOffRedM + kCW * 8 * 4;
  static constexpr int kOffRedZ = kOffRedL + kCW * 8 * 4;
  static constexpr int kOffQ = kOffRedZ + kCW * kMergeHeads * 4 * 4;
  static constexpr int kQStride = 144;          // q row stride (floats): see q_off
  static constexpr int kOffRope = kOffQ + 8 * kQStride * 4;  // 8-byte aligned
  static constexpr int kSmemBytes = kOffRope + kRopeBytes + 1024;  // + alignment slack
  static_assert(kSmemBytes <= smem_for(kStages, kMergeHeads), "layout within its accounting");
  static_assert(kMinBlocks * (kSmemBytes + 1024) <= kSmPerSm, "the resident CTAs must fit in shared memory");
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

// Walks a CTA's contiguous range of the flattened tile list without per-tile divisions.
struct TileIter {
  int t, tb, te;
  int b, hh, j, npt;  // sequence, (kv head, head group) index in the sequence, tile in pair, tiles per pair
  int L;              // paged: sequence length

  __device__ __forceinline__ void init(const DecodeParams& p, const Sched& s, int tb_, int te_) {
    t = tb = tb_;
    te = te_;
    L = 0;
    if (p.paged) {
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.plan[mid] <= t) lo = mid; else hi = mid - 1;
      }
      b = lo;
      npt = (p.plan[lo + 1] - p.plan[lo]) / s.per_seq;
      const int local = t - p.plan[lo];
      hh = local / npt;
      j = local % npt;
      L = p.plan[p.B + 1 + lo];
    } else {
      npt = p.nq + p.nr;
      const int pair = t / npt;
      j = t % npt;
      b = pair / s.per_seq;
      hh = pair % s.per_seq;
    }
  }

  __device__ __forceinline__ void next(const DecodeParams& p, const Sched& s) {
    ++t;
    if (++j < npt) return;
    j = 0;
    if (++hh < s.per_seq) return;
    hh = 0;
    ++b;
    if (p.paged && t < te) {
      while ((npt = (p.plan[b + 1] - p.plan[b]) / s.per_seq) == 0) ++b;  // skip empty sequences
      L = p.plan[p.B + 1 + b];
    }
  }

  __device__ __forceinline__ TileDesc desc(const DecodeParams& p, const Sched& s) const {
    TileDesc d;
    d.b = b;
    d.pair = b * s.per_seq + hh;
    if (p.HG == 1) {
      d.hk = hh;
      d.hg = 0;
    } else {
      d.hk = hh / p.HG;
      d.hg = hh - d.hk * p.HG;
    }
    if (p.paged) {
      d.kind = 0;
      d.t0 = j * p.ts;
      d.n = min(p.ts, L - d.t0);
    } else if (j < p.nq) {
      d.kind = 0;
      d.t0 = j * p.ts;
      d.n = min(p.ts, p.len_q - d.t0);
    } else {
      d.kind = 1;
      d.t0 = (j - p.nq) * kRT;
      d.n = min(kRT, p.len_res - d.t0);
    }
    d.first = (t == tb) || (j == 0);
    d.last = (t == te - 1) || (j == npt - 1);
    d.valid = 0xFFFFFFFFu;
    return d;
  }
};

// ------------------------------------------------------------------ TMA
// The cache is streamed once per decode: its tiles are copied with an L2 evict-first policy,
// so they do not push out what is read again (the split partials, the queries).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar,
                                       uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s_ef(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
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
// Issue the copies of tile d into stage `cur`: its descriptor, the expected transaction bytes
// on the stage's full barrier, then 2-D TMA boxes of codes and 1-D bulk copies of metadata (or
// the bf16 residual rows).
template <class C>
__device__ void issue_tile(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                           const CUtensorMap* tks, const CUtensorMap* tkz, uint8_t* stages, TileDesc* descs,
                           uint32_t full0, int cur, TileDesc d, const int (&pages)[C::kTS / 16]) {
  const uint32_t sb = smem_addr(stages + cur * C::kStageBytes);
  const uint32_t bar = full0 + 8 * cur;
  const uint64_t pol = l2_evict_first();
  if (C::kEarlyPairStart && d.first) {  // the pair's queries toward L2, a few tiles before they are loaded
    const int h0 = d.hg * 8, nh = min(8, p.G - h0);
    const size_t es = p.q_bf16 ? 2 : 4;
    const uint8_t* qrow = static_cast<const uint8_t*>(p.q) + ((size_t)d.b * p.Hq + (size_t)d.hk * p.G + h0) * kHeadDim * es;
    if ((reinterpret_cast<uintptr_t>(qrow) & 15) == 0) bulk_prefetch_l2(qrow, (uint32_t)(nh * kHeadDim * es));
  }
  const size_t pair_row = (size_t)d.b * p.Hkv + d.hk;
  if (d.kind == 1) {  // KIVI residual: bf16 rows, whole 32-token slab (inside rcap)
    const size_t r0 = (pair_row * p.rcap + d.t0) * kHeadDim;
    descs[cur] = d;
    mbar_arrive_expect_tx(bar, 2 * kRT * kHeadDim * 2);
    bulk_g2s_ef(sb, p.k_res + r0, kRT * kHeadDim * 2, bar, pol);
    bulk_g2s_ef(sb + kRT * kHeadDim * 2, p.v_res + r0, kRT * kHeadDim * 2, bar, pol);
    return;
  }
  if constexpr (!C::kPaged) {
    // whole tile: capacity is a multiple of 128 tokens, so the tile lies inside the row
    const size_t row0 = pair_row * p.cap + d.t0;
    const uint32_t bytes = C::kTS * (C::kKRow + C::kVRow) + C::kKMeta + C::kVMeta;
    descs[cur] = d;
    mbar_arrive_expect_tx(bar, bytes);
    tma_2d(sb + C::kOffK, tk, 0, (int)row0, bar, pol);
    tma_2d(sb + C::kOffV, tv, 0, (int)row0, bar, pol);
    if constexpr (C::kKivi) {
      const size_t g0 = (pair_row * (p.cap / 32) + d.t0 / 32) * kHeadDim;
      // element offsets in bytes: fp32 or fp16 metadata
      const uint8_t* vs8 = reinterpret_cast<const uint8_t*>(p.v_scale);
      const uint8_t* vz8 = reinterpret_cast<const uint8_t*>(p.v_zero);
      // key scales and minima as 128-byte rows through TMA with the 128-byte swizzle, so the query
      // build's reads (four lanes a 128-byte row apart) fall in distinct banks
      const int krow = (int)(g0 * C::kMetaElem / 128);
      tma_2d(sb + C::kOffKM, tks, 0, krow, bar, pol);
      tma_2d(sb + C::kOffKM + C::kKMeta / 2, tkz, 0, krow, bar, pol);
      bulk_g2s_ef(sb + C::kOffVM, vs8 + row0 * 4 * C::kMetaElem, C::kVMeta / 2, bar, pol);
      bulk_g2s_ef(sb + C::kOffVM + C::kVMeta / 2, vz8 + row0 * 4 * C::kMetaElem, C::kVMeta / 2, bar, pol);
    } else {
      if constexpr (C::kKFold == FOLD_TOKEN) bulk_g2s_ef(sb + C::kOffKM, p.k_scale + row0, C::kKMeta, bar, pol);
      if constexpr (C::kVFold == FOLD_TOKEN) bulk_g2s_ef(sb + C::kOffVM, p.v_scale + row0, C::kVMeta, bar, pol);
      if constexpr (C::kKFold == FOLD_GROUP) bulk_g2s_ef(sb + C::kOffKM, p.k_scale + row0 * C::kNG, C::kKMeta, bar, pol);
      if constexpr (C::kVFold == FOLD_GROUP) bulk_g2s_ef(sb + C::kOffVM, p.v_scale + row0 * C::kNG, C::kVMeta, bar, pol);
    }
  } else {
    // paged: page i of the tile -> rows (page * Hkv + hk) * page_size of the pool
    const int ps = p.page_size;
    const int npg = (d.n + ps - 1) / ps;
    int page[C::kTS / 16];
    uint32_t valid = 0, nvalid = 0;
#pragma unroll
    for (int i = 0; i < C::kTS / 16; ++i) {
      page[i] = -1;
      if (i < npg) {
        const int id = pages[i];  // read from the page table one tile ahead (load_tile_pages)
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
    descs[cur] = d;
    uint32_t per_page = ps * (C::kKRow + C::kVRow);
    if constexpr (C::kKFold == FOLD_TOKEN) per_page += ps * 4;
    if constexpr (C::kVFold == FOLD_TOKEN) per_page += ps * 4;
    if constexpr (C::kKFold == FOLD_GROUP) per_page += ps * C::kNG * 4;
    if constexpr (C::kVFold == FOLD_GROUP) per_page += ps * C::kNG * 4;
    mbar_arrive_expect_tx(bar, nvalid * per_page);
#pragma unroll
    for (int i = 0; i < C::kTS / 16; ++i) {
      if (i >= npg || !((valid >> i) & 1u)) continue;
      const size_t prow = ((size_t)page[i] * p.Hkv + d.hk) * ps;
      tma_2d(sb + C::kOffK + i * ps * C::kKRow, tk, 0, (int)prow, bar, pol);
      tma_2d(sb + C::kOffV + i * ps * C::kVRow, tv, 0, (int)prow, bar, pol);
      if constexpr (C::kKFold == FOLD_TOKEN) bulk_g2s_ef(sb + C::kOffKM + i * ps * 4, p.k_scale + prow, ps * 4, bar, pol);
      if constexpr (C::kVFold == FOLD_TOKEN) bulk_g2s_ef(sb + C::kOffVM + i * ps * 4, p.v_scale + prow, ps * 4, bar, pol);
      if constexpr (C::kKFold == FOLD_GROUP)
        bulk_g2s_ef(sb + C::kOffKM + i * ps * C::kNG * 4, p.k_scale + prow * C::kNG, ps * C::kNG * 4, bar, pol);
      if constexpr (C::kVFold == FOLD_GROUP)
        bulk_g2s_ef(sb + C::kOffVM + i * ps * C::kNG * 4, p.v_scale + prow * C::kNG, ps * C::kNG * 4, bar, pol);
    }
  }
}

// Paged: the page ids of tile d's pages (ids outside the table read as -1; validated when
// the tile is issued). Called one tile ahead, so the loads overlap the wait for a free stage.
template <class C>
__device__ __forceinline__ void load_tile_pages(const DecodeParams& p, const TileDesc& d, int (&pages)[C::kTS / 16]) {
  const int ps = p.page_size;
  const int npg = (d.n + ps - 1) / ps;
  const int pi0 = d.t0 / ps;
#pragma unroll
  for (int i = 0; i < C::kTS / 16; ++i) {
    const int pi = pi0 + i;
    pages[i] = (i < npg && pi < p.max_pages) ? p.page_table[(size_t)d.b * p.max_pages + pi] : -1;
  }
}

// The producer warp's loop (one elected lane): each stage is refilled once the consumer warps
// have released it.
template <class C>
__device__ void producer(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                         const CUtensorMap* tks, const CUtensorMap* tkz, uint8_t* stages, TileDesc* descs,
                         uint32_t full0, uint32_t empty0, const Sched& s, int tb, int te) {
  TileIter ti;
  ti.init(p, s, tb, te);
  bool waited = !C::kOverlapAppend || p.early_from < 0;
  int pages[C::kTS / 16];
  TileDesc d;
  if (ti.t < te) {
    d = ti.desc(p, s);
    if constexpr (C::kPaged) load_tile_pages<C>(p, d, pages);
  }
  for (int it = 0, st = 0, phase = 0; ti.t < te; ++it) {
    if (it >= C::kStages && !mbar_wait(empty0 + 8 * st, phase ^ 1, p.status)) return;
    if (!waited && d.t0 + p.ts > p.early_from) {  // this tile holds positions the append writes
      grid_dependency_wait();
      waited = true;
    }
    const int cur = st;
    if (++st == C::kStages) {
      st = 0;
      phase ^= 1;
    }
    issue_tile<C>(p, tk, tv, tks, tkz, stages, descs, full0, cur, d, pages);
    ti.next(p, s);
    if (ti.t < te) {  // the next tile's descriptor and (paged) page ids, ahead of its stage
      d = ti.desc(p, s);
      if constexpr (C::kPaged) load_tile_pages<C>(p, d, pages);
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

// Bytes 0,1 (lo) and 2,3 (hi) of a word of 8-bit codes -> two f16x2 of the code values.
template <int FMT>
__device__ __forceinline__ void cvt8x4(uint32_t w, uint32_t zlo, uint32_t zhi, uint32_t& lo, uint32_t& hi) {
  if constexpr (FMT == FMT_E4M3) {
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n cvt.rn.f16x2.e4m3x2 %0, l;\n cvt.rn.f16x2.e4m3x2 %1, h;\n}\n"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
  } else if constexpr (FMT == FMT_E5M2) {  // an E5M2 byte is the high byte of the equal f16
    lo = prmt(w, 0u, 0x1404u);
    hi = prmt(w, 0u, 0x3424u);
  } else if constexpr (FMT == FMT_S8) {  // word already XORed with 0x80808080: codes biased by 128
    lo = hsub2_u(prmt(w, 0x64646464u, 0x5150u), 0x64806480u);  // (1024 + 128 + q) - 1152
    hi = hsub2_u(prmt(w, 0x64646464u, 0x5352u), 0x64806480u);
  } else {  // FMT_U8: subtract 1024 + zero point
    lo = hsub2_u(prmt(w, 0x64646464u, 0x5150u), zlo);
    hi = hsub2_u(prmt(w, 0x64646464u, 0x5352u), zhi);
  }
}

// Nibble pairs of a 32-bit word: k = 0..3 -> (nibble k, nibble k + 4).
__device__ __forceinline__ uint32_t u4_pair(uint32_t w, int k) {
  const uint32_t x = (k & 2) ? (w >> 8) : w;
  if (k & 1) return hfma2_u(and_or(x, 0x00F000F0u, kF16Magic1024x2), 0x2C002C00u, 0xD400D400u);  // /16 - 64
  return hsub2_u(and_or(x, 0x000F000Fu, kF16Magic1024x2), kF16Magic1024x2);
}

// Signed (two's-complement) nibbles: XOR with 8 turns a code n into n + 8, which the LOP3 does
// while it places the nibble under the f16 magic number; the offsets then remove 8 more than
// in the unsigned form. Nibble pairs of a word as in u4_pair.
__device__ __forceinline__ uint32_t s4_pair(uint32_t w, int k) {
  const uint32_t x = (k & 2) ? (w >> 8) : w;
  if (k & 1) return hfma2_u(and_xor(x, 0x00F000F0u, 0x64806480u), 0x2C002C00u, 0xD480D480u);  // /16 - 72
  return hsub2_u(and_xor(x, 0x000F000Fu, 0x64086408u), 0x64086408u);                            // - 1032
}

// Byte `sel` selects (0x4040 + 0x101 c) of a word of signed nibbles -> f16x2 of its two
// channels (low nibble, high nibble).
__device__ __forceinline__ uint32_t s4_byte(uint32_t w, uint32_t sel) {
  return hfma2_u(and_xor(prmt(w, 0u, sel), 0x00F0000Fu, 0x64806408u), 0x2C003C00u, 0xD480E408u);
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

// Two bf16 values times the power of two f, as f16x2 (exact when the products lie in the f16
// range with their 8 significant bits).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float f) {
  return float2_to_f16x2(__uint_as_float(w << 16) * f, __uint_as_float(w & 0xFFFF0000u) * f);
}

// Power-of-two exponent that brings a bf16 residual row into the f16 range: lane i scans row i
// (256-byte rows of 128 bf16 values at `row0`; rows >= n are empty) and returns the range shift
// of the row's largest magnitude (0 for a zero row). Each lane starts at its own 16-byte chunk
// so the 32 rows' loads spread over the banks.
__device__ __forceinline__ int residual_row_shift(const uint8_t* row0, int n, int lane) {
  uint32_t m = 0u;
  if (lane < n) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const uint4 v = *reinterpret_cast<const uint4*>(row0 + lane * 256 + (((q + lane) & 15) << 4));
      m = __vmaxu2(m, __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu));
      m = __vmaxu2(m, __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    }
  }
  const uint32_t top = max(m & 0xFFFFu, m >> 16);  // bf16 magnitudes order like their bits
  return top ? range_shift(bf16_bits_to_float(top)) : 0;
}

template <class T>
__device__ __forceinline__ T lds(const uint8_t* p) {
  return *reinterpret_cast<const T*>(p);
}

// A shared-memory load the compiler keeps where it is written (loop-invariant values it would
// otherwise hoist into registers for the whole loop).
__device__ __forceinline__ float2 lds_here_f2(const void* p) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(smem_addr(p)));
  return v;
}
__device__ __forceinline__ float lds_here_f(const void* p) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_addr(p)));
  return v;
}

// Four 8x8 matrices of 16-bit elements, transposed: lane 8m + r supplies the shared address of
// row r of matrix m; the thread with row group g and column group c receives, for each m,
// elements (row 2c, column g) in its low half and (row 2c + 1, column g) in its high half.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

// Column of channel dd of head `head` in the merge staging rows: an XOR within the channel's
// aligned group of 16 (8-bit layout) or 4 (KIVI layout) so that the accumulator stores of a warp
// (lanes spread over heads 2c and channels 16g or 4g) and the merge's channel-order reads both
// touch 32 distinct banks.
template <bool kKivi>
__device__ __forceinline__ int red_col(int dd, int head) {
  const int c = (head >> 1) & 3;
  return dd ^ (kKivi ? c : (c | (((dd >> 5) & 3) << 2)));
}

// ------------------------------------------------------------------ consumer state
template <class C>
struct Consumer {
  int w, g, c;
  float o[8][4];
  float m[2], l[2];
  int ev;            // O accumulator holds (true value) * 2^ev
  bool ev_set;
  float zacc[4];     // KIVI: sum p * min per channel group, head g
  uint32_t qh[8][2], ql[8][2];
  bool qsplit;
  float kmul;        // score multiplier (log2 domain)
  float bias[2];     // KIVI group bias (raw units), heads 2c, 2c+1
  float qabs;        // KIVI: the largest |q| of the pair's staged queries (all heads)
  int qmode;         // 0: fragments for codes built, 1: for bf16 residual rows
  uint32_t zpk[8][2], zpv[8][2];  // uint8 asymmetric: f16x2 (1024 + zero point)
};

// Staged query rows: head j, channel d at j * 144 + d + 4 * (d >> 5). Each 32-channel block
// starts on a 16-byte boundary, so a lane reads its block with eight 128-bit loads, and the
// lanes of a quarter warp (two heads, four blocks) cover all 32 banks.
__device__ __forceinline__ int q_off(int j, int d) { return j * 144 + d + 4 * (d >> 5); }

// Shared memory after the query staging, in kernels for keys cached before RoPE: the 64 inverse
// frequencies (fp64), each consumer warp's 64 (base angle, frequency) pairs of its current tile,
// and the kv head's 128 per-channel key scales.
__device__ __forceinline__ double* rope_theta_s(const float* q_s) {
  return reinterpret_cast<double*>(const_cast<float*>(q_s) + 8 * 144);
}
__device__ __forceinline__ float2* rope_angles(const float* q_s) {
  return reinterpret_cast<float2*>(rope_theta_s(q_s) + 64);
}
__device__ __forceinline__ float* rope_key_scales(const float* q_s) {
  return reinterpret_cast<float*>(rope_angles(q_s) + kCW * 64);
}

// Elements 4i .. 4i + 3 of a metadata array of fp32 or (kHalf) fp16 values, as fp32.
template <bool kHalf>
__device__ __forceinline__ float4 meta4(const void* base, int i) {
  if constexpr (kHalf) {
    const uint2 u = reinterpret_cast<const uint2*>(base)[i];
    const float2 a = f16x2_to_float2(u.x), b = f16x2_to_float2(u.y);
    return make_float4(a.x, a.y, b.x, b.y);
  } else {
    return reinterpret_cast<const float4*>(base)[i];
  }
}

// Elements 4i .. 4i + 3 (fp32, or fp16 when kHalf) of KIVI key group `grp` in a stage region the
// producer filled by TMA as 128-byte rows with the 128-byte swizzle (16-byte chunk index XOR row).
template <bool kHalf>
__device__ __forceinline__ float4 kmeta4_swz(const void* region, int grp, int i) {
  constexpr int es = kHalf ? 2 : 4;
  const int b = grp * kHeadDim * es + i * 4 * es;  // byte offset before the swizzle
  const int row = b >> 7, within = b & 127;
  const uint8_t* a = static_cast<const uint8_t*>(region) + swz<128>(row, within >> 4) + (within & 15);
  if constexpr (kHalf) {
    const uint2 u = *reinterpret_cast<const uint2*>(a);
    const float2 x = f16x2_to_float2(u.x), y = f16x2_to_float2(u.y);
    return make_float4(x.x, x.y, y.x, y.y);
  } else {
    return *reinterpret_cast<const float4*>(a);
  }
}

// Build Q' fragments (head g, this thread's 32 channels 32c..32c+31) from q_s, optionally
// multiplied by a per-channel fold; with `zmin` also returns sum_d q_d * zmin_d over those
// channels (the KIVI key-minimum term). fold and zmin hold fp32, or fp16 when kHalf. The
// power-of-two shift applied to Q' (returned) comes from the largest |q'| of the warp, or is
// given (kGivenShift: from a bound on |q'|, which skips that pass).
// kSwz: fold and zmin are swizzled KIVI key-metadata regions (kmeta4_swz) of group `grp`.
template <int FMT, bool kHalf = false, bool kGivenShift = false, bool kSwz = false>
__device__ __forceinline__ int build_q(const float* q_s, const void* fold, const void* zmin, int g, int c,
                                       uint32_t (&qh)[8][2], uint32_t (&ql)[8][2], float* bias = nullptr,
                                       int given_shift = 0, int grp = 0) {
  const float4* qrow = reinterpret_cast<const float4*>(q_s + q_off(g, 32 * c));
  auto meta = [&](const void* base, int i) -> float4 {
    if constexpr (kSwz) return kmeta4_swz<kHalf>(base, grp, 8 * c + i);
    return meta4<kHalf>(base, 8 * c + i);
  };
  int eq = given_shift;
  if constexpr (!kGivenShift) {
    // pass 1: the largest |q'| of the warp sets the range shift
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 q4 = qrow[i];
      if (fold) {
        const float4 f4 = meta(fold, i);
        q4.x *= f4.x; q4.y *= f4.y; q4.z *= f4.z; q4.w *= f4.w;
      }
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(q4.x), fabsf(q4.y)), fmaxf(fabsf(q4.z), fabsf(q4.w))));
    }
    mx = warp_max(mx);
    eq = range_shift(mx);
  }
  const float sh = pow2i(eq);
  // pass 2: scaled products by local channel, then the fragment split
  float pl[32];
  float bs = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 q4 = qrow[i];
    float4 m4 = make_float4(sh, sh, sh, sh);
    if (fold) {
      const float4 f4 = meta(fold, i);
      m4 = make_float4(f4.x * sh, f4.y * sh, f4.z * sh, f4.w * sh);
    }
    if (zmin) {
      const float4 z4 = meta(zmin, i);
      bs = fmaf(q4.x, z4.x, fmaf(q4.y, z4.y, fmaf(q4.z, z4.z, fmaf(q4.w, z4.w, bs))));
    }
    pl[4 * i] = q4.x * m4.x;
    pl[4 * i + 1] = q4.y * m4.y;
    pl[4 * i + 2] = q4.z * m4.z;
    pl[4 * i + 3] = q4.w * m4.w;
  }
  if (bias) *bias = bs;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      split_f16x2(pl[dmap_k<FMT>(0, ks, h, 0)], pl[dmap_k<FMT>(0, ks, h, 1)], qh[ks][h], ql[ks][h]);
  return eq;
}

// Q' fragments for INT4 per-group keys: k-step ks covers channels 16 ks .. 16 ks + 15 (one
// half of group ks / 2), slot pair h of column group c holding channels 16 ks + 8 h + 2 c and
// + 1, so every MMA sums one group only. No fold: the group scales multiply the partial sums.
__device__ __forceinline__ int build_q_s4(const float* q_s, int g, int c, uint32_t (&qh)[8][2], uint32_t (&ql)[8][2]) {
  float pl[8][2][2];
  float mx = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 v = *reinterpret_cast<const float2*>(q_s + q_off(g, 16 * ks + 8 * h + 2 * c));
      pl[ks][h][0] = v.x;
      pl[ks][h][1] = v.y;
      mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
    }
  mx = warp_max(mx);
  const int eq = range_shift(mx);
  const float sh = pow2i(eq);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h) split_f16x2(pl[ks][h][0] * sh, pl[ks][h][1] * sh, qh[ks][h], ql[ks][h]);
  return eq;
}

// Q fragments for keys cached before RoPE: lane c holds the rotation pairs i = 16c .. 16c + 15,
// k-step ks and slot pair h holding the two channels (i, i + 64) of pair i = 16c + 2ks + h, so a
// lane rotates a key pair without exchanging values. No fold (per-channel key scales are applied
// to the keys before the rotation). Returns the power-of-two shift applied to Q.
__device__ __forceinline__ int build_q_rope(const float* q_s, int g, int c, uint32_t (&qh)[8][2],
                                            uint32_t (&ql)[8][2]) {
  float pl[8][2][2];
  float mx = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 16 * c + 2 * ks + h;
      pl[ks][h][0] = q_s[q_off(g, i)];
      pl[ks][h][1] = q_s[q_off(g, i + 64)];
      mx = fmaxf(mx, fmaxf(fabsf(pl[ks][h][0]), fabsf(pl[ks][h][1])));
    }
  mx = warp_max(mx);
  const int eq = range_shift(mx);
  const float sh = pow2i(eq);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int h = 0; h < 2; ++h) split_f16x2(pl[ks][h][0] * sh, pl[ks][h][1] * sh, qh[ks][h], ql[ks][h]);
  return eq;
}

// 2 pi as a double-double and 1 / (2 pi): angle reduction of position * frequency
constexpr double kTwoPiHi = 6.283185307179586;
constexpr double kTwoPiLo = 2.4492935982947064e-16;
constexpr double kInvTwoPi = 0.15915494309189535;

// A warp's RoPE angles for one tile: for pair i (frequency theta_i = base^(-2i/128), fp64 in
// shared memory), the angle at the warp's first position pos0 is reduced modulo 2 pi in fp64
// (positions up to 2^31 keep it accurate to ~1e-11 rad at 131072) and kept as fp32 with theta_i
// in fp32; the angle at pos0 + j (j < 32) is then fma(j, theta_i, base_i), within ~2e-6 rad.
__device__ __forceinline__ void rope_warp_angles(const double* theta, float2* rw, int pos0, int lane) {
  __syncwarp();  // the previous tile's reads of rw are done
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int i = 2 * lane + k;
    const double a = (double)pos0 * theta[i];
    const double n = rint(a * kInvTwoPi);
    const double r = fma(-n, kTwoPiLo, fma(-n, kTwoPiHi, a));
    rw[i] = make_float2((float)r, (float)theta[i]);
  }
  __syncwarp();
}

// The value scales of token tok for the four 32-channel blocks of a row (KIVI, INT4 per group;
// groups of 64 or 128 channels repeat each scale over the blocks they cover).
template <class C>
__device__ __forceinline__ float4 vscale4(const uint8_t* base, int tok) {
  if constexpr (C::kKivi) {
    return meta4<C::kHalfMeta>(base + C::kOffVM, tok);
  } else if constexpr (C::kNG == 4) {
    return lds<float4>(base + C::kOffVM + tok * 16);
  } else if constexpr (C::kNG == 2) {
    const float2 s = lds<float2>(base + C::kOffVM + tok * 8);
    return make_float4(s.x, s.x, s.y, s.y);
  } else {
    const float s = lds<float>(base + C::kOffVM + tok * 4);
    return make_float4(s, s, s, s);
  }
}

// ------------------------------------------------------------------ one tile, one warp
// kMasked: the warp's tokens are not all valid (ragged tail or missing pages). kResidual: a tile
// of KIVI's bf16 residual rows (a separate instantiation, so the code tiles' path carries none
// of the residual work).
template <class C, bool kMasked, bool kResidual>
__device__ __forceinline__ void warp_tile(Consumer<C>& S, const DecodeParams& p, const uint8_t* base,
                                          const TileDesc& d, uint32_t valid, int tok_base, float sc_log2,
                                          const float* q_s) {
  constexpr bool residual = kResidual;
  const int g = S.g, c = S.c, w = S.w;
  // validity of a token of this warp's range (tile-relative index)
  auto tok_ok = [&](int tok) -> bool {
    if constexpr (!kMasked) return true;
    bool ok = tok < d.n;
    if constexpr (C::kPaged) ok = ok && ((valid >> (tok / p.page_size)) & 1u);
    return ok;
  };

  // bf16 residual rows (warp 0 alone) are brought into the f16 range row by row: lane i holds the
  // power-of-two exponents of key row i and value row i; scores and probabilities take the
  // inverse factors, so the products are unchanged and every bf16 value stays exact
  int res_kx = 0, res_vx = 0;
  if (C::kKivi && residual) {
    res_kx = residual_row_shift(base, d.n, 4 * g + c);
    res_vx = residual_row_shift(base + kRT * kHeadDim * 2, d.n, 4 * g + c);
  }

  // (1) per-tile state: RoPE angles at the warp's positions; query fragments that change per
  // tile (KIVI key groups, residual rows)
  if constexpr (C::kRope) rope_warp_angles(rope_theta_s(q_s), rope_angles(q_s) + w * 64, d.t0 + tok_base, 4 * g + c);
  if constexpr (C::kKivi) {
    if (!residual) {
      // the tile's key scales and minima: swizzled 128-byte rows, group w is this warp's
      const uint8_t* ksm = base + C::kOffKM;
      const uint8_t* kzm = base + C::kOffKM + C::kKMeta / 2;
      // range shift of the group's Q' = q * s from the bound max|q| * max s (one 4-scale load a
      // lane instead of a pass over the 32 products): Q' stays below 2^15, and its smaller
      // values keep their ~22 bits in the hi + lo split while within 2^20 of the bound
      const float4 s4 = kmeta4_swz<C::kHalfMeta>(ksm, w, 4 * g + c);
      const float sgrp = warp_max(fmaxf(fmaxf(s4.x, s4.y), fmaxf(s4.z, s4.w)));
      float bs;
      const int eq = build_q<C::kKFmt, C::kHalfMeta, true, true>(q_s, ksm, kzm, g, c, S.qh, S.ql, &bs,
                                                                  range_shift(S.qabs * sgrp), w);
      bs += __shfl_xor_sync(0xffffffffu, bs, 1);
      bs += __shfl_xor_sync(0xffffffffu, bs, 2);
      S.bias[0] = __shfl_sync(0xffffffffu, bs, 4 * (2 * c));
      S.bias[1] = __shfl_sync(0xffffffffu, bs, 4 * (2 * c + 1));
      S.kmul = pow2i(-eq);
      S.qsplit = true;
      S.qmode = 0;
    } else if (S.qmode != 1) {
      const int eq = build_q<FMT_S8>(q_s, nullptr, nullptr, g, c, S.qh, S.ql);
      S.kmul = sc_log2 * pow2i(-eq);
      S.qsplit = !p.q_bf16;
      S.qmode = 1;
    }
  }

  // (2) S^T = K . Q'^T for kNSub blocks of 16 tokens; two accumulators halve the MMA chain
  float acc[C::kNSub][4];
  float res_kinv[C::kNSub][2];  // residual: 2^-shift of the lane's key rows g and g + 8
#pragma unroll
  for (int sb = 0; sb < C::kNSub; ++sb) {
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
    const int r0 = tok_base + sb * 16 + g, r1 = r0 + 8;
    auto mma2 = [&](int ks, uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, bool split) {
      float(&acc_k)[4] = (ks & 1) ? a1 : a0;
      mma_16816(acc_k, x0, x1, x2, x3, S.qh[ks][0], S.qh[ks][1]);
      if (split) mma_16816(acc_k, x0, x1, x2, x3, S.ql[ks][0], S.ql[ks][1]);
    };
    if (residual) {
      const uint8_t* kr = base;  // bf16 rows of 256 bytes
      uint32_t w0[16], w1[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 x = lds<uint4>(kr + r0 * 256 + c * 64 + i * 16);
        const uint4 y = lds<uint4>(kr + r1 * 256 + c * 64 + i * 16);
        w0[4 * i] = x.x; w0[4 * i + 1] = x.y; w0[4 * i + 2] = x.z; w0[4 * i + 3] = x.w;
        w1[4 * i] = y.x; w1[4 * i + 1] = y.y; w1[4 * i + 2] = y.z; w1[4 * i + 3] = y.w;
      }
      const bool split = S.qsplit;
      const int x0 = __shfl_sync(0xffffffffu, res_kx, r0), x1 = __shfl_sync(0xffffffffu, res_kx, r1);
      const float f0 = pow2i(x0), f1 = pow2i(x1);
      res_kinv[sb][0] = pow2i(-x0);
      res_kinv[sb][1] = pow2i(-x1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma2(ks, bf16x2_to_f16x2_scaled(w0[2 * ks], f0), bf16x2_to_f16x2_scaled(w1[2 * ks], f1),
             bf16x2_to_f16x2_scaled(w0[2 * ks + 1], f0), bf16x2_to_f16x2_scaled(w1[2 * ks + 1], f1), split);
    } else if constexpr (C::kKFmt == FMT_U4) {
      const uint4 x = lds<uint4>(base + C::kOffK + swz<64>(r0, c));
      const uint4 y = lds<uint4>(base + C::kOffK + swz<64>(r1, c));
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int i = ks >> 1, k0 = 2 * (ks & 1);
        const uint32_t u = word_of(x, i), v = word_of(y, i);
        mma2(ks, u4_pair(u, k0), u4_pair(v, k0), u4_pair(u, k0 + 1), u4_pair(v, k0 + 1), true);
      }
    } else if constexpr (C::kKFmt == FMT_S4) {
      // whole 64-byte rows g and g + 8; lane c takes byte c of every word, so each k-step
      // covers 16 channels of one 32-channel group and each group's partial sum takes the
      // (token, group) scale before it joins the score
      uint4 x[4], y[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[i] = lds<uint4>(base + C::kOffK + swz<64>(r0, i));
        y[i] = lds<uint4>(base + C::kOffK + swz<64>(r1, i));
      }
      const float* ksc = reinterpret_cast<const float*>(base + C::kOffKM);
      const uint32_t sel = 0x4040u + 0x101u * (uint32_t)c;
      const bool split = S.qsplit;
      constexpr int kSteps = 8 / C::kNG;  // 16-channel k-steps per group
#pragma unroll
      for (int grp = 0; grp < C::kNG; ++grp) {
        float ag[4] = {0.f, 0.f, 0.f, 0.f}, ah[4] = {0.f, 0.f, 0.f, 0.f};  // two chains per group
#pragma unroll
        for (int st2 = 0; st2 < kSteps; ++st2) {
          const int ks = grp * kSteps + st2, ch = ks >> 1, h2 = ks & 1;  // 32-channel chunk, half
          const uint32_t f0 = s4_byte(word_of(x[ch], 2 * h2), sel), f1 = s4_byte(word_of(y[ch], 2 * h2), sel);
          const uint32_t f2 = s4_byte(word_of(x[ch], 2 * h2 + 1), sel);
          const uint32_t f3 = s4_byte(word_of(y[ch], 2 * h2 + 1), sel);
          float(&acc_k)[4] = (kSteps > 2 && (st2 & 1)) ? ah : ag;
          mma_16816(acc_k, f0, f1, f2, f3, S.qh[ks][0], S.qh[ks][1]);
          if (split) mma_16816(acc_k, f0, f1, f2, f3, S.ql[ks][0], S.ql[ks][1]);
        }
        if constexpr (kSteps > 2) {
#pragma unroll
          for (int k = 0; k < 4; ++k) ag[k] += ah[k];
        }
        const float s0 = ksc[r0 * C::kNG + grp], s1 = ksc[r1 * C::kNG + grp];
        float(&dst)[4] = (grp & 1) ? a1 : a0;
        dst[0] = fmaf(s0, ag[0], dst[0]);
        dst[1] = fmaf(s0, ag[1], dst[1]);
        dst[2] = fmaf(s1, ag[2], dst[2]);
        dst[3] = fmaf(s1, ag[3], dst[3]);
      }
    } else if constexpr (C::kKFmt == FMT_U2) {
      const uint2 x = lds<uint2>(base + C::kOffK + swz<32>(r0, c >> 1) + 8 * (c & 1));
      const uint2 y = lds<uint2>(base + C::kOffK + swz<32>(r1, c >> 1) + 8 * (c & 1));
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int i = ks >> 2, k0 = 2 * (ks & 3);
        const uint32_t u = i ? x.y : x.x, v = i ? y.y : y.x;
        mma2(ks, u2_pair(u, k0), u2_pair(v, k0), u2_pair(u, k0 + 1), u2_pair(v, k0 + 1), true);
      }
    } else if constexpr (C::kRope) {
      // keys cached before RoPE: chunk c (channels 16c .. 16c + 15) and chunk 4 + c (their RoPE
      // partners 64 + 16c ..) of rows g and g + 8; each pair is dequantized (per-channel scales
      // here; per-tensor and per-token scales multiply the score), rotated at its position in
      // fp32 and split into f16 hi + lo, which both meet the exact query fragments
      const uint4 xa = lds<uint4>(base + C::kOffK + swz<128>(r0, c));
      const uint4 xb = lds<uint4>(base + C::kOffK + swz<128>(r0, 4 + c));
      const uint4 ya = lds<uint4>(base + C::kOffK + swz<128>(r1, c));
      const uint4 yb = lds<uint4>(base + C::kOffK + swz<128>(r1, 4 + c));
      const float2* rw = rope_angles(q_s) + w * 64;
      const float* kch = rope_key_scales(q_s);
      const float j0 = (float)(r0 - tok_base), j1 = (float)(r1 - tok_base);
      const bool split = S.qsplit;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t wa0 = word_of(xa, q), wb0 = word_of(xb, q), wa1 = word_of(ya, q), wb1 = word_of(yb, q);
        if constexpr (C::kKFmt == FMT_S8) {
          wa0 ^= 0x80808080u; wb0 ^= 0x80808080u; wa1 ^= 0x80808080u; wb1 ^= 0x80808080u;
        }
        uint32_t h[4][2];  // [row r0 A, r0 B, r1 A, r1 B][bytes 0-1, bytes 2-3] as f16x2
        cvt8x4<C::kKFmt>(wa0, S.zpk[q][0], S.zpk[q][1], h[0][0], h[0][1]);
        cvt8x4<C::kKFmt>(wb0, S.zpk[4 + q][0], S.zpk[4 + q][1], h[1][0], h[1][1]);
        cvt8x4<C::kKFmt>(wa1, S.zpk[q][0], S.zpk[q][1], h[2][0], h[2][1]);
        cvt8x4<C::kKFmt>(wb1, S.zpk[4 + q][0], S.zpk[4 + q][1], h[3][0], h[3][1]);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {  // k-step 2q + kk: pairs e = 2kk (slot 0) and 2kk + 1 (slot 1)
          uint32_t ahi[2][2], alo[2][2];  // [row g / g + 8][slot]: f16x2 (channel i, channel i + 64)
          const float2 fa0 = f16x2_to_float2(h[0][kk]), fb0 = f16x2_to_float2(h[1][kk]);
          const float2 fa1 = f16x2_to_float2(h[2][kk]), fb1 = f16x2_to_float2(h[3][kk]);
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) {
            const int i = 16 * c + 4 * q + 2 * kk + hs;
            const float2 bt = lds_here_f2(rw + i);
            // key pair (x, y) = (channel i, channel i + 64) of rows g and g + 8
            float x0 = hs ? fa0.y : fa0.x, y0 = hs ? fb0.y : fb0.x;
            float x1 = hs ? fa1.y : fa1.x, y1 = hs ? fb1.y : fb1.x;
            if constexpr (C::kKFold == FOLD_CHANNEL) {
              const float sx = lds_here_f(kch + i), sy = lds_here_f(kch + i + 64);
              x0 *= sx; x1 *= sx; y0 *= sy; y1 *= sy;
            }
            float sn0, cs0, sn1, cs1;
            __sincosf(fmaf(j0, bt.y, bt.x), &sn0, &cs0);
            __sincosf(fmaf(j1, bt.y, bt.x), &sn1, &cs1);
            // (x, y) -> (x cos - y sin, y cos + x sin)
            split_f16x2(fmaf(x0, cs0, -y0 * sn0), fmaf(y0, cs0, x0 * sn0), ahi[0][hs], alo[0][hs]);
            split_f16x2(fmaf(x1, cs1, -y1 * sn1), fmaf(y1, cs1, x1 * sn1), ahi[1][hs], alo[1][hs]);
          }
          const int ks = 2 * q + kk;
          float(&acc_k)[4] = kk ? a1 : a0;
          mma_16816(acc_k, ahi[0][0], ahi[1][0], ahi[0][1], ahi[1][1], S.qh[ks][0], S.qh[ks][1]);
          mma_16816(acc_k, alo[0][0], alo[1][0], alo[0][1], alo[1][1], S.qh[ks][0], S.qh[ks][1]);
          if (split) mma_16816(acc_k, ahi[0][0], ahi[1][0], ahi[0][1], ahi[1][1], S.ql[ks][0], S.ql[ks][1]);
        }
      }
    } else {
      // 8-bit codes, 128-byte rows: chunks 2c and 2c+1 of rows g and g+8 (swizzled)
      const uint4 x0 = lds<uint4>(base + C::kOffK + swz<128>(r0, 2 * c));
      const uint4 x1 = lds<uint4>(base + C::kOffK + swz<128>(r0, 2 * c + 1));
      const uint4 y0 = lds<uint4>(base + C::kOffK + swz<128>(r1, 2 * c));
      const uint4 y1 = lds<uint4>(base + C::kOffK + swz<128>(r1, 2 * c + 1));
      const bool split = S.qsplit;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t u = word_of(ks < 4 ? x0 : x1, ks & 3), v = word_of(ks < 4 ? y0 : y1, ks & 3);
        if constexpr (C::kKFmt == FMT_S8) {
          u ^= 0x80808080u;
          v ^= 0x80808080u;
        }
        uint32_t u_lo, u_hi, v_lo, v_hi;
        cvt8x4<C::kKFmt>(u, S.zpk[ks][0], S.zpk[ks][1], u_lo, u_hi);
        cvt8x4<C::kKFmt>(v, S.zpk[ks][0], S.zpk[ks][1], v_lo, v_hi);
        mma2(ks, u_lo, v_lo, u_hi, v_hi, split);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[sb][k] = a0[k] + a1[k];
  }

  // (3) scores (log2 domain) with masking
  float sco[C::kNSub][4];
#pragma unroll
  for (int sb = 0; sb < C::kNSub; ++sb)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int tok = tok_base + sb * 16 + g + 8 * r;
      const bool ok = tok_ok(tok);
      float mul = S.kmul;
      if constexpr (C::kKFold == FOLD_TOKEN) mul *= reinterpret_cast<const float*>(base + C::kOffKM)[tok];
      if (C::kKivi && residual) mul *= res_kinv[sb][r];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float sv;
        if (C::kKivi && !residual)
          sv = fmaf(acc[sb][2 * r + j], S.kmul, S.bias[j]) * sc_log2;
        else
          sv = acc[sb][2 * r + j] * mul;
        sco[sb][2 * r + j] = ok ? sv : kNegInf;
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
  const bool odd = g & 1;
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
    pt[sb][0] = odd ? a1 : a0;
    pt[sb][1] = odd ? b1 : b0;
    pt[sb][2] = odd ? a3 : a2;
    pt[sb][3] = odd ? b3 : b2;
  }

  // (6) value-side fold and accumulator exponent
  constexpr bool kVPerToken = C::kVFold == FOLD_TOKEN || C::kGroupV;
  // folded value scale of token tok, group j (per-token fold: group 0); 0 for masked tokens.
  // Read from shared memory where it is used, so the 16 (KIVI: 32) values are not held live.
  auto vscale = [&](int tok, int j) -> float {
    if (!tok_ok(tok)) return 0.0f;
    if constexpr (C::kGroupV) return reinterpret_cast<const float*>(base + C::kOffVM)[tok * C::kNG + j * C::kNG / 4];
    return reinterpret_cast<const float*>(base + C::kOffVM)[tok];
  };
  int evn = 15;
  if (kVPerToken && !residual) {
    float smax = 0.0f;
#pragma unroll
    for (int sb = 0; sb < C::kNSub; ++sb)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int tok = tok_base + sb * 16 + 2 * c + (k & 1) + 8 * (k >> 1);
        const bool ok = tok_ok(tok);
        if constexpr (C::kGroupV) {
          const float4 s4 = vscale4<C>(base, tok);
          const float m4 = fmaxf(fmaxf(s4.x, s4.y), fmaxf(s4.z, s4.w));
          smax = fmaxf(smax, ok ? m4 : 0.0f);
        } else {
          const float s1 = reinterpret_cast<const float*>(base + C::kOffVM)[tok];
          smax = fmaxf(smax, ok ? s1 : 0.0f);
        }
      }
    smax = warp_max(smax);
    evn = smax > 0.0f ? range_shift(smax) : (S.ev_set ? S.ev : 15);
  }
  if (C::kKivi && residual) {  // each value row's inverse factor plays the role of its scale
    const float smax = warp_max(4 * g + c < d.n ? pow2i(-res_vx) : 0.0f);
    evn = smax > 0.0f ? range_shift(smax) : (S.ev_set ? S.ev : 15);
  }
  // rescale the accumulator only when some head's max moved or the exponent changed
  const bool moved = (alpha[0] != 1.0f) || (alpha[1] != 1.0f) || (S.ev_set && evn != S.ev);
  if (__any_sync(0xffffffffu, moved)) {
    float f0 = alpha[0], f1 = alpha[1];
    if (S.ev_set) {
      const float r = fast_exp2((float)(evn - S.ev));
      f0 *= r;
      f1 *= r;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      S.o[mt][0] *= f0;
      S.o[mt][1] *= f1;
      S.o[mt][2] *= f0;
      S.o[mt][3] *= f1;
    }
  }
  S.ev = evn;
  S.ev_set = true;
  const float pscale = pow2i(evn);

  // (7) O^T += V^T . P'^T
  if constexpr (C::kKivi) {
    // alpha for head g rescales the min-term accumulator
    const float ag0 = __shfl_sync(0xffffffffu, alpha[0], g >> 1);
    const float ag1 = __shfl_sync(0xffffffffu, alpha[1], g >> 1);
    const float ag = odd ? ag1 : ag0;
#pragma unroll
    for (int j = 0; j < 4; ++j) S.zacc[j] *= ag;
  }
#pragma unroll
  for (int sb = 0; sb < C::kNSub; ++sb) {
    const int tb0 = tok_base + sb * 16;
    const int tk[4] = {tb0 + 2 * c, tb0 + 2 * c + 1, tb0 + 2 * c + 8, tb0 + 2 * c + 9};
    bool ok[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) ok[k] = tok_ok(tk[k]);
    if constexpr (!C::kGroupV) {
      float pv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) pv[k] = (C::kVFold == FOLD_TOKEN ? pt[sb][k] * vscale(tk[k], 0) : pt[sb][k]) * pscale;
      uint32_t bh0, bl0, bh1, bl1;
      split_f16x2(pv[0], pv[1], bh0, bl0);
      split_f16x2(pv[2], pv[3], bh1, bl1);
      uint4 W[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        W[k] = lds<uint4>(base + C::kOffV + swz<128>(tk[k], g));
        if (kMasked && !ok[k]) W[k] = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (C::kVFmt == FMT_S8) {
          W[k].x ^= 0x80808080u; W[k].y ^= 0x80808080u; W[k].z ^= 0x80808080u; W[k].w ^= 0x80808080u;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t x0 = word_of(W[0], q), x1 = word_of(W[1], q);
        const uint32_t x2 = word_of(W[2], q), x3 = word_of(W[3], q);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int mt = 2 * q + half;
          // (token 2c, token 2c+1) bytes at channels d (lo) and d+1 (hi) of this m-tile
          const uint32_t ta = prmt(x0, x1, half ? 0x7362u : 0x5140u);
          const uint32_t tb2 = prmt(x2, x3, half ? 0x7362u : 0x5140u);
          uint32_t a0, a1, a2, a3;
          cvt8x4<C::kVFmt>(ta, S.zpv[mt][0], S.zpv[mt][1], a0, a1);
          cvt8x4<C::kVFmt>(tb2, S.zpv[mt][0], S.zpv[mt][1], a2, a3);
          mma_16816(S.o[mt], a0, a1, a2, a3, bh0, bh1);
          mma_16816(S.o[mt], a0, a1, a2, a3, bl0, bl1);
        }
      }
    } else {
      // one B operand per 32-channel group, built just before that group's MMAs; KIVI's
      // zero-point term on CUDA cores
      // value scales of this thread's four tokens, groups 0..3 (fp16 metadata stays packed as
      // halves until its group is used, which halves the registers it holds)
      float4 s4[4];
      uint2 s4h[4];
      float rv[4];   // residual: the power of two each of the four tokens' value rows is scaled by
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        s4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        s4h[k] = make_uint2(0u, 0u);
        rv[k] = 1.0f;
        if constexpr (C::kHalfMeta) {
          if (!residual && ok[k]) s4h[k] = lds<uint2>(base + C::kOffVM + tk[k] * 8);
        } else {
          if (!residual && ok[k]) s4[k] = vscale4<C>(base, tk[k]);
        }
        if (C::kKivi && residual) {
          const int x = __shfl_sync(0xffffffffu, res_vx, tk[k] & 31);
          rv[k] = pow2i(x);
          s4[k] = make_float4(pow2i(-x), 0.f, 0.f, 0.f);
        }
      }
      if (C::kKivi && !residual) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (!ok[k]) continue;
          const float4 z4 = meta4<C::kHalfMeta>(base + C::kOffVM + C::kVMeta / 2, tk[k]);
          S.zacc[0] = fmaf(pt[sb][k], z4.x, S.zacc[0]);
          S.zacc[1] = fmaf(pt[sb][k], z4.y, S.zacc[1]);
          S.zacc[2] = fmaf(pt[sb][k], z4.z, S.zacc[2]);
          S.zacc[3] = fmaf(pt[sb][k], z4.w, S.zacc[3]);
        }
      }
      // INT4 codes: one transposed matrix load per 8 tokens gives every lane its (token 2c,
      // token 2c + 1) pair of 16-bit words (4 channels) for all four channel groups
      uint32_t v4[2][4];
      if constexpr (C::kVFmt == FMT_U4 || C::kVFmt == FMT_S4) {
        if (!residual) {
          const int lane = threadIdx.x & 31;
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            ldsm_x4_trans(smem_addr(base + C::kOffV + swz<64>(tb0 + 8 * pp + (lane & 7), lane >> 3)), v4[pp]);
            if constexpr (kMasked) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                v4[pp][j] &= (ok[2 * pp] ? 0x0000FFFFu : 0u) | (ok[2 * pp + 1] ? 0xFFFF0000u : 0u);
            }
          }
        }
      }
      // p * 2^evn once per token (a power of two: exact, so p * 2^evn * s rounds as p * s * 2^evn);
      // KIVI INT4 keeps the per-group form, whose fewer live registers its allocation prefers
      constexpr bool kHoist = C::kVFmt != FMT_U4;
      float pp2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) pp2[k] = kHoist ? pt[sb][k] * pscale : pt[sb][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t bh[2], bl[2];  // P' of group j: tokens (2c, 2c + 1) and (2c + 8, 2c + 9), hi + lo
        {
          float pv[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float sj;
            if constexpr (C::kHalfMeta) {
              const float2 h2 = f16x2_to_float2((j >> 1) ? s4h[k].y : s4h[k].x);
              sj = (j & 1) ? h2.y : h2.x;
            } else {
              sj = j == 0 ? s4[k].x : j == 1 ? s4[k].y : j == 2 ? s4[k].z : s4[k].w;
            }
            if constexpr (kHoist)
              pv[k] = residual ? pp2[k] * s4[k].x : pp2[k] * sj;
            else
              pv[k] = residual ? pp2[k] * s4[k].x * pscale : pp2[k] * sj * pscale;
          }
          split_f16x2(pv[0], pv[1], bh[0], bl[0]);
          split_f16x2(pv[2], pv[3], bh[1], bl[1]);
        }
        uint32_t pr[2][4];  // [token pair][channel e]: f16x2 (token even, token odd)
        if (residual) {
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            const uint8_t* vr = base + kRT * kHeadDim * 2;
            uint2 u0 = lds<uint2>(vr + tk[2 * pp] * 256 + (32 * j + 4 * g) * 2);
            uint2 u1 = lds<uint2>(vr + tk[2 * pp + 1] * 256 + (32 * j + 4 * g) * 2);
            if (!ok[2 * pp]) u0 = make_uint2(0u, 0u);
            if (!ok[2 * pp + 1]) u1 = make_uint2(0u, 0u);
            const float fa = rv[2 * pp], fb = rv[2 * pp + 1];
            pr[pp][0] = float2_to_f16x2(bf16_bits_to_float(u0.x & 0xFFFFu) * fa, bf16_bits_to_float(u1.x & 0xFFFFu) * fb);
            pr[pp][1] = float2_to_f16x2(bf16_bits_to_float(u0.x >> 16) * fa, bf16_bits_to_float(u1.x >> 16) * fb);
            pr[pp][2] = float2_to_f16x2(bf16_bits_to_float(u0.y & 0xFFFFu) * fa, bf16_bits_to_float(u1.y & 0xFFFFu) * fb);
            pr[pp][3] = float2_to_f16x2(bf16_bits_to_float(u0.y >> 16) * fa, bf16_bits_to_float(u1.y >> 16) * fb);
          }
        } else if constexpr (C::kVFmt == FMT_U4) {
#pragma unroll
          for (int pp = 0; pp < 2; ++pp)
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[pp][e] = u4_pair(v4[pp][j], e);
        } else if constexpr (C::kVFmt == FMT_S4) {
#pragma unroll
          for (int pp = 0; pp < 2; ++pp)
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[pp][e] = s4_pair(v4[pp][j], e);
        } else {
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            uint32_t u0 = lds<uint8_t>(base + C::kOffV + swz<32>(tk[2 * pp], j >> 1) + 8 * (j & 1) + g);
            uint32_t u1 = lds<uint8_t>(base + C::kOffV + swz<32>(tk[2 * pp + 1], j >> 1) + 8 * (j & 1) + g);
            if (kMasked && !ok[2 * pp]) u0 = 0u;
            if (kMasked && !ok[2 * pp + 1]) u1 = 0u;
            const uint32_t wv = prmt(u0, u1, 0x5410u);
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[pp][e] = u2_pair(wv, e);
          }
        }
        // channel e = 2 * (mt & 1) + rh within the group: mt = 2j + (e >> 1)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int mt = 2 * j + half;
          mma_16816(S.o[mt], pr[0][2 * half], pr[0][2 * half + 1], pr[1][2 * half], pr[1][2 * half + 1], bh[0], bh[1]);
          mma_16816(S.o[mt], pr[0][2 * half], pr[0][2 * half + 1], pr[1][2 * half], pr[1][2 * half + 1], bl[0], bl[1]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ the kernel
template <int KS, int VS, bool PAGED, int NG, bool ROPE>
__global__ void __launch_bounds__(Cfg<KS, VS, PAGED, NG, ROPE>::kThreadsCta, Cfg<KS, VS, PAGED, NG, ROPE>::kMinBlocks)
    decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_ks,
                  const __grid_constant__ CUtensorMap tmap_kz) {
  using C = Cfg<KS, VS, PAGED, NG, ROPE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  // the cache, the queries and the plan come from earlier kernels (after an overlapped append,
  // only the tiles it writes: the producer waits before the first of them)
  if (!C::kOverlapAppend || p.early_from < 0) grid_dependency_wait();
  grid_launch_dependents();  // the merge may be scheduled now; it waits for this grid to finish
  const Sched sc = make_sched(p);
  const int tb = blockIdx.x * sc.W;
  const int te = min(sc.N, tb + sc.W);
  if (tb >= te) return;
  TileDesc* descs = reinterpret_cast<TileDesc*>(smem + C::kOffDesc);
  const uint32_t full0 = smem_addr(smem + C::kOffBar);
  const uint32_t empty0 = full0 + 8 * C::kStages;
  // self-fed pipeline: releases of each stage counted in the slack after the barriers
  uint32_t* releases = reinterpret_cast<uint32_t*>(smem + C::kOffBar + 2 * C::kStages * 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kCW);
      releases[i] = 0u;
    }
    fence_barrier_init();
  }
  __syncthreads();
  const int no_pages[C::kTS / 16] = {};  // dense tiles: no page ids
  if constexpr (C::kSelfFed) {
    if (threadIdx.x == 0) {  // the first stages; the rest are refilled by the consumer warps
      TileIter f;
      f.init(p, sc, tb, te);
      for (int s0 = 0; s0 < C::kStages && f.t < te; ++s0, f.next(p, sc))
        issue_tile<C>(p, &tmap_k, &tmap_v, &tmap_ks, &tmap_kz, smem, descs, full0, s0, f.desc(p, sc), no_pages);
    }
  } else if (warp == kCW) {
    if (lane == 0) producer<C>(p, &tmap_k, &tmap_v, &tmap_ks, &tmap_kz, smem, descs, full0, empty0, sc, tb, te);
    return;
  }

  // ---------------------------------------------------------------- consumers
  Consumer<C> S;
  S.w = warp;
  S.g = lane >> 2;
  S.c = lane & 3;
  const int g = S.g, c = S.c, w = S.w;
  float* red_o = reinterpret_cast<float*>(smem + C::kOffRedO);
  float* red_m = reinterpret_cast<float*>(smem + C::kOffRedM);
  float* red_l = reinterpret_cast<float*>(smem + C::kOffRedL);
  float* red_z = reinterpret_cast<float*>(smem + C::kOffRedZ);
  float* q_s = reinterpret_cast<float*>(smem + C::kOffQ);
  const float sc_log2 = p.softmax_scale * kLog2e;
  if constexpr (C::kRope) {  // inverse frequencies base^(-2i/128) in fp64 (visible after the first pair start)
    if (threadIdx.x < 64)
      rope_theta_s(q_s)[threadIdx.x] = pow((double)p.rope_theta, -2.0 * (double)threadIdx.x / (double)kHeadDim);
  }
  bool dead = false;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) S.zpk[ks][0] = S.zpk[ks][1] = S.zpv[ks][0] = S.zpv[ks][1] = 0u;

  TileIter ti;
  ti.init(p, sc, tb, te);
  for (int st = 0, phase = 0; ti.t < te; ti.next(p, sc)) {
    const TileDesc d = ti.desc(p, sc);
    if constexpr (!C::kEarlyPairStart) {
      if (!dead && !mbar_wait(full0 + 8 * st, phase, p.status)) dead = true;
    }

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
        q_s[q_off(j, dd)] = v;
      }
      if constexpr (C::kRope && C::kKFold == FOLD_CHANNEL)  // per-channel key scales, applied before the rotation
        rope_key_scales(q_s)[tid] = p.k_scale[(size_t)d.hk * kHeadDim + tid];
      named_sync(1, kCW * 32);
      if (p.rotate) {  // H q: butterflies of span 1 .. 64 over the staged rows, then 1/sqrt(128)
        for (int h = 1; h < kHeadDim; h <<= 1) {
          for (int idx = tid; idx < 8 * kHeadDim / 2; idx += kCW * 32) {
            const int j = idx >> 6, i = idx & 63;
            const int lo = ((i & ~(h - 1)) << 1) | (i & (h - 1));
            const float a = q_s[q_off(j, lo)], b = q_s[q_off(j, lo + h)];
            q_s[q_off(j, lo)] = a + b;
            q_s[q_off(j, lo + h)] = a - b;
          }
          named_sync(1, kCW * 32);
        }
        for (int idx = tid; idx < 8 * kHeadDim; idx += kCW * 32) q_s[q_off(idx >> 7, idx & 127)] *= kInvSqrt128;
        named_sync(1, kCW * 32);
      }
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
      if constexpr (C::kKivi) {  // first factor of the key groups' shift bound: max |q| of the pair
        const float4* qrow = reinterpret_cast<const float4*>(q_s + q_off(g, 32 * c));
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 q4 = qrow[i];
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(q4.x), fabsf(q4.y)), fmaxf(fabsf(q4.z), fabsf(q4.w))));
        }
        S.qabs = warp_max(mx);
      }
      if constexpr (!C::kKivi) {
        const float* fold = nullptr;
        if constexpr (C::kKFold == FOLD_CHANNEL) fold = p.k_scale + (size_t)d.hk * kHeadDim;
        int eq;
        if constexpr (C::kRope)
          eq = build_q_rope(q_s, g, c, S.qh, S.ql);
        else if constexpr (C::kKFmt == FMT_S4)
          eq = build_q_s4(q_s, g, c, S.qh, S.ql);
        else
          eq = build_q<C::kKFmt>(q_s, fold, nullptr, g, c, S.qh, S.ql);
        // bf16 queries are exact in f16 (after the power-of-two shift) unless a fold multiplies them
        S.qsplit = (!C::kRope && C::kKFold == FOLD_CHANNEL) || !p.q_bf16 || p.rotate;
        float mul = sc_log2 * pow2i(-eq);
        if constexpr (C::kKFold == FOLD_TENSOR) mul *= p.k_scale[0];
        S.kmul = mul;
        S.qmode = 0;
        if constexpr (C::kKFmt == FMT_U8) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // RoPE keys: word ks & 3 of chunk c (ks < 4) or of chunk 4 + c, bytes 2h, 2h + 1
              const int d0 = C::kRope ? (ks >> 2) * 64 + 16 * c + 4 * (ks & 3) + 2 * h : dmap_k<C::kKFmt>(c, ks, h, 0);
              const float z0 = 1024.0f + p.k_zp[d.hk * kHeadDim + d0];
              const float z1 = 1024.0f + p.k_zp[d.hk * kHeadDim + d0 + 1];
              S.zpk[ks][h] = float2_to_f16x2(z0, z1);
            }
        }
      }
      if constexpr (C::kVFmt == FMT_U8) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int rh = 0; rh < 2; ++rh) {
            const float z = 1024.0f + p.v_zp[d.hk * kHeadDim + dmap_v<false>(g, mt, rh)];
            S.zpv[mt][rh] = float2_to_f16x2(z, z);
          }
      }
    }

    // ------------------------------------------------ tile work
    if constexpr (C::kEarlyPairStart) {  // the pair start above overlapped the tile's arrival
      if (!dead && !mbar_wait(full0 + 8 * st, phase, p.status)) dead = true;
    }
    const uint8_t* base = smem + st * C::kStageBytes;
    const uint32_t valid = C::kPaged ? descs[st].valid : 0xFFFFFFFFu;
    const bool residual = C::kKivi && d.kind == 1;
    const int tok_base = residual ? 0 : w * C::kTPW;
    const bool busy = !dead && (residual ? (w == 0) : true) && (d.n - tok_base > 0);
    if (busy) {
      const bool full = d.n - tok_base >= C::kTPW && (!C::kPaged || valid == 0xFFFFFFFFu ||
                                                       ((valid >> (tok_base / p.page_size)) &
                                                        ((1u << (C::kTPW + p.page_size - 1) / p.page_size) - 1u)) ==
                                                           ((1u << (C::kTPW + p.page_size - 1) / p.page_size) - 1u));
      if (C::kKivi && residual)
        warp_tile<C, true, C::kKivi>(S, p, base, d, valid, tok_base, sc_log2, q_s);
      else if (full)
        warp_tile<C, false, false>(S, p, base, d, valid, tok_base, sc_log2, q_s);
      else
        warp_tile<C, true, false>(S, p, base, d, valid, tok_base, sc_log2, q_s);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * st);
    if constexpr (C::kSelfFed) {
      // the last warp to release this stage refills it with the tile kStages ahead (the wait on
      // the completed release orders every warp's reads of the stage before the copies)
      if (lane == 0 && atomicAdd(releases + st, 1u) == kCW - 1) {
        releases[st] = 0u;
        const int tn = ti.t + C::kStages;
        if (tn < te && mbar_wait(empty0 + 8 * st, phase, p.status)) {
          TileIter f;
          f.init(p, sc, tn, te);
          issue_tile<C>(p, &tmap_k, &tmap_v, &tmap_ks, &tmap_kz, smem, descs, full0, st, f.desc(p, sc), no_pages);
        }
      }
    }
    if (++st == C::kStages) {
      st = 0;
      phase ^= 1;
    }

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
      const int dd = threadIdx.x;  // channel
      const int slot = d.pair + blockIdx.x;
      float vsc = 1.0f;
      if constexpr (C::kVFold == FOLD_TENSOR) vsc = p.v_scale[0];
      if constexpr (C::kVFold == FOLD_CHANNEL) vsc = p.v_scale[(size_t)d.hk * kHeadDim + dd];
      if constexpr (C::kKivi) {  // minimum-term sums of head g over the four lanes c
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S.zacc[j] += __shfl_xor_sync(0xffffffffu, S.zacc[j], 1);
          S.zacc[j] += __shfl_xor_sync(0xffffffffu, S.zacc[j], 2);
        }
      }
      // O is staged and merged kMergeHeads heads at a time (lanes hold heads 2c, 2c + 1); the
      // group's padding heads (G < 8) are neither merged nor written
      constexpr int kMH = C::kMergeHeads;
      const int nh = min(8, p.G - d.hg * 8);
#pragma unroll
      for (int half = 0; half < 8 / kMH; ++half) {
        if (kMH * half >= nh) break;  // uniform over the CTA
        if ((2 * c) / kMH == half) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int rh = 0; rh < 2; ++rh) {
              const int ch = dmap_v<C::kGroupV>(g, mt, rh);
              red_o[(w * kMH + 2 * c - kMH * half) * kHeadDim + red_col<C::kGroupV>(ch, 2 * c)] = S.o[mt][2 * rh] * oscale;
              red_o[(w * kMH + 2 * c + 1 - kMH * half) * kHeadDim + red_col<C::kGroupV>(ch, 2 * c + 1)] =
                  S.o[mt][2 * rh + 1] * oscale;
            }
        }
        if constexpr (C::kKivi) {
          if (c == 0 && g / kMH == half) {
#pragma unroll
            for (int j = 0; j < 4; ++j) red_z[(w * kMH + g - kMH * half) * 4 + j] = S.zacc[j];
          }
        }
        named_sync(1, kCW * 32);
#pragma unroll 1
        for (int j = kMH * half; j < kMH * half + kMH && j < nh; ++j) {
          float M = kNegInf;
#pragma unroll
          for (int ww = 0; ww < kCW; ++ww) M = fmaxf(M, red_m[ww * 8 + j]);
          float ov = 0.0f, L = 0.0f;
          if (M != kNegInf) {
#pragma unroll
            for (int ww = 0; ww < kCW; ++ww) {
              const float a = fast_exp2(red_m[ww * 8 + j] - M);
              float x = red_o[(ww * kMH + j - kMH * half) * kHeadDim + red_col<C::kGroupV>(dd, j)];
              if constexpr (C::kKivi) x += red_z[(ww * kMH + j - kMH * half) * 4 + (dd >> 5)];
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
}

// ------------------------------------------------------------------ merge
// One warp per query head (b, hq): lanes read the partials' (m, l) in parallel and combine
// them with shuffles; each lane then accumulates a float4 of channels over the partials.
// The grid is small (two CTAs of four warps an SM at most, each warp looping over query
// heads): launched as the decode grid's programmatic dependent, its CTAs take the room the
// decode CTAs leave on each SM (one next to two 8-bit decode CTAs, the rest as decode CTAs
// retire) and wait in griddepcontrol.wait, so they start the moment the decode grid completes.
constexpr int kMergeThreads = 128;

__global__ void __launch_bounds__(kMergeThreads, 6) merge_kernel(const DecodeParams p) {
  grid_dependency_wait();  // the partials of the decode kernel
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (kMergeThreads / 32);
  const int per_seq = p.Hkv * p.HG;
  for (int u = blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5); u < p.B * p.Hq; u += nwarps) {
    const int b = u / p.Hq, hq = u - b * p.Hq;
    const int hk = hq / p.G, hl = hq - hk * p.G;
    const int hg = hl >> 3, j = hl & 7;
    const int hh = hk * p.HG + hg;
    const int pair = b * per_seq + hh;
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
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float M = kNegInf, L = 0.0f;
    if (n > 0) {
      const int W = (N + p.ncta - 1) / p.ncta;
      const int c0 = off / W, c1 = (off + n - 1) / W;
      for (int base = c0; base <= c1; base += 32) {
        const int cnt = min(32, c1 - base + 1);
        const float4* po =
            reinterpret_cast<const float4*>(p.part_o) + ((size_t)(pair + base) * 8 + j) * (kHeadDim / 4) + lane;
        // the first partials' rows are loaded together with the (m, l) pairs: one memory round trip
        constexpr int kEarly = 2;
        float4 early[kEarly];
#pragma unroll
        for (int i = 0; i < kEarly; ++i)
          if (i < cnt) early[i] = po[(size_t)i * 8 * (kHeadDim / 4)];
        float mi = kNegInf, li = 0.0f;
        if (lane < cnt) {
          const size_t sl = (size_t)(pair + base + lane) * 8 + j;
          mi = p.part_ml[sl * 2];
          li = p.part_ml[sl * 2 + 1];
        }
        const float mc = warp_max(fmaxf(M, mi));
        const float f = (M == kNegInf || mc == kNegInf) ? 0.0f : fast_exp2(M - mc);
        const float ai = (mi == kNegInf || mc == kNegInf) ? 0.0f : fast_exp2(mi - mc);
        float lw = ai * li;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
        L = fmaf(L, f, lw);
        acc.x *= f; acc.y *= f; acc.z *= f; acc.w *= f;
#pragma unroll
        for (int i = 0; i < kEarly; ++i) {
          const float a = __shfl_sync(0xffffffffu, ai, i);
          if (i < cnt) {
            acc.x = fmaf(a, early[i].x, acc.x);
            acc.y = fmaf(a, early[i].y, acc.y);
            acc.z = fmaf(a, early[i].z, acc.z);
            acc.w = fmaf(a, early[i].w, acc.w);
          }
        }
        for (int i = kEarly; i < cnt; ++i) {
          const float a = __shfl_sync(0xffffffffu, ai, i);
          const float4 o4 = po[(size_t)i * 8 * (kHeadDim / 4)];
          acc.x = fmaf(a, o4.x, acc.x);
          acc.y = fmaf(a, o4.y, acc.y);
          acc.z = fmaf(a, o4.z, acc.z);
          acc.w = fmaf(a, o4.w, acc.w);
        }
        M = mc;
      }
    }
    float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
    float lse = kNegInf;
    if (M != kNegInf && L > 0.0f) {
      // one reciprocal and the hardware log2: the merge is on the call's critical path, and
      // both stay far inside the attention tolerance
      const float inv = __frcp_rn(L);
      ov = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      float lg;
      asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(L));
      lse = (M + lg) * 0.69314718055994531f;
    }
    if (p.rotate) {  // sum p (H v) = H (sum p v): rotate the output back
      float r[4] = {ov.x, ov.y, ov.z, ov.w};
      fwht_row32(r, lane);
      ov = make_float4(r[0], r[1], r[2], r[3]);
    }
    reinterpret_cast<float4*>(p.out + ((size_t)b * p.Hq + hq) * kHeadDim)[lane] = ov;
    if (lane == 0 && p.lse) p.lse[(size_t)b * p.Hq + hq] = lse;
  }
}

// ------------------------------------------------------------------ paged plan
// plan[b] = tiles before sequence b (all its pairs), plan[B] = total, plan[B+1+b] = length.
__global__ void __launch_bounds__(1024) plan_kernel(const DecodeParams p) {
  __shared__ int warp_sum[32];
  __shared__ int carry;
  grid_dependency_wait();  // sequence lengths advanced by the append
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
  int k, v, paged, ng, rope;
  void (*kernel)(const DecodeParams, const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap);
  int smem, ts, threads;
};

template <int KS, int VS, bool PG, int NG = 4, bool ROPE = false>
Variant variant() {
  using C = Cfg<KS, VS, PG, NG, ROPE>;
  return Variant{KS, VS, PG ? 1 : 0, NG, ROPE ? 1 : 0, decode_kernel<KS, VS, PG, NG, ROPE>, C::kSmemBytes, C::kTS,
                 C::kThreadsCta};
}

constexpr int kNumVariants = 40;
constexpr int kMaxDevices = 64;

const Variant* variants() {
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
      variant<KVQ_INT8_SYM_PER_TOKEN, KVQ_UINT8_ASYM_PER_CHANNEL, false>(),
      variant<KVQ_INT8_SYM_PER_TOKEN, KVQ_UINT8_ASYM_PER_CHANNEL, true>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_INT8_SYM_PER_TOKEN, false>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_INT8_SYM_PER_TOKEN, true>(),
      variant<KVQ_FP8_E4M3_PER_TENSOR, KVQ_INT8_SYM_PER_TENSOR, false>(),
      variant<KVQ_FP8_E4M3_PER_TENSOR, KVQ_INT8_SYM_PER_TENSOR, true>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_FP8_E4M3_PER_TENSOR, false>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_FP8_E4M3_PER_TENSOR, true>(),
      variant<KVQ_FP8_E5M2_PER_TENSOR, KVQ_FP8_E5M2_PER_TENSOR, false>(),
      variant<KVQ_FP8_E5M2_PER_TENSOR, KVQ_FP8_E5M2_PER_TENSOR, true>(),
      variant<KVQ_INT4_SYM_PER_GROUP, KVQ_INT4_SYM_PER_GROUP, false>(),
      variant<KVQ_INT4_SYM_PER_GROUP, KVQ_INT4_SYM_PER_GROUP, true>(),
      variant<KVQ_INT4_SYM_PER_GROUP, KVQ_INT4_SYM_PER_GROUP, false, 2>(),
      variant<KVQ_INT4_SYM_PER_GROUP, KVQ_INT4_SYM_PER_GROUP, true, 2>(),
      variant<KVQ_INT4_SYM_PER_GROUP, KVQ_INT4_SYM_PER_GROUP, false, 1>(),
      variant<KVQ_INT4_SYM_PER_GROUP, KVQ_INT4_SYM_PER_GROUP, true, 1>(),
      variant<KVQ_KIVI_INT4, KVQ_KIVI_INT4, false>(),
      variant<KVQ_KIVI_INT2, KVQ_KIVI_INT2, false>(),
      variant<KVQ_KIVI_INT4_F16, KVQ_KIVI_INT4_F16, false>(),
      variant<KVQ_KIVI_INT2_F16, KVQ_KIVI_INT2_F16, false>(),
      // keys cached before RoPE
      variant<KVQ_FP8_E4M3_PER_TENSOR, KVQ_FP8_E4M3_PER_TENSOR, false, 4, true>(),
      variant<KVQ_FP8_E4M3_PER_TENSOR, KVQ_FP8_E4M3_PER_TENSOR, true, 4, true>(),
      variant<KVQ_INT8_SYM_PER_CHANNEL, KVQ_UINT8_ASYM_PER_CHANNEL, false, 4, true>(),
      variant<KVQ_INT8_SYM_PER_CHANNEL, KVQ_UINT8_ASYM_PER_CHANNEL, true, 4, true>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_UINT8_ASYM_PER_CHANNEL, false, 4, true>(),
      variant<KVQ_INT8_SYM_PER_TENSOR, KVQ_UINT8_ASYM_PER_CHANNEL, true, 4, true>(),
  };
  static_assert(sizeof(table) / sizeof(table[0]) == kNumVariants, "variant count");
  return table;
}

// ng: scales per row of an INT4 per-group scheme (128 / group size); 4 for the others
const Variant* find_variant(int k, int v, int paged, int ng, bool rope) {
  const Variant* table = variants();
  for (int i = 0; i < kNumVariants; ++i)
    if (table[i].k == k && table[i].v == v && table[i].paged == paged && table[i].ng == ng &&
        table[i].rope == (rope ? 1 : 0))
      return &table[i];
  return nullptr;
}

int groups_per_row(int k_scheme, int group) {
  return (k_scheme == KVQ_INT4_SYM_PER_GROUP && group > 0) ? kHeadDim / group : 4;
}



}  // namespace

bool decode_supported(int k_scheme, int v_scheme, int paged, int group, bool rope) {
  return find_variant(k_scheme, v_scheme, paged, groups_per_row(k_scheme, group), rope) != nullptr;
}

cudaError_t launch_decode(DecodeParams p, cudaStream_t st) {
  const Variant* var =
      find_variant(p.k_scheme, p.v_scheme, p.paged, groups_per_row(p.k_scheme, p.group), p.rope_theta > 0.0f);
  if (!var) return cudaErrorNotSupported;
  p.ts = var->ts;
  if (!p.paged) {
    p.nq = (p.len_q + var->ts - 1) / var->ts;
    p.nr = is_kivi(p.k_scheme) ? (p.len_res + kRT - 1) / kRT : 0;
  } else {
    p.nq = p.nr = 0;
  }
  // shared-memory opt-in and resident CTAs per SM: set up once per (variant, device)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<int> occ_cache[kNumVariants][kMaxDevices];
  const int vi = (int)(var - variants());
  int occ = dev < kMaxDevices ? occ_cache[vi][dev].load(std::memory_order_relaxed) : 0;
  if (occ <= 0) {
    e = cudaFuncSetAttribute(var->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, var->smem);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, var->kernel, var->threads, var->smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    if (dev < kMaxDevices) occ_cache[vi][dev].store(occ, std::memory_order_relaxed);
  }
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
  // KIVI key scales and minima seen as 128-byte rows (4 rows per 32-token group of fp32, 2 of fp16);
  // a tile's 4 groups are one box
  CUtensorMap tks = tk, tkz = tk;
  if (is_kivi(p.k_scheme)) {
    const int es = kivi_f16(p.k_scheme) ? 2 : 4;
    const uint64_t mrows = (uint64_t)p.B * p.Hkv * (uint64_t)(p.cap / 32) * es;  // 128 channels * es / 128
    const int mbox = (var->ts / 32) * es;
    if (!make_map(&tks, p.k_scale, 128, mrows, mbox) || !make_map(&tkz, p.k_zero, 128, mrows, mbox))
      return cudaErrorInvalidValue;
  }
  // Programmatic dependent launches: each kernel may be scheduled while its predecessor
  // drains and waits in griddepcontrol.wait, hiding the launch gaps between the three.
  if (p.paged) {
    e = launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, st, p);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(var->kernel, dim3(ncta), dim3(var->threads), (size_t)var->smem, st, p, tk, tv, tks, tkz);
  if (e != cudaSuccess) {
    if (dev < kMaxDevices) occ_cache[vi][dev].store(0, std::memory_order_relaxed);  // set up again next call
    return e;
  }
  // merge: two CTAs an SM at most, fewer when there are fewer query heads than warps
  const long long heads = (long long)p.B * p.Hq;
  const int mgrid =
      (int)std::min<long long>(2LL * sm_count(), (heads + kMergeThreads / 32 - 1) / (kMergeThreads / 32));
  e = launch_pdl(merge_kernel, dim3(mgrid > 0 ? mgrid : 1), dim3(kMergeThreads), 0, st, p);
  if (e != cudaSuccess) return e;
  count_launches(p.paged ? 3 : 2);
  return cudaGetLastError();
}

}  // namespace kvq

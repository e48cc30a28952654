// Absorbed MLA decode attention on pairs of SMs: cta_group::2 tensor-core
// MMAs (tcgen05, TMEM accumulators) fed by TMA, with split-KV work lists.
//
// What it computes ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide",
// "The Matrix Absorption Trick", parts 2-4, and "Step 3" of the PyTorch
// implementation): for one query token of one sequence and all heads h,
//   s_hi = (q~_h . c_i + q^R_h . k^R_i) * scale      (cached tokens i <= qpos)
//   o_h  = sum_i softmax(s_h)_i c_i                   (512-dim latent output)
// with the latent cache read once from HBM and shared by every head.
//
// Work split. One work list runs on a cluster of two CTAs (two SMs) that issue
// pair MMAs (M = 128 heads split 64 + 64, N = 256):
//   * scores: S = Q C^T over all 576 columns. A = the CTA's 64 query rows
//     (shared memory), B = the cached rows of a 4-page tile, CTA r supplying
//     pages 2r and 2r+1 of it. Each CTA receives the full 256-token score rows
//     of its own 64 heads, so each CTA runs the softmax of its heads alone:
//     nothing is exchanged between the CTAs.
//   * output: O += P C[:, 0:512] in two N = 256 column chunks. A = the CTA's
//     64 rows of P, B = C^T columns [256j + 128r, +128) of all four pages
//     (loaded by CTA r). Each CTA's TMEM holds its heads' full 512-column
//     accumulator (64 rows folded onto 128 lanes).
// Each page is read from HBM once per (item, query): its rows by one CTA for the
// scores and its latent columns by both CTAs (one half each) for the output;
// the second read of a row hits L2. Both MMAs run at the full per-SM tensor
// rate (64 x 256 per SM per instruction).
//
// Warp roles (320 threads per CTA): warps 0-7 softmax + epilogue (thread =
// (TMEM lane, column group) = (head, page of the tile)), warp 8 TMA producer,
// warp 9 MMA issuer (even CTA) and TMEM owner (both CTAs).
// Pipeline: QK(t+1) is issued before PV(t), so the softmax of tile t overlaps
// the next tile's score MMAs; two TMEM score buffers; a ring of 16 KB shared
// memory stages carries score chunks (128 rows x 64 columns) and output chunks
// (64 rows x 128 columns) in the order the MMAs consume them.
// The running max is rescaled lazily: O and the sum are rescaled only when a
// row's max grows by more than 8 (log2 units); the final normalisation uses the
// same reference max, so the result is exact up to rounding.
//
// FP8 cache instance (448 threads: warps 10-13 convert). The stages run in
// the same order, each loaded to its own CTA's barriers and expanded in place
// before the MMA issuer takes it: a score chunk pair lands as the pages' 128
// code columns in the first of its two stages, an output stage as one page's
// code columns in its upper half, and the converter warp that owns the stage
// writes code * scale as fp16 over the stage (each row overwrites only its
// own codes). The latent MMAs take fp16 operands: the query's latent columns
// are converted to fp16 when they land (exact for the bf16 values in the
// fp16 range), the probabilities are rounded to fp16, and code * scale is
// exact on the fp16 grid for scales in [2^-15, 2^7]. The RoPE chunk (bf16 k^R
// and q^R) stays bf16 with its own bf16 MMA into the same accumulator. A value
// outside the fp16 range sets MLA_DEV_RANGE. The producer brings each tile's
// pages into L2 one tile ahead.
//
// Every wait is bounded (about one second); on expiry the kernel sets
// MLA_DEV_TIMEOUT, stops issuing work, drains what it issued and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp0 = 10;                       // FP8 cache: converter warps 10..13
constexpr int kConvWarps = 4;
constexpr int kTilePages = 4;                       // pages per score tile (256 tokens)
constexpr int kChunksQK = MLA_ROW / 64;              // 9 column chunks of the score MMA
constexpr uint32_t kBox = 64 * 128;                  // 64 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kStageBytes = 2 * kBox;           // 16384
constexpr uint32_t kOffQ = 0;                        // 9 x [64 heads][64 cols]
constexpr uint32_t kOffP = kOffQ + kChunksQK * kBox; // 73728: 4 x [64 heads][64 tokens]
constexpr uint32_t kOffRing = kOffP + kTilePages * kBox;  // 106496: bf16 operand stages
constexpr uint32_t kHalfStage = kStageBytes / 2;     // FP8: codes land in a stage's upper half
constexpr uint32_t kScaleSlot = 512;                 // FP8: the scales of a stage's <= 2 pages
constexpr uint32_t kBarArea = 384;

constexpr int kMaxStages = 7;                        // capacity of the stage barrier arrays
// FP8: the producer brings a tile's pages into L2 this many tiles before it
// loads them. With half the bytes of a bf16 stage in each stage, the ring
// keeps too few bytes in flight to cover a load from HBM.
constexpr int kFp8PrefetchTiles = 1;

enum {
  B_FULL0 = 0,                          // [kMaxStages] stage ready (even CTA)
  B_EMPTY0 = B_FULL0 + kMaxStages,      // [kMaxStages] stage consumed (both CTAs)
  B_LFULL0 = B_EMPTY0 + kMaxStages,     // [kMaxStages] FP8 codes of a stage landed (local)
  B_QFULL = B_LFULL0 + kMaxStages,      // query rows loaded (even CTA: both CTAs' bytes)
  B_QEMPTY,                        // last score MMA of the item done (both)
  B_QCONV,                         // FP8: query rows converted to fp16 (even CTA: 8 warps)
  B_SFULL0, B_SFULL1,              // scores of a tile ready (both)
  B_SFREE0, B_SFREE1,              // scores read out (even CTA: 16 warps of both CTAs)
  B_PFULL,                         // P written (even CTA: 16 warps)
  B_PVDONE,                        // output MMAs of a tile done (both)
  B_PMAX0, B_PMAX1,                // the four page maxes of every row posted (local, 8 warps)
  B_EPI,                           // the four page sums posted (local, 8 warps)
  B_FINAL,                         // MMA drain (even CTA)
  B_COUNT
};
static_assert(8 * B_COUNT + 8 <= kBarArea, "barrier area overflow");

// Shared-memory layout of the two instances: a 7-stage ring of bf16 operand
// stages. bf16 cache: TMA fills the stages. FP8 cache: TMA lands a stage's
// E4M3 codes in its upper half (and the tokens' scales in the stage's scale
// slot), and the converter warps expand them in place into the bf16 stage.
template <bool kFp8>
struct Cfg {
  static constexpr int kThreads = kFp8 ? 32 * (kConvWarp0 + kConvWarps) : 320;
  static constexpr int kStages = 7;
  static constexpr uint32_t kOffScale = kOffRing + kStages * kStageBytes;
  static constexpr uint32_t kOffBar = kOffScale + (kFp8 ? kStages * kScaleSlot : 0);
  static constexpr uint32_t kOffTmemPtr = kOffBar + 8 * B_COUNT;
  static constexpr uint32_t kOffAbort = kOffTmemPtr + 4;
  static constexpr uint32_t kOffPM = kOffBar + kBarArea;  // row maxes [2 parity][4 pages][64]
  static constexpr uint32_t kOffPL = kOffPM + 2 * 4 * 64 * 4;  // row sums [4 pages][64]
  static constexpr uint32_t kSmemBytes = kOffPL + 4 * 64 * 4;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert((kOffScale & 15) == 0, "scale slot alignment");
  static_assert(kStages <= kMaxStages, "barrier arrays too small");
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;      // [0, 256): output accumulator, chunk j at 128 j
constexpr uint32_t kTmemS = 256;    // [256, 512): two 128-column score buffers
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct PairArgs {
  const unsigned char *plan;
  const int32_t *block_table;
  int max_pages, num_pages;
  int q_len, n_h;
  float scale_log2;
  float *ws_o, *ws_lse;
  uint16_t *o_latent;
  float *lse;
  uint32_t *status;
  uint64_t wait_ns;     // bound of every barrier wait
  int suppress_arrive;  // test hook: skip the first arrival on stage 0
  const float *scales;  // FP8 cache: [num_pages][64] per-token scales
  const unsigned char *fp8_pool;  // FP8 cache: [num_pages][64][640] (L2 prefetch)
};

struct Ctx {
  uint32_t bar_base;
  volatile int *abort_flag;
  uint32_t *status;
  uint64_t wait_ns;
  __device__ uint32_t bar(int i) const { return bar_base + 8u * i; }
};

// Bounded wait on an mbarrier phase (acquire at cluster scope when `cluster`).
// Returns false on timeout or when another thread of the CTA has aborted.
__device__ __noinline__ bool wait_bar(const Ctx &c, uint32_t bar, uint32_t parity, bool cluster) {
  if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*c.abort_flag) return false;
      if (globaltimer_ns() - t0 > c.wait_ns) {
        *c.abort_flag = 1;
        report(c.status, MLA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// Wait used to drain work this CTA issued before it leaves: ignores the abort
// flag (the loads and MMAs in flight must land first) but keeps the time cap.
__device__ __noinline__ bool wait_drain(const Ctx &c, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 63 && globaltimer_ns() - t0 > c.wait_ns) {
      report(c.status, MLA_DEV_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ bool wait_fast(const Ctx &c, uint32_t bar, uint32_t parity,
                                          bool cluster) {
  if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  return wait_bar(c, bar, parity, cluster);
}

// Whole warp: every lane polls, the warp proceeds only if all succeeded.
__device__ __forceinline__ bool wait_warp(const Ctx &c, uint32_t bar, uint32_t parity,
                                          bool cluster) {
  const bool ok = wait_fast(c, bar, parity, cluster);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

// 2^x with the MUFU approximation (relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// float -> bf16 with round-to-nearest-even on the bit pattern (integer ALU
// only, leaving the conversion unit to ex2). The rounded value is returned in
// the high half with the low half zero, i.e. as the bits of the float it
// equals. Inputs are finite.
__device__ __forceinline__ uint32_t rne_bf16_hi(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return u & 0xFFFF0000u;
}

// two rounded values (bf16 in the high halves) -> packed bf16 pair, a low
__device__ __forceinline__ uint32_t pack_hi_pair(uint32_t a_hi, uint32_t b_hi) {
  return __byte_perm(a_hi, b_hi, 0x7632);
}

__device__ __forceinline__ int tiles_of(int np) { return (np + kTilePages - 1) / kTilePages; }

// fp16 helpers of the FP8 instance (its MMA operands are fp16: every E4M3
// code times a power-of-two scale, every bf16 query and k^R value in the
// normal fp16 range, and the probabilities are exact or correctly rounded
// there).
// 4 E4M3 codes (element 0 lowest) -> two packed fp16 pairs, exactly.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t &d0, uint32_t &d1) {
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n"
      " cvt.rn.f16x2.e4m3x2 %1, hi;\n}"
      : "=r"(d0), "=r"(d1)
      : "r"(w));
}
__device__ __forceinline__ uint32_t hmul2_f16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// (lo, hi) floats -> packed fp16 pair, round to nearest even
__device__ __forceinline__ uint32_t f16x2_pack(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint32_t f16x2_splat(float x) { return f16x2_pack(x, x); }
// packed bf16 pair -> packed fp16 pair
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return f16x2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// 1 when either half is an fp16 infinity or NaN
__device__ __forceinline__ uint32_t f16x2_inf_bits(uint32_t d) {
  return ((d & 0x7C00u) == 0x7C00u || (d & 0x7C000000u) == 0x7C000000u) ? 1u : 0u;
}

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<kFp8>::kThreads, 1)
decode_pair_kernel(const __grid_constant__ CUtensorMap tm_cache,
                   const __grid_constant__ CUtensorMap tm_q, const PairArgs a) {
  constexpr int kStages = Cfg<kFp8>::kStages;
  constexpr uint32_t kOffTmemPtr = Cfg<kFp8>::kOffTmemPtr;
  constexpr uint32_t kOffAbort = Cfg<kFp8>::kOffAbort;
  constexpr uint32_t kOffPM = Cfg<kFp8>::kOffPM;
  constexpr uint32_t kOffPL = Cfg<kFp8>::kOffPL;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  unsigned char *smem = smem_raw;
  if (base & 1023u) {
    // the swizzled tiles need a 1024-byte aligned base; both CTAs of the
    // cluster see the same layout, so both leave here
    if (threadIdx.x == 0) report(a.status, MLA_DEV_BAD_PLAN);
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int list = blockIdx.x >> 1;

  Ctx c;
  c.bar_base = base + Cfg<kFp8>::kOffBar;
  c.abort_flag = reinterpret_cast<volatile int *>(smem + kOffAbort);
  c.status = a.status;
  c.wait_ns = a.wait_ns;

  if (threadIdx.x == 0) {
    *c.abort_flag = 0;
    for (int i = 0; i < kStages; ++i) {
      // FP8: the converter warp that owns the stage arrives, in both CTAs
      mbar_init(c.bar(B_FULL0 + i), kFp8 ? 2 : 1);
      mbar_init(c.bar(B_EMPTY0 + i), 1);
    }
    if (kFp8)
      for (int i = 0; i < kStages; ++i) mbar_init(c.bar(B_LFULL0 + i), 1);
    mbar_init(c.bar(B_QFULL), 1);
    mbar_init(c.bar(B_QEMPTY), 1);
    mbar_init(c.bar(B_QCONV), 2 * kConvWarps);
    mbar_init(c.bar(B_SFULL0), 1);
    mbar_init(c.bar(B_SFULL1), 1);
    mbar_init(c.bar(B_SFREE0), 16);
    mbar_init(c.bar(B_SFREE1), 16);
    mbar_init(c.bar(B_PFULL), 16);
    mbar_init(c.bar(B_PVDONE), 1);
    mbar_init(c.bar(B_PMAX0), 8);
    mbar_init(c.bar(B_PMAX1), 8);
    mbar_init(c.bar(B_EPI), 8);
    mbar_init(c.bar(B_FINAL), 1);
    fence_mbar_init_cluster();
  }
  if (warp == kMmaWarp) tmem_alloc_pair(base + kOffTmemPtr, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before any remote arrive or load
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffTmemPtr);

  const PlanHeader *ph = reinterpret_cast<const PlanHeader *>(a.plan);
  const int32_t *cta_begin = reinterpret_cast<const int32_t *>(a.plan + ph->cta_off);
  const WorkItem *items = reinterpret_cast<const WorkItem *>(a.plan + ph->items_off);
  const int i0 = cta_begin[list], i1 = cta_begin[list + 1];

  const uint32_t q_s = base + kOffQ, p_s = base + kOffP, ring = base + kOffRing;
  const uint32_t scale_s = base + Cfg<kFp8>::kOffScale;
  // barriers of the even CTA, as seen from this CTA
  const uint32_t lead_full0 = mapa_shared(c.bar(B_FULL0), 0);
  const uint32_t lead_qfull = mapa_shared(c.bar(B_QFULL), 0);
  // page ids of tile t of an item: -2 for pages past the item's end; a bad id
  // is reported and replaced by page 0 (loaded, then masked by the softmax)
  auto tile_pages = [&](const WorkItem &wi, int t, bool check, int (&ids)[kTilePages]) {
    const int32_t *row_pages = a.block_table + (size_t)wi.b * a.max_pages;
#pragma unroll
    for (int p = 0; p < kTilePages; ++p) {
      const int pg = wi.page_begin + kTilePages * t + p;
      int id = -2;
      if (pg < wi.page_end) {
        id = pg < a.max_pages ? row_pages[pg] : -1;
        if (id < 0 || id >= a.num_pages) {
          if (check) report(a.status, MLA_DEV_BAD_PAGE);
          id = 0;
        }
      }
      ids[p] = id;
    }
  };

  if (kFp8 && warp == kProducerWarp) {
    // ------------------------------------------------ FP8 producer ---
    // The same stage sequence as the bf16 producer, every load to this CTA's
    // own barriers. Score chunks 2g and 2g+1 come as a pair of stages: the
    // CTA's two pages' code columns [128 g, +128) (128-byte swizzle) land in
    // the first stage, which the converters expand into both; the RoPE stage
    // gets the pages' bf16 k^R as it is; an output stage gets one page's
    // code columns in its upper half. Code stages also get the pages' token
    // scales in the stage's scale slot. Every stage's landing barrier
    // completes once per use (a pair's second stage by a plain arrive).
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(&tm_q);
      uint32_t sg = 0, ic = 0, q_armed = 0;
      bool ok = true;
      auto acquire = [&](uint32_t seq, uint32_t &stg) -> bool {
        stg = seq % kStages;
        return seq < (uint32_t)kStages ||
               wait_fast(c, c.bar(B_EMPTY0 + stg), ((seq / kStages) - 1) & 1, false);
      };
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        const int T = tiles_of(wi.page_end - wi.page_begin);
        if (ic > 0 && !wait_bar(c, c.bar(B_QEMPTY), (ic - 1) & 1, false)) { ok = false; break; }
        // this CTA's 64 query rows, to its own barrier (the converters make
        // the latent part fp16 before the MMA issuer sees it)
        mbar_arrive_expect_tx(c.bar(B_QFULL), kChunksQK * kBox);
        ++q_armed;
        const int tq = wi.b * a.q_len + wi.j;
        for (int ch = 0; ch < kChunksQK; ++ch)
          tma_load_3d(q_s + ch * kBox, &tm_q, 64 * ch, 64 * (int)rank, tq, c.bar(B_QFULL));
        int ids_prev[kTilePages], ids_cur[kTilePages];
        // this CTA's two pages of tile u (codes, k^R and scales) into L2
        auto prefetch_tile = [&](int u) {
          if (u >= T) return;
          int ids[kTilePages];
          tile_pages(wi, u, false, ids);
          for (int e = 0; e < 2; ++e) {
            const int id = ids[2 * rank + e];
            if (id < 0) continue;
            bulk_prefetch_l2(a.fp8_pool + (size_t)id * 64 * kFp8RowBytes, 64 * kFp8RowBytes);
            bulk_prefetch_l2(a.scales + (size_t)id * 64, 256);
          }
        };
        for (int u = 0; u < kFp8PrefetchTiles; ++u) prefetch_tile(u);
        auto load_qk = [&](const int (&ids)[kTilePages]) -> bool {
          const int id0 = ids[2 * rank], id1 = ids[2 * rank + 1];
          const uint32_t npres = (id0 != -2 ? 1u : 0u) + (id1 != -2 ? 1u : 0u);
          for (int g = 0; g < (kChunksQK - 1) / 2; ++g, sg += 2) {
            uint32_t s0, s1;
            if (!acquire(sg, s0) || !acquire(sg + 1, s1)) return false;
            const uint32_t bar = c.bar(B_LFULL0 + s0);
            mbar_arrive_expect_tx(bar, npres * (kBox + 256));
            for (int e = 0; e < 2; ++e) {
              const int id = e ? id1 : id0;
              if (id == -2) continue;
              tma_load_2d(ring + s0 * kStageBytes + e * kBox, &tm_cache, 128 * g, id * 64, bar);
              bulk_load(scale_s + s0 * kScaleSlot + e * 256, a.scales + (size_t)id * 64, 256, bar);
            }
            mbar_arrive(c.bar(B_LFULL0 + s1));
          }
          uint32_t st;
          if (!acquire(sg, st)) return false;
          const uint32_t bar = c.bar(B_LFULL0 + st);
          mbar_arrive_expect_tx(bar, npres * kBox);
          for (int e = 0; e < 2; ++e) {
            const int id = e ? id1 : id0;
            if (id != -2) tma_load_2d(ring + st * kStageBytes + e * kBox, &tm_cache, MLA_D_C,
                                      id * 64, bar);
          }
          ++sg;
          return true;
        };
        auto load_pv = [&](const int (&ids)[kTilePages]) -> bool {
          for (int j = 0; j < 2; ++j)
            for (int p = 0; p < kTilePages; ++p) {
              if (ids[p] == -2) continue;
              uint32_t stg;
              if (!acquire(sg, stg)) return false;
              const uint32_t st = ring + stg * kStageBytes, bar = c.bar(B_LFULL0 + stg);
              mbar_arrive_expect_tx(bar, kHalfStage + 256);
              tma_load_2d(st + kHalfStage, &tm_cache, 256 * j + 128 * (int)rank, ids[p] * 64, bar);
              bulk_load(scale_s + stg * kScaleSlot, a.scales + (size_t)ids[p] * 64, 256, bar);
              ++sg;
            }
          return true;
        };
        for (int t = 0; t < T && ok; ++t) {
          tile_pages(wi, t, true, ids_cur);
          if (kFp8PrefetchTiles > 0) prefetch_tile(t + kFp8PrefetchTiles);
          if (!load_qk(ids_cur)) { ok = false; break; }
          if (t >= 1 && !load_pv(ids_prev)) { ok = false; break; }
#pragma unroll
          for (int p = 0; p < kTilePages; ++p) ids_prev[p] = ids_cur[p];
        }
        if (ok && !load_pv(ids_prev)) ok = false;
      }
      // drain: every load completes on this CTA's own barriers
      bool drained = true;
      for (uint32_t k = sg > (uint32_t)kStages ? sg - kStages : 0; k < sg && drained; ++k)
        drained = wait_drain(c, c.bar(B_LFULL0 + k % kStages), (k / kStages) & 1);
      if (q_armed && drained) wait_drain(c, c.bar(B_QFULL), (q_armed - 1) & 1);
    }
  } else if (kFp8 && warp >= kConvWarp0) {
    // ------------------------------------------------ FP8 converters ---
    // Walk the MMA issuer's stage sequence in units: a score chunk pair, the
    // RoPE stage, an output stage. Converter warp w owns the units whose
    // number is w modulo kConvWarps and expands each alone: wait for its
    // loads, then 16 rows at a time read the rows' codes into registers and
    // write their fp16 values (times each token's scale; 128-byte swizzle),
    // and hand the unit's stages to the MMA issuer. A row's fp16 values
    // overwrite only that row's own codes, so a batch reads before it writes
    // and no warp waits for another.
    const int cw = warp - kConvWarp0;
    const uint32_t lead_full = leader ? c.bar(B_FULL0) : lead_full0;
    const uint32_t lead_qconv = mapa_shared(c.bar(B_QCONV), 0);
    uint32_t sg = 0, ic = 0, un = 0;
    bool ok = true, range_bad = false;
    auto landed = [&](uint32_t seq, uint32_t &stg) -> bool {
      stg = seq % kStages;
      return wait_warp(c, c.bar(B_LFULL0 + stg), (seq / kStages) & 1, false);
    };
    auto arrive_full = [&](uint32_t seq) {
      if (lane == 0) {
        if (leader)
          mbar_arrive(lead_full + 8 * (seq % kStages));
        else
          mbar_arrive_remote(lead_full + 8 * (seq % kStages));
      }
    };
    auto mine = [&]() { return (int)(un++ % kConvWarps) == cw; };
    // 16 codes of one token -> 16 fp16 values code * scale (exact for scales
    // in [2^-15, 2^7]: the products are on the fp16 grid; larger scales can
    // overflow and are reported)
    // (Integer bit placement of the codes, code * 2^-8 then times scale *
    // 2^8, measured slower than the conversion instruction, alone or for
    // half the codes: 201 and 186 against 174 us on the 64 x 4096 workload.)
    auto expand16 = [&](const uint4 &v, float sc, uint4 &o0, uint4 &o1) {
      range_bad |= sc > 128.f;
      const uint32_t s2 = f16x2_splat(sc);
      uint32_t d[8];
      e4m3x4_to_f16x2(v.x, d[0], d[1]);
      e4m3x4_to_f16x2(v.y, d[2], d[3]);
      e4m3x4_to_f16x2(v.z, d[4], d[5]);
      e4m3x4_to_f16x2(v.w, d[6], d[7]);
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = hmul2_f16(d[i], s2);
      o0 = make_uint4(d[0], d[1], d[2], d[3]);
      o1 = make_uint4(d[4], d[5], d[6], d[7]);
    };
    // Rows [r_begin, r_end) of 128 codes (128-byte swizzle) at `src` + row *
    // 128, scales at `sc_s` + row * 4: codes [0, 64) of a row go to `dst0`,
    // [64, 128) to `dst1` (both 64 fp16 a row, 128-byte swizzle). When dst0
    // or dst1 is src, each row overwrites only itself.
    auto expand_rows = [&](uint32_t src, uint32_t sc_s, uint32_t dst0, uint32_t dst1,
                           int r_begin, int r_end) {
#pragma unroll 1
      for (int r0 = r_begin; r0 < r_end; r0 += 16) {
        uint4 v[4];
        float sc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int U = 32 * k + lane, t = r0 + (U >> 3), u = U & 7;
          v[k] = lds128(src + t * 128 + ((u ^ (t & 7)) << 4));
          sc[k] = lds_f32(sc_s + 4 * t);
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int U = 32 * k + lane, t = r0 + (U >> 3), u = U & 7, sw = t & 7;
          uint4 o0, o1;
          expand16(v[k], sc[k], o0, o1);
          const uint32_t row = ((u >> 2) ? dst1 : dst0) + t * 128;
          const int lu = 2 * (u & 3);
          sts128(row + ((lu ^ sw) << 4), o0);
          sts128(row + (((lu + 1) ^ sw) << 4), o1);
        }
        __syncwarp();
      }
    };
    auto conv_pv = [&](const int (&ids)[kTilePages]) -> bool {
      for (int j = 0; j < 2; ++j)
        for (int p = 0; p < kTilePages; ++p) {
          if (ids[p] == -2) continue;
          const uint32_t seq = sg++;
          if (!mine()) continue;
          uint32_t stg;
          if (!landed(seq, stg)) return false;
          // one page: the second 64-column box of row t is row t's codes
          const uint32_t st = ring + stg * kStageBytes;
          expand_rows(st + kHalfStage, scale_s + stg * kScaleSlot, st, st + kBox, 0, 64);
          fence_proxy_async_smem();
          __syncwarp();
          arrive_full(seq);
        }
      return true;
    };
    for (int it = i0; it < i1 && ok; ++it, ++ic) {
      const WorkItem wi = items[it];
      const int T = tiles_of(wi.page_end - wi.page_begin);
      // the item's latent query columns (chunks 0-7) to fp16, a quarter per
      // warp; the RoPE chunk stays bf16
      {
        if (!wait_warp(c, c.bar(B_QFULL), ic & 1, false)) { ok = false; break; }
        constexpr int kQUnits = (kChunksQK - 1) * (int)kBox / 16 / kConvWarps;
        uint32_t bad = 0;
        const uint32_t q0 = q_s + 16 * kQUnits * cw;
#pragma unroll 4
        for (int k = lane; k < kQUnits; k += 32) {
          const uint4 v = lds128(q0 + 16 * k);
          const uint4 o = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y),
                                     bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
          bad |= f16x2_inf_bits(o.x) | f16x2_inf_bits(o.y) | f16x2_inf_bits(o.z) |
                 f16x2_inf_bits(o.w);
          sts128(q0 + 16 * k, o);
        }
        range_bad |= bad != 0;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(c.bar(B_QCONV));
          else
            mbar_arrive_remote(lead_qconv);
        }
      }
      int ids_prev[kTilePages], ids_cur[kTilePages];
      for (int t = 0; t < T && ok; ++t) {
        tile_pages(wi, t, false, ids_cur);
        const bool pres[2] = {ids_cur[2 * rank] != -2, ids_cur[2 * rank + 1] != -2};
        // score chunk pairs: page e's codes at e * 8 KB of the first stage
        for (int g = 0; g < (kChunksQK - 1) / 2; ++g, sg += 2) {
          if (!mine()) continue;
          uint32_t s0;
          if (!landed(sg, s0)) { ok = false; break; }
          const uint32_t s1 = (sg + 1) % kStages;
          for (int e = 0; e < 2; ++e) {
            if (!pres[e]) continue;
            const uint32_t src = ring + s0 * kStageBytes + e * kBox;
            expand_rows(src, scale_s + s0 * kScaleSlot + e * 256, src,
                        ring + s1 * kStageBytes + e * kBox, 0, 64);
          }
          fence_proxy_async_smem();
          __syncwarp();
          arrive_full(sg);
          arrive_full(sg + 1);
        }
        if (!ok) break;
        // the RoPE stage: the pages' bf16 k^R as landed
        if (mine()) {
          uint32_t st;
          if (!landed(sg, st)) { ok = false; break; }
          arrive_full(sg);
        }
        ++sg;
        if (t >= 1 && !conv_pv(ids_prev)) { ok = false; break; }
#pragma unroll
        for (int p = 0; p < kTilePages; ++p) ids_prev[p] = ids_cur[p];
      }
      if (ok && !conv_pv(ids_prev)) ok = false;
    }
    if (__any_sync(0xffffffffu, range_bad) && lane == 0) report(a.status, MLA_DEV_RANGE);
  } else if (!kFp8 && warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(&tm_q);
      uint32_t sg = 0, ic = 0, q_armed = 0;
      uint32_t armed[kStages] = {};
      bool ok = true;
      auto acquire_stage = [&](uint32_t &stg) -> bool {
        stg = sg % kStages;
        if (sg >= kStages && !wait_fast(c, c.bar(B_EMPTY0 + stg), ((sg / kStages) - 1) & 1, false))
          return false;
        return true;
      };
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        const int np = wi.page_end - wi.page_begin;
        const int T = tiles_of(np);
        if (ic > 0 && !wait_bar(c, c.bar(B_QEMPTY), (ic - 1) & 1, false)) { ok = false; break; }
        if (leader) {
          mbar_arrive_expect_tx(c.bar(B_QFULL), 2 * kChunksQK * kBox);
          ++q_armed;
        }
        const int tq = wi.b * a.q_len + wi.j;
        for (int ch = 0; ch < kChunksQK; ++ch)
          tma_load_3d_pair(q_s + ch * kBox, &tm_q, 64 * ch, 64 * (int)rank, tq, lead_qfull);

        int ids_prev[kTilePages], ids_cur[kTilePages];
        auto load_qk = [&](const int (&ids)[kTilePages]) -> bool {
          int present = 0;
#pragma unroll
          for (int p = 0; p < kTilePages; ++p) present += ids[p] != -2;
          for (int ch = 0; ch < kChunksQK; ++ch, ++sg) {
            uint32_t stg;
            if (!acquire_stage(stg)) return false;
            if (leader && !(a.suppress_arrive && sg == 0)) {
              mbar_arrive_expect_tx(c.bar(B_FULL0 + stg), present * kBox);
              ++armed[stg];
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int id = ids[2 * rank + h];
              if (id != -2)
                tma_load_2d_pair(ring + stg * kStageBytes + h * kBox, &tm_cache, 64 * ch, id * 64,
                                 lead_full0 + 8 * stg);
            }
          }
          return true;
        };
        auto load_pv = [&](const int (&ids)[kTilePages]) -> bool {
          for (int j = 0; j < 2; ++j)
            for (int p = 0; p < kTilePages; ++p) {
              if (ids[p] == -2) continue;
              uint32_t stg;
              if (!acquire_stage(stg)) return false;
              if (leader) {
                mbar_arrive_expect_tx(c.bar(B_FULL0 + stg), 4 * kBox);
                ++armed[stg];
              }
              const int vc = 256 * j + 128 * (int)rank;
              tma_load_2d_pair(ring + stg * kStageBytes, &tm_cache, vc, ids[p] * 64,
                               lead_full0 + 8 * stg);
              tma_load_2d_pair(ring + stg * kStageBytes + kBox, &tm_cache, vc + 64, ids[p] * 64,
                               lead_full0 + 8 * stg);
              ++sg;
            }
          return true;
        };
        for (int t = 0; t < T && ok; ++t) {
          tile_pages(wi, t, true, ids_cur);
          if (!load_qk(ids_cur)) { ok = false; break; }
          if (t >= 1 && !load_pv(ids_prev)) { ok = false; break; }
#pragma unroll
          for (int p = 0; p < kTilePages; ++p) ids_prev[p] = ids_cur[p];
        }
        if (ok && !load_pv(ids_prev)) ok = false;
      }
      // drain: the loads issued into every stage have landed before the CTA
      // leaves (the even CTA sees both CTAs' bytes on its barriers; the odd
      // CTA sees its stages consumed). After an abort a barrier may never
      // complete; one expired wait (>= the wait cap) is then long enough for
      // every load in flight to have landed, so the drain stops there.
      bool drained = true;
      if (leader) {
        for (int s = 0; s < kStages && drained; ++s)
          if (armed[s]) drained = wait_drain(c, c.bar(B_FULL0 + s), (armed[s] - 1) & 1);
        if (q_armed && drained) wait_drain(c, c.bar(B_QFULL), (q_armed - 1) & 1);
      } else {
        for (uint32_t k = sg > kStages ? sg - kStages : 0; k < sg && drained; ++k)
          drained = wait_drain(c, c.bar(B_EMPTY0 + k % kStages), (k / kStages) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    if (leader && lane == 0) {
      // the FP8 instance's latent operands are fp16 (converted), its RoPE
      // chunk and every operand of the bf16 instance bf16
      constexpr uint32_t idesc_qk = idesc_f16kind(128, 256, 0, 0, !kFp8);
      constexpr uint32_t idesc_qr = idesc_f16kind(128, 256, 0, 0, true);
      constexpr uint32_t idesc_pv = idesc_f16kind(128, 256, 0, 1, !kFp8);
      uint32_t sg = 0, tg = 0, ic = 0, npv = 0;
      bool ok = true;
      auto take_stage = [&](uint32_t &stg) -> bool {
        stg = sg % kStages;
        if (!wait_fast(c, c.bar(B_FULL0 + stg), (sg / kStages) & 1, true)) return false;
        tc_fence_after();
        return true;
      };
      // output MMAs of tile u of the current item (npg pages)
      auto pv = [&](int u, int npg) -> bool {
        if (!wait_fast(c, c.bar(B_PFULL), npv & 1, true)) return false;
        ++npv;
        tc_fence_after();
        for (int j = 0; j < 2; ++j)
          for (int p = 0; p < npg; ++p, ++sg) {
            uint32_t stg;
            if (!take_stage(stg)) return false;
            const uint32_t st = ring + stg * kStageBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc(p_s + p * kBox + kk * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(st + kk * 2048, kBox, 1024, kSwizzle128B);
              mma_f16_ss_pair(tmem + kTmemO + 128 * j, ad, bd, idesc_pv,
                              (u == 0 && p == 0 && kk == 0) ? 0u : 1u);
            }
            mma_commit_pair(c.bar(B_EMPTY0 + stg));
          }
        mma_commit_pair(c.bar(B_PVDONE));
        return true;
      };
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        const int np = wi.page_end - wi.page_begin;
        const int T = tiles_of(np);
        if (!wait_bar(c, c.bar(kFp8 ? B_QCONV : B_QFULL), ic & 1, true)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < T; ++t, ++tg) {
          const int sb = tg & 1;
          if (tg >= 2 && !wait_fast(c, c.bar(B_SFREE0 + sb), ((tg >> 1) - 1) & 1, true)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + kTmemS + 128 * sb;
          for (int ch = 0; ch < kChunksQK && ok; ++ch, ++sg) {
            uint32_t stg;
            if (!take_stage(stg)) { ok = false; break; }
            const uint32_t st = ring + stg * kStageBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc(q_s + ch * kBox + kk * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(st + kk * 32, 16, 1024, kSwizzle128B);
              mma_f16_ss_pair(d, ad, bd, ch == kChunksQK - 1 ? idesc_qr : idesc_qk,
                              (ch | kk) ? 1u : 0u);
            }
            mma_commit_pair(c.bar(B_EMPTY0 + stg));
          }
          if (!ok) break;
          mma_commit_pair(c.bar(B_SFULL0 + sb));
          if (t == T - 1) mma_commit_pair(c.bar(B_QEMPTY));
          if (t >= 1 && !pv(t - 1, kTilePages)) { ok = false; break; }
        }
        if (!ok) break;
        if (!pv(T - 1, np - kTilePages * (T - 1))) { ok = false; break; }
      }
      mma_commit_pair_leader(c.bar(B_FINAL));
      wait_drain(c, c.bar(B_FINAL), 0);  // every MMA issued has completed
    }
  } else if (warp < kProducerWarp) {
    // ------------------------------------------- softmax + epilogue warps ---
    const int q4 = warp & 3;                 // TMEM lane quarter
    const int grp = warp >> 2;               // column group
    const int tl = 32 * q4 + lane;           // TMEM lane
    const int hh = tl & 63;                  // head within this CTA's 64
    const int half = tl >> 6;                // score columns hold tokens [128 half, +128)
    const int pidx = 2 * half + grp;         // the page of each tile this thread handles
    const int head = 64 * (int)rank + hh;
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const uint32_t p_row = p_s + pidx * kBox + (hh >> 3) * 1024 + (hh & 7) * 128;
    const int swz = hh & 7;
    float *pm = reinterpret_cast<float *>(smem + kOffPM);  // [parity][page][row]
    float *pl = reinterpret_cast<float *>(smem + kOffPL);  // [page][row]
    const uint32_t sfree0 = leader ? c.bar(B_SFREE0) : mapa_shared(c.bar(B_SFREE0), 0);
    const uint32_t pfull = leader ? c.bar(B_PFULL) : mapa_shared(c.bar(B_PFULL), 0);
    auto arrive_lead = [&](uint32_t bar) {
      if (leader)
        mbar_arrive(bar);
      else
        mbar_arrive_remote(bar);
    };
    uint32_t tg = 0, ic = 0;
    bool ok = true;

    for (int it = i0; it < i1 && ok; ++it, ++ic) {
      const WorkItem wi = items[it];
      const int np = wi.page_end - wi.page_begin;
      const int T = tiles_of(np);
      const int32_t *row_pages = a.block_table + (size_t)wi.b * a.max_pages;
      auto page_id = [&](int t) -> int {
        const int pg = wi.page_begin + kTilePages * t + pidx;
        if (t >= T || pg >= wi.page_end || pg >= a.max_pages) return -1;
        return row_pages[pg];
      };
      float m_ref = -INFINITY, lsum = 0.f;
      int id_next = page_id(0);
      for (int t = 0; t < T; ++t, ++tg) {
        const int sb = tg & 1;
        const int id = id_next;
        id_next = page_id(t + 1);
        const int pg = wi.page_begin + kTilePages * t + pidx;
        const bool valid = pg < wi.page_end && id >= 0 && id < a.num_pages;
        const int nvis = valid ? min(64, max(0, wi.qpos - pg * 64 + 1)) : 0;

        if (!wait_warp(c, c.bar(B_SFULL0 + sb), (tg >> 1) & 1, false)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[64];
        {
          uint32_t (&r0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[0]);
          uint32_t (&r1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[32]);
          const uint32_t s_addr = tmem + lane_off + kTmemS + 128 * sb + 64 * grp;
          tmem_ld32(s_addr, r0);
          tmem_ld32(s_addr + 32, r1);
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_lead(sfree0 + 8 * sb);

        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float v = i < nvis ? u2f(r[i]) * a.scale_log2 : -INFINITY;
          r[i] = f2u(v);
          mx4[i & 3] = fmaxf(mx4[i & 3], v);
        }
        // tile max of the row = max over its four pages (four threads)
        float mblk = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        pm[(sb * 4 + pidx) * 64 + hh] = mblk;
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(B_PMAX0 + sb));
        if (!wait_warp(c, c.bar(B_PMAX0 + sb), (tg >> 1) & 1, false)) { ok = false; break; }
        mblk = fmaxf(fmaxf(pm[(sb * 4 + 0) * 64 + hh], pm[(sb * 4 + 1) * 64 + hh]),
                     fmaxf(pm[(sb * 4 + 2) * 64 + hh], pm[(sb * 4 + 3) * 64 + hh]));
        float alpha = 1.f;
        bool resc = false;
        if (mblk > m_ref + kRescaleThreshold || (m_ref == -INFINITY && mblk > -INFINITY)) {
          if (m_ref > -INFINITY) {
            alpha = ex2_approx(m_ref - mblk);
            resc = true;
          }
          m_ref = mblk;
        }
        uint32_t pk[32];
        float ls4[4] = {0.f, 0.f, 0.f, 0.f};
        if (m_ref == -INFINITY) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        } else {
          if constexpr (kFp8) {
            // fp16 probabilities (p <= 2^8 under the lazy rescale); the sum
            // takes the unrounded values
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float p0 = ex2_approx(u2f(r[2 * i]) - m_ref);
              const float p1 = ex2_approx(u2f(r[2 * i + 1]) - m_ref);
              pk[i] = f16x2_pack(p0, p1);
              ls4[i & 3] += p0 + p1;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const uint32_t p0 = rne_bf16_hi(ex2_approx(u2f(r[2 * i]) - m_ref));
              const uint32_t p1 = rne_bf16_hi(ex2_approx(u2f(r[2 * i + 1]) - m_ref));
              pk[i] = pack_hi_pair(p0, p1);
              ls4[i & 3] += u2f(p0) + u2f(p1);  // the weights P*V uses
            }
          }
        }
        lsum = lsum * alpha + ((ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));

        // the previous tile's output MMAs are done: P buffer free, O stable
        if (t > 0) {
          if (!wait_warp(c, c.bar(B_PVDONE), (tg - 1) & 1, false)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, resc)) {
            // this thread's quarter of its head's accumulator: lane tl,
            // columns [128 grp, +128)
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t o[32];
              tmem_ld32(tmem + lane_off + kTmemO + 128 * grp + 32 * ch, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = f2u(u2f(o[e]) * alpha);
              tmem_st32(tmem + lane_off + kTmemO + 128 * grp + 32 * ch, o);
            }
            tmem_wait_st();
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4 *>(smem + (p_row - base) + ((q ^ swz) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_lead(pfull);
      }
      if (!ok) break;

      // epilogue: wait for the item's last output MMAs, combine the four page
      // sums of each row, write o (or a partial result)
      if (!wait_warp(c, c.bar(B_PVDONE), (tg - 1) & 1, false)) { ok = false; break; }
      tc_fence_after();
      pl[pidx * 64 + hh] = lsum;
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(B_EPI));
      if (!wait_warp(c, c.bar(B_EPI), ic & 1, false)) { ok = false; break; }
      const float lt = (pl[0 * 64 + hh] + pl[1 * 64 + hh]) + (pl[2 * 64 + hh] + pl[3 * 64 + hh]);
      const bool write = head < a.n_h;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const size_t row = ((size_t)wi.b * a.q_len + wi.j) * a.n_h + head;
      // TMEM columns [128 grp, +128) of lane tl are latent columns
      // [256 grp + 128 half, +128)
      const int d_base = 256 * grp + 128 * half;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + kTmemO + 128 * grp + 32 * ch, o);
        tmem_wait_ld();
        if (!write) continue;
        const int d0 = d_base + 32 * ch;
        if (wi.slot < 0) {
          uint4 *dst = reinterpret_cast<uint4 *>(a.o_latent + row * MLA_D_C + d0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(u2f(o[8 * q]) * inv, u2f(o[8 * q + 1]) * inv),
                                pack_bf16x2(u2f(o[8 * q + 2]) * inv, u2f(o[8 * q + 3]) * inv),
                                pack_bf16x2(u2f(o[8 * q + 4]) * inv, u2f(o[8 * q + 5]) * inv),
                                pack_bf16x2(u2f(o[8 * q + 6]) * inv, u2f(o[8 * q + 7]) * inv));
        } else {
          float4 *dst = reinterpret_cast<float4 *>(
              a.ws_o + ((size_t)wi.slot * a.n_h + head) * MLA_D_C + d0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(u2f(o[4 * q]) * inv, u2f(o[4 * q + 1]) * inv,
                                 u2f(o[4 * q + 2]) * inv, u2f(o[4 * q + 3]) * inv);
        }
      }
      tc_fence_before();
      if (write && pidx == 0) {
        const float lse = lt > 0.f ? (m_ref + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        if (wi.slot < 0) {
          if (a.lse != nullptr) a.lse[row] = lse;
        } else {
          a.ws_lse[(size_t)wi.slot * a.n_h + head] = lse;
        }
      }
      // The next item's first P (whose arrival the next output MMAs wait for)
      // is written only after this thread's accumulator reads completed.

    }
  }

  __syncthreads();
  cluster_sync();  // neither CTA leaves (or frees TMEM) while the pair may still use it
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
  __syncwarp();
  cluster_sync();
}

}  // namespace

// ------------------------------------------------------------------ host ---

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Cache pool [rows][576] bf16 as 64 x 64 tiles, 128-byte swizzle.
mla_status_t make_cache_map(CUtensorMap *tm, const void *base, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)MLA_ROW, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)MLA_ROW * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

// q_full [T][n_h][576] bf16 as (64 columns) x (64 heads) x (1 token) boxes;
// heads beyond n_h read as zeros.
mla_status_t make_query_map(CUtensorMap *tm, const void *base, int T, int n_h) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)MLA_ROW, (cuuint64_t)n_h, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)MLA_ROW * 2, (cuuint64_t)n_h * MLA_ROW * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

// failure-detection switch (mla_debug_decode_wait)
static uint64_t g_wait_ns = 1000000000ull;
static int g_suppress_arrive = 0;

mla_status_t set_decode_wait(double seconds, int suppress_arrive) {
  if (!(seconds > 0.0 && seconds <= 10.0))
    return fail(MLA_ERR_INVALID_ARGUMENT, "wait cap %g s outside (0, 10]", seconds);
  g_wait_ns = (uint64_t)(seconds * 1e9);
  g_suppress_arrive = suppress_arrive ? 1 : 0;
  return MLA_OK;
}

// FP8 cache pool [rows][640 bytes] as 64-row x 128-byte boxes, 128-byte
// swizzle: latent byte columns [128 g, +128) or the bf16 k^R at byte 512.
mla_status_t make_fp8_cache_map(CUtensorMap *tm, const void *base, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)kFp8RowBytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kFp8RowBytes};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

template <bool kFp8>
static mla_status_t launch_pair(const DecodeArgs &a, cudaStream_t stream) {
  const PlanHeader *ph = a.plan_host;
  if (ph->num_items == 0 || ph->num_ctas == 0) return MLA_OK;
  CUtensorMap tm_cache, tm_q;
  const uint64_t rows = (uint64_t)a.num_pages * MLA_PAGE;
  mla_status_t st = kFp8 ? make_fp8_cache_map(&tm_cache, a.cache, rows)
                         : make_cache_map(&tm_cache, a.cache, rows);
  if (st != MLA_OK) return st;
  st = make_query_map(&tm_q, a.q_full, a.batch * a.q_len, a.n_h);
  if (st != MLA_OK) return st;
  PairArgs t;
  t.plan = a.plan_dev;
  t.block_table = a.block_table;
  t.max_pages = a.max_pages;
  t.num_pages = a.num_pages;
  t.q_len = a.q_len;
  t.n_h = a.n_h;
  t.scale_log2 = a.scale_log2;
  t.ws_o = a.ws_o;
  t.ws_lse = a.ws_lse;
  t.o_latent = a.o_latent;
  t.lse = a.lse;
  t.status = a.status;
  t.wait_ns = g_wait_ns;
  t.suppress_arrive = g_suppress_arrive;
  t.scales = a.fp8_scales;
  t.fp8_pool = kFp8 ? reinterpret_cast<const unsigned char *>(a.cache) : nullptr;
  // the shared-memory opt-in is a per-device attribute: set it once per device
  static std::mutex mu;
  static bool set[64] = {};
  int dev = 0;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MLA_ERR_UNSUPPORTED, "device index %d", dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set[dev]) {
      MLA_CUDA_TRY(cudaFuncSetAttribute(decode_pair_kernel<kFp8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)Cfg<kFp8>::kSmemBytes));
      set[dev] = true;
    }
  }
  decode_pair_kernel<kFp8><<<2 * ph->num_ctas, Cfg<kFp8>::kThreads, Cfg<kFp8>::kSmemBytes,
                             stream>>>(tm_cache, tm_q, t);
  MLA_LAUNCH_CHECK(kFp8 ? "decode_pair_kernel<fp8>" : "decode_pair_kernel");
  return MLA_OK;
}

mla_status_t launch_decode_pair(const DecodeArgs &a, cudaStream_t stream) {
  return launch_pair<false>(a, stream);
}

mla_status_t launch_decode_fp8(const DecodeArgs &a, cudaStream_t stream) {
  return launch_pair<true>(a, stream);
}

}  // namespace mla

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
constexpr int kConvThreads = 32 * kConvWarps;
constexpr int kTilePages = 4;                       // pages per score tile (256 tokens)
constexpr int kChunksQK = MLA_ROW / 64;              // 9 column chunks of the score MMA
constexpr uint32_t kBox = 64 * 128;                  // 64 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kStageBytes = 2 * kBox;           // 16384
constexpr uint32_t kOffQ = 0;                        // 9 x [64 heads][64 cols]
constexpr uint32_t kOffP = kOffQ + kChunksQK * kBox; // 73728: 4 x [64 heads][64 tokens]
constexpr uint32_t kOffRing = kOffP + kTilePages * kBox;  // 106496: bf16 operand stages
constexpr uint32_t kLandStride = kBox + 1024;        // FP8 landing slot: 8 KB rows + scales
constexpr uint32_t kBarArea = 384;

constexpr int kMaxStages = 7;                        // capacity of the stage barrier arrays
constexpr int kMaxLand = 9;                          // capacity of the landing barrier arrays

enum {
  B_FULL0 = 0,                          // [kMaxStages] stage ready (even CTA)
  B_EMPTY0 = B_FULL0 + kMaxStages,      // [kMaxStages] stage consumed (both CTAs)
  B_LFULL0 = B_EMPTY0 + kMaxStages,     // [kMaxLand] FP8 landing slot loaded (local)
  B_LEMPTY0 = B_LFULL0 + kMaxLand,      // [kMaxLand] FP8 landing slot converted (local)
  B_QFULL = B_LEMPTY0 + kMaxLand,       // query rows loaded (even CTA: both CTAs' bytes)
  B_QEMPTY,                        // last score MMA of the item done (both)
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

// Shared-memory layout of the two instances. bf16 cache: a 7-stage ring of
// bf16 operand stages filled by TMA. FP8 cache: a 4-stage ring of the same
// bf16 stages, written by converter warps from a 6-slot ring of FP8 landing
// slots (one page x 128 byte columns, plus the page's 64 token scales).
template <bool kFp8>
struct Cfg {
  static constexpr int kThreads = kFp8 ? 32 * (kConvWarp0 + kConvWarps) : 320;
  static constexpr int kStages = kFp8 ? 2 : 7;
  static constexpr int kLand = kFp8 ? 9 : 0;
  static constexpr uint32_t kOffLand = kOffRing + kStages * kStageBytes;
  static constexpr uint32_t kOffBar = kOffLand + kLand * kLandStride;
  static constexpr uint32_t kOffTmemPtr = kOffBar + 8 * B_COUNT;
  static constexpr uint32_t kOffAbort = kOffTmemPtr + 4;
  static constexpr uint32_t kOffPM = kOffBar + kBarArea;  // row maxes [2 parity][4 pages][64]
  static constexpr uint32_t kOffPL = kOffPM + 2 * 4 * 64 * 4;  // row sums [4 pages][64]
  static constexpr uint32_t kSmemBytes = kOffPL + 4 * 64 * 4;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert((kOffLand & 1023) == 0 && (kLandStride & 1023) == 0, "landing alignment");
  static_assert(kStages <= kMaxStages && kLand <= kMaxLand, "barrier arrays too small");
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

// E4M3 -> float by bit placement: the code's sign goes to bit 31 and its 7
// exponent/mantissa bits to bits 26..20, which is the float 2^-120 times the
// code's value for normal and subnormal codes alike (the E4M3 subnormal
// 0.mmm x 2^-6 lands on the float subnormal 0.mmm x 2^-126). Multiplying by
// 2^120 and then by the power-of-two scale is exact, and so is keeping the
// upper 16 bits as the bf16 value (4 significant bits). Integer and FMA
// pipes only.
// 16 E4M3 codes (16 bytes, element 0 lowest) -> 16 bf16 values code * sc.
__device__ __forceinline__ void fp8x16_to_bf16(const uint4 &v, float sc, uint4 &o0, uint4 &o1) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const float k120 = 1.329227995784916e36f;   // 2^120
  uint32_t r[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = w[i];
    const uint32_t f0 = ((x << 24) & 0x80000000u) | ((x << 20) & 0x07F00000u);
    const uint32_t f1 = ((x << 16) & 0x80000000u) | ((x << 12) & 0x07F00000u);
    const uint32_t f2 = ((x << 8) & 0x80000000u) | ((x << 4) & 0x07F00000u);
    const uint32_t f3 = (x & 0x80000000u) | ((x >> 4) & 0x07F00000u);
    const float g0 = __uint_as_float(f0) * k120 * sc, g1 = __uint_as_float(f1) * k120 * sc;
    const float g2 = __uint_as_float(f2) * k120 * sc, g3 = __uint_as_float(f3) * k120 * sc;
    r[2 * i] = __byte_perm(__float_as_uint(g0), __float_as_uint(g1), 0x7632);
    r[2 * i + 1] = __byte_perm(__float_as_uint(g2), __float_as_uint(g3), 0x7632);
  }
  o0 = make_uint4(r[0], r[1], r[2], r[3]);
  o1 = make_uint4(r[4], r[5], r[6], r[7]);
}

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<kFp8>::kThreads, 1)
decode_pair_kernel(const __grid_constant__ CUtensorMap tm_cache,
                   const __grid_constant__ CUtensorMap tm_q, const PairArgs a) {
  constexpr int kStages = Cfg<kFp8>::kStages;
  constexpr int kLand = Cfg<kFp8>::kLand > 0 ? Cfg<kFp8>::kLand : 1;  // the bf16 instance has none
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
      // FP8: every converter warp of both CTAs arrives once per stage
      mbar_init(c.bar(B_FULL0 + i), kFp8 ? 2 * kConvWarps : 1);
      mbar_init(c.bar(B_EMPTY0 + i), 1);
    }
    for (int i = 0; i < kLand; ++i) {
      mbar_init(c.bar(B_LFULL0 + i), 1);
      mbar_init(c.bar(B_LEMPTY0 + i), kConvWarps);
    }
    mbar_init(c.bar(B_QFULL), 1);
    mbar_init(c.bar(B_QEMPTY), 1);
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
  const uint32_t land_s = base + Cfg<kFp8>::kOffLand;
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
    // ---------------------------------------- FP8 landing producer ---
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(&tm_q);
      uint32_t lc = 0, ic = 0, q_armed = 0;
      bool ok = true;
      // one landing slot: 64 rows x 128 bytes of the page at byte column x
      // (+ the page's 64 scales)
      auto land = [&](int x, int id, bool with_scales) -> bool {
        const uint32_t l = lc % kLand;
        if (lc >= kLand && !wait_fast(c, c.bar(B_LEMPTY0 + l), ((lc / kLand) - 1) & 1, false))
          return false;
        const uint32_t dst = land_s + l * kLandStride;
        mbar_arrive_expect_tx(c.bar(B_LFULL0 + l), kBox + (with_scales ? 256u : 0u));
        tma_load_2d(dst, &tm_cache, x, id * 64, c.bar(B_LFULL0 + l));
        if (with_scales) bulk_load(dst + kBox, a.scales + (size_t)id * 64, 256, c.bar(B_LFULL0 + l));
        ++lc;
        return true;
      };
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        const int T = tiles_of(wi.page_end - wi.page_begin);
        if (ic > 0 && !wait_bar(c, c.bar(B_QEMPTY), (ic - 1) & 1, false)) { ok = false; break; }
        if (leader) {
          mbar_arrive_expect_tx(c.bar(B_QFULL), 2 * kChunksQK * kBox);
          ++q_armed;
        }
        const int tq = wi.b * a.q_len + wi.j;
        for (int ch = 0; ch < kChunksQK; ++ch)
          tma_load_3d_pair(q_s + ch * kBox, &tm_q, 64 * ch, 64 * (int)rank, tq, lead_qfull);
        int ids_prev[kTilePages], ids_cur[kTilePages];
        auto land_qk = [&](const int (&ids)[kTilePages]) -> bool {
          for (int g = 0; g < 4; ++g)
            for (int e = 0; e < 2; ++e)
              if (ids[2 * rank + e] != -2 && !land(128 * g, ids[2 * rank + e], true)) return false;
          for (int e = 0; e < 2; ++e)
            if (ids[2 * rank + e] != -2 && !land(MLA_D_C, ids[2 * rank + e], false)) return false;
          return true;
        };
        auto land_pv = [&](const int (&ids)[kTilePages]) -> bool {
          for (int j = 0; j < 2; ++j)
            for (int p = 0; p < kTilePages; ++p)
              if (ids[p] != -2 && !land(128 * (2 * j + (int)rank), ids[p], true)) return false;
          return true;
        };
        for (int t = 0; t < T && ok; ++t) {
          tile_pages(wi, t, true, ids_cur);
          if (!land_qk(ids_cur)) { ok = false; break; }
          if (t >= 1 && !land_pv(ids_prev)) { ok = false; break; }
#pragma unroll
          for (int p = 0; p < kTilePages; ++p) ids_prev[p] = ids_cur[p];
        }
        if (ok && !land_pv(ids_prev)) ok = false;
      }
      // drain: every landing load completes on this CTA's own barriers
      bool drained = true;
      for (uint32_t k = lc > (uint32_t)kLand ? lc - kLand : 0; k < lc && drained; ++k)
        drained = wait_drain(c, c.bar(B_LFULL0 + k % kLand), (k / kLand) & 1);
      if (leader && q_armed && drained) wait_drain(c, c.bar(B_QFULL), (q_armed - 1) & 1);
    }
  } else if (kFp8 && warp >= kConvWarp0) {
    // ------------------------------------------------ FP8 converters ---
    // Walk the same stage sequence as the MMA issuer and the same landing
    // sequence as the producer; write bf16 operand stages (128-byte
    // swizzle) from the E4M3 landing slots, times each token's scale.
    const int ci = threadIdx.x - 32 * kConvWarp0;   // 0..kConvThreads-1
    const uint32_t lead_full = leader ? c.bar(B_FULL0) : lead_full0;
    uint32_t sg = 0, lc = 0;
    bool ok = true;
    auto take_stage = [&](uint32_t &stg) -> bool {
      stg = sg % kStages;
      return sg < (uint32_t)kStages ||
             wait_warp(c, c.bar(B_EMPTY0 + stg), ((sg / kStages) - 1) & 1, false);
    };
    auto give_stage = [&](uint32_t stg) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(lead_full + 8 * stg);
        else
          mbar_arrive_remote(lead_full + 8 * stg);
      }
      ++sg;
    };
    auto wait_land = [&](uint32_t k) {
      return wait_warp(c, c.bar(B_LFULL0 + k % kLand), (k / kLand) & 1, false);
    };
    auto free_land = [&](uint32_t k) {
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(B_LEMPTY0 + k % kLand));
    };
    auto slot = [&](uint32_t k) { return land_s + (k % kLand) * kLandStride; };
    for (int it = i0; it < i1 && ok; ++it) {
      const WorkItem wi = items[it];
      const int T = tiles_of(wi.page_end - wi.page_begin);
      int ids_prev[kTilePages], ids_cur[kTilePages];
      auto conv_pv = [&](const int (&ids)[kTilePages]) -> bool {
        for (int j = 0; j < 2; ++j)
          for (int p = 0; p < kTilePages; ++p) {
            if (ids[p] == -2) continue;
            uint32_t stg;
            if (!wait_land(lc) || !take_stage(stg)) return false;
            const uint32_t src = slot(lc), dst = ring + stg * kStageBytes;
#pragma unroll 4
            for (int k = 0; k < 512 / kConvThreads; ++k) {
              const int U = ci + kConvThreads * k, t = U >> 3, u = U & 7, sw = t & 7;
              const uint4 v = lds128(src + t * 128 + ((u ^ sw) << 4));
              uint4 o0, o1;
              fp8x16_to_bf16(v, lds_f32(src + kBox + 4 * t), o0, o1);
              const uint32_t row = dst + (u >> 2) * kBox + t * 128;
              const int lu = 2 * (u & 3);
              sts128(row + ((lu ^ sw) << 4), o0);
              sts128(row + (((lu + 1) ^ sw) << 4), o1);
            }
            give_stage(stg);
            free_land(lc);
            ++lc;
          }
        return true;
      };
      for (int t = 0; t < T && ok; ++t) {
        tile_pages(wi, t, false, ids_cur);
        const bool pres[2] = {ids_cur[2 * rank] != -2, ids_cur[2 * rank + 1] != -2};
        // score chunks 2g, 2g+1 from group g of the CTA's two pages
        for (int g = 0; g < 4 && ok; ++g) {
          const uint32_t k0 = lc, k1 = lc + (pres[0] ? 1 : 0);
          lc += (pres[0] ? 1 : 0) + (pres[1] ? 1 : 0);
          if ((pres[0] && !wait_land(k0)) || (pres[1] && !wait_land(k1))) { ok = false; break; }
          for (int h = 0; h < 2; ++h) {
            uint32_t stg;
            if (!take_stage(stg)) { ok = false; break; }
            const uint32_t dst = ring + stg * kStageBytes;
#pragma unroll 4
            for (int k = 0; k < 512 / kConvThreads; ++k) {
              const int U = ci + kConvThreads * k, e = U >> 8, t = (U >> 2) & 63, uu = U & 3,
                        sw = t & 7;
              if (!pres[e]) continue;
              const uint32_t src = slot(e ? k1 : k0);
              const int u = 4 * h + uu;
              const uint4 v = lds128(src + t * 128 + ((u ^ sw) << 4));
              uint4 o0, o1;
              fp8x16_to_bf16(v, lds_f32(src + kBox + 4 * t), o0, o1);
              const uint32_t row = dst + e * kBox + t * 128;
              sts128(row + (((2 * uu) ^ sw) << 4), o0);
              sts128(row + (((2 * uu + 1) ^ sw) << 4), o1);
            }
            give_stage(stg);
          }
          if (!ok) break;
          if (pres[0]) free_land(k0);
          if (pres[1]) free_land(k1);
        }
        if (!ok) break;
        // the RoPE chunk: bf16 rows copied unit by unit (same swizzle)
        {
          const uint32_t k0 = lc, k1 = lc + (pres[0] ? 1 : 0);
          lc += (pres[0] ? 1 : 0) + (pres[1] ? 1 : 0);
          uint32_t stg;
          if ((pres[0] && !wait_land(k0)) || (pres[1] && !wait_land(k1)) || !take_stage(stg)) {
            ok = false;
            break;
          }
          const uint32_t dst = ring + stg * kStageBytes;
#pragma unroll 4
          for (int k = 0; k < 1024 / kConvThreads; ++k) {
            const int U = ci + kConvThreads * k, e = U >> 9, t = (U >> 3) & 63, u = U & 7;
            if (!pres[e]) continue;
            const int off = t * 128 + ((u ^ (t & 7)) << 4);
            sts128(dst + e * kBox + off, lds128(slot(e ? k1 : k0) + off));
          }
          give_stage(stg);
          if (pres[0]) free_land(k0);
          if (pres[1]) free_land(k1);
        }
        if (t >= 1 && !conv_pv(ids_prev)) { ok = false; break; }
#pragma unroll
        for (int p = 0; p < kTilePages; ++p) ids_prev[p] = ids_cur[p];
      }
      if (ok && !conv_pv(ids_prev)) ok = false;
    }
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
      constexpr uint32_t idesc_qk = idesc_bf16(128, 256, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
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
        if (!wait_bar(c, c.bar(B_QFULL), ic & 1, true)) { ok = false; break; }
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
              mma_f16_ss_pair(d, ad, bd, idesc_qk, (ch | kk) ? 1u : 0u);
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
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t p0 = rne_bf16_hi(ex2_approx(u2f(r[2 * i]) - m_ref));
            const uint32_t p1 = rne_bf16_hi(ex2_approx(u2f(r[2 * i + 1]) - m_ref));
            pk[i] = pack_hi_pair(p0, p1);
            ls4[i & 3] += u2f(p0) + u2f(p1);  // the weights P*V uses
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
  mla_status_t st = kFp8 ? make_fp8_cache_map(&tm_cache, a.cache, (uint64_t)a.num_pages * MLA_PAGE)
                         : make_cache_map(&tm_cache, a.cache, (uint64_t)a.num_pages * MLA_PAGE);
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

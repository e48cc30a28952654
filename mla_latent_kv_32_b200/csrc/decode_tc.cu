// Absorbed MLA decode attention on the sm_100a tensor cores (tcgen05 + TMEM),
// fed by TMA, with split-KV work lists.
//
// What it computes ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide",
// "The Matrix Absorption Trick", parts 2-4, and "Step 3" of the PyTorch
// implementation): for one query token of one sequence and all heads h,
//   s_hi = (q~_h . c_i + q^R_h . k^R_i) * scale      (cached tokens i <= qpos)
//   o_h  = sum_i softmax(s_h)_i c_i                   (512-dim latent output)
// with the latent cache read once and shared by every head: the 128 heads are
// the M dimension of the MMAs, the 64 tokens of a cache page the N (scores) or
// K (output) dimension.
//
// Work split. The 128 x 512 fp32 latent accumulator alone fills one SM's tensor
// memory, so each work item runs on a cluster of two CTAs (two SMs):
//   CTA r = 0 owns latent columns [0, 256), CTA 1 owns [256, 576) (the last 64
//   are k^R). Each CTA TMA-loads only its column slab of every page, and of the
//   query rows, computes the partial scores S_r = Q_r C_r^T (M=128, N=64,
//   K=256 or 320), and sends them to its peer through distributed shared
//   memory. Both add S_0 + S_1 (the same bits in both, since fp32 addition
//   commutes), run the same online softmax, and accumulate
//   O[:, 256r : 256r+256] += P C[:, 256r : 256r+256] in their own TMEM.
// Every cache byte is read from global memory once per (item, query), and each
// MMA does distinct work: no head or column is computed twice.
//
// Warp roles (320 threads): warps 0-7 softmax + epilogue in two groups of four
// (thread = head = TMEM lane; group g handles score columns [32g, 32g+32) of
// every page and accumulator columns [128g, 128g+128); they also stage each
// item's query slab into TMEM), warp 8 TMA producer, warp 9 MMA issuer (and
// TMEM owner).
// Pipeline per page g: TMA(g) -> QK(g) -> [exchange, softmax](g) -> PV(g), with
// QK(g+1) issued before PV(g), four shared-memory page stages and two TMEM
// score buffers. The query is the A operand of QK straight from TMEM (its
// 256 latent columns; CTA 1's 64 RoPE columns come from shared memory), which
// leaves shared memory for the page stages that hide HBM latency.
// The running max is rescaled lazily: O and the sum are rescaled only when a
// row's max grows by more than 8 (log2 units); the final normalisation uses
// the same reference max, so the result is exact up to rounding.
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

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStages = 4;                            // page stages in shared memory
constexpr int kMaxBoxes = 5;                          // 64-column boxes per slab (CTA 1)
constexpr uint32_t kBoxQ = 128 * 128;                 // 128 query rows x 64 bf16
constexpr uint32_t kBoxT = 64 * 128;                  // 64 tokens x 64 bf16
constexpr uint32_t kStageBytes = kMaxBoxes * kBoxT;   // 40960
constexpr uint32_t kOffT = 0;
constexpr uint32_t kOffQR = kOffT + kStages * kStageBytes;  // 163840: RoPE query box (CTA 1)
constexpr uint32_t kOffP = kOffQR + kBoxQ;                  // 180224: P, 128 x 64 bf16
constexpr uint32_t kOffX = kOffP + 128 * 128;               // 196608: exchange, 2 x 128 x 64 bf16
constexpr uint32_t kXBytes = 128 * 128;                     // one exchange buffer
constexpr uint32_t kOffBar = kOffX + 128 * 256;             // 229376
constexpr uint32_t kOffPM = kOffBar + 256;                  // per-row partial maxes [2][2][128]
constexpr uint32_t kOffPL = kOffPM;  // per-row partial sums [2][128], epilogue only (reuses PM)
constexpr uint32_t kSmemUsed = kOffPM + 2 * 2 * 128 * 4;
// The dynamic shared window of sm_100 starts 1024-byte aligned (after the
// 1 KB reserved area); the kernel checks this and refuses to run otherwise.
constexpr uint32_t kSmemBytes = kSmemUsed;

// barrier slots (8 bytes each) in the barrier area
enum {
  B_TFULL0 = 0,                 // [kStages]
  B_TEMPTY0 = B_TFULL0 + kStages,  // [kStages]
  B_QFULL = B_TEMPTY0 + kStages,   // query slab staged in TMEM (softmax warps)
  B_QRFULL, B_QEMPTY, B_SFULL0, B_SFULL1, B_SFREE0, B_SFREE1, B_PFULL, B_PFREE, B_XFULL0,
  B_XFULL1, B_XEMPTY0, B_XEMPTY1, B_FINAL,
  B_PMAX0, B_PMAX1,  // both softmax groups posted their row maxes (per page parity)
  B_EPI,             // both groups posted their row sums (per item)
  B_COUNT
};
constexpr uint32_t kOffTmemPtr = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemPtr + 4;
static_assert(kOffAbort + 4 <= kOffPM, "barrier area overflow");
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;      // columns [0, 256): latent accumulator (fp32)
constexpr uint32_t kTmemQ = 256;    // columns [256, 384): query slab (bf16 pairs)
constexpr uint32_t kTmemS = 384;    // columns [384, 512): two 64-column score buffers
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct TcArgs {
  const unsigned char *plan;
  const uint16_t *q_full;
  long long q_rows;  // rows of q_full: batch * q_len * n_h
  const int32_t *block_table;
  int max_pages, num_pages;
  int q_len, n_h;
  float scale_log2;
  float *ws_o, *ws_lse;
  uint16_t *o_latent;
  float *lse;
  uint32_t *status;
};

struct Ctx {
  uint32_t base;   // shared address of the aligned smem area
  volatile int *abort_flag;
  uint32_t *status;
  __device__ uint32_t bar(int i) const { return base + kOffBar + 8u * i; }
};

// Bounded wait on an mbarrier phase. Returns false on timeout or when another
// thread of the CTA has already aborted.
__device__ __noinline__ bool wait_bar(const Ctx &c, uint32_t bar, uint32_t parity, bool cluster) {
  if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*c.abort_flag) return false;
      if (globaltimer_ns() - t0 > kTimeoutNs) {
        *c.abort_flag = 1;
        report(c.status, MLA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// Fast path inline (the phase is usually complete already), slow path bounded.
__device__ __forceinline__ bool wait_fast(const Ctx &c, uint32_t bar, uint32_t parity,
                                          bool cluster) {
  if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  return wait_bar(c, bar, parity, cluster);
}

// Same, for a whole warp: every lane polls, the warp proceeds only if all did.
__device__ __forceinline__ bool wait_bar_warp(const Ctx &c, uint32_t bar, uint32_t parity,
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

// float -> bf16 with round-to-nearest-even done on the bit pattern (integer
// ALU ops only; the conversion unit stays free for ex2). The rounded value is
// returned in the high half with the low half zero, i.e. as the bits of the
// float it equals. Inputs here are finite.
__device__ __forceinline__ uint32_t rne_bf16_hi(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return u & 0xFFFF0000u;
}

// two rounded values (bf16 in the high halves) -> packed bf16 pair, a low
__device__ __forceinline__ uint32_t pack_hi_pair(uint32_t a_hi, uint32_t b_hi) {
  return __byte_perm(a_hi, b_hi, 0x7632);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_cache,
                 const __grid_constant__ CUtensorMap tm_q, const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  unsigned char *smem = smem_raw;
  if (base & 1023u) {
    // the 128-byte swizzled tiles need a 1024-byte aligned base; both CTAs of
    // the cluster see the same layout, so both leave here
    if (threadIdx.x == 0) report(a.status, MLA_DEV_BAD_PLAN);
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int list = blockIdx.x >> 1;
  const int nbox = rank == 0 ? 4 : 5;
  const int col0 = rank == 0 ? 0 : 256;

  Ctx c;
  c.base = base;
  c.abort_flag = reinterpret_cast<volatile int *>(smem + kOffAbort);
  c.status = a.status;

  if (threadIdx.x == 0) {
    *c.abort_flag = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(c.bar(B_TFULL0 + i), 1);
      mbar_init(c.bar(B_TEMPTY0 + i), 1);
    }
    mbar_init(c.bar(B_QFULL), 8);    // the eight softmax warps
    mbar_init(c.bar(B_QRFULL), 1);
    mbar_init(c.bar(B_QEMPTY), 1);
    mbar_init(c.bar(B_SFULL0), 1);
    mbar_init(c.bar(B_SFULL1), 1);
    mbar_init(c.bar(B_SFREE0), 8);
    mbar_init(c.bar(B_SFREE1), 8);
    mbar_init(c.bar(B_PFULL), 8);
    mbar_init(c.bar(B_PFREE), 1);
    mbar_init(c.bar(B_XFULL0), 1);   // own arm (expect_tx) + the peer's st.async bytes
    mbar_init(c.bar(B_XFULL1), 1);
    mbar_init(c.bar(B_XEMPTY0), 8);  // the peer's eight softmax warps
    mbar_init(c.bar(B_XEMPTY1), 8);
    mbar_init(c.bar(B_FINAL), 1);
    mbar_init(c.bar(B_PMAX0), 8);
    mbar_init(c.bar(B_PMAX1), 8);
    mbar_init(c.bar(B_EPI), 8);
    // both exchange buffers start armed for the first two pages
    mbar_arrive_expect_tx(c.bar(B_XFULL0), kXBytes);
    mbar_arrive_expect_tx(c.bar(B_XFULL1), kXBytes);
    fence_mbar_init_cluster();
  }
  if (warp == kMmaWarp) tmem_alloc(base + kOffTmemPtr, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffTmemPtr);

  const PlanHeader *ph = reinterpret_cast<const PlanHeader *>(a.plan);
  const int32_t *cta_begin = reinterpret_cast<const int32_t *>(a.plan + ph->cta_off);
  const WorkItem *items = reinterpret_cast<const WorkItem *>(a.plan + ph->items_off);
  const int i0 = cta_begin[list], i1 = cta_begin[list + 1];

  const uint32_t qr_s = base + kOffQR, t_s = base + kOffT, p_s = base + kOffP, x_s = base + kOffX;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(&tm_q);
      uint32_t gb = 0, ic = 0, q_armed = 0, armed[kStages] = {};
      bool ok = true;
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        if (rank == 1) {
          // the 64 RoPE columns of the query rows (the rest is staged in TMEM)
          if (ic > 0 && !wait_bar(c, c.bar(B_QEMPTY), (ic - 1) & 1, false)) { ok = false; break; }
          mbar_arrive_expect_tx(c.bar(B_QRFULL), kBoxQ);
          ++q_armed;
          tma_load_2d(qr_s, &tm_q, MLA_D_C, (wi.b * a.q_len + wi.j) * a.n_h, c.bar(B_QRFULL));
        }
        const int32_t *row_pages = a.block_table + (size_t)wi.b * a.max_pages;
        int ids[4];  // page ids loaded four pages ahead
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int p = wi.page_begin + i;
          ids[i] = (p < wi.page_end && p < a.max_pages) ? row_pages[p] : -1;
        }
        for (int pg = wi.page_begin; pg < wi.page_end; ++pg, ++gb) {
          int page = ids[0];
          ids[0] = ids[1];
          ids[1] = ids[2];
          ids[2] = ids[3];
          {
            const int p = pg + 4;
            ids[3] = (p < wi.page_end && p < a.max_pages) ? row_pages[p] : -1;
          }
          const int s = gb % kStages;
          if (gb >= kStages &&
              !wait_fast(c, c.bar(B_TEMPTY0 + s), ((gb / kStages) - 1) & 1, false)) {
            ok = false;
            break;
          }
          if (page < 0 || page >= a.num_pages) {
            report(a.status, MLA_DEV_BAD_PAGE);
            page = 0;  // load something valid; the softmax warps mask the whole page
          }
          mbar_arrive_expect_tx(c.bar(B_TFULL0 + s), nbox * kBoxT);
          ++armed[s];
          for (int x = 0; x < nbox; ++x)
            tma_load_2d(t_s + s * kStageBytes + x * kBoxT, &tm_cache, col0 + 64 * x, page * 64,
                        c.bar(B_TFULL0 + s));
        }
      }
      // drain: every load this thread issued has landed before the CTA exits
      for (int s = 0; s < kStages; ++s)
        if (armed[s]) wait_bar(c, c.bar(B_TFULL0 + s), (armed[s] - 1) & 1, false);
      if (q_armed) wait_bar(c, c.bar(B_QRFULL), (q_armed - 1) & 1, false);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
      uint32_t gb = 0, ic = 0;
      bool ok = true;
      auto pv = [&](uint32_t g, uint32_t g0) -> bool {
        if (!wait_fast(c, c.bar(B_PFULL), g & 1, false)) return false;
        tc_fence_after();
        const uint32_t st = t_s + (g % kStages) * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = smem_desc(p_s + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(st + kk * 2048, 8192, 1024, kSwizzle128B);
          mma_f16_ss(tmem + kTmemO, ad, bd, idesc_pv, (g != g0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(c.bar(B_TEMPTY0 + (g % kStages)));
        mma_commit(c.bar(B_PFREE));
        return true;
      };
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        if (!wait_bar(c, c.bar(B_QFULL), ic & 1, false)) { ok = false; break; }
        if (rank == 1 && !wait_bar(c, c.bar(B_QRFULL), ic & 1, false)) { ok = false; break; }
        tc_fence_after();
        const uint32_t g0 = gb;
        const int np = wi.page_end - wi.page_begin;
        // QK runs two pages ahead of PV, so the scores of page k+1 are ready
        // while the softmax warps still work on page k.
        for (int k = 0; k < np; ++k, ++gb) {
          const int s = gb & 1;
          const int stg = gb % kStages;
          if (!wait_fast(c, c.bar(B_TFULL0 + stg), (gb / kStages) & 1, false)) { ok = false; break; }
          if (gb >= 2 && !wait_fast(c, c.bar(B_SFREE0 + s), ((gb >> 1) - 1) & 1, false)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = t_s + stg * kStageBytes;
          const uint32_t d = tmem + kTmemS + 64 * s;
          // latent columns: A (query) from TMEM, 8 columns per 16-element k-step
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {
            const uint64_t bd = smem_desc(st + (ks >> 2) * kBoxT + (ks & 3) * 32, 16, 1024,
                                          kSwizzle128B);
            mma_f16_ts(d, tmem + kTmemQ + 8 * ks, bd, idesc_qk, ks > 0 ? 1u : 0u);
          }
          if (rank == 1) {
            // RoPE columns: A from shared memory
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = smem_desc(qr_s + ks * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(st + 4 * kBoxT + ks * 32, 16, 1024, kSwizzle128B);
              mma_f16_ss(d, ad, bd, idesc_qk, 1u);
            }
          }
          mma_commit(c.bar(B_SFULL0 + s));
          if (k == np - 1) mma_commit(c.bar(B_QEMPTY));
          if (k >= 2 && !pv(gb - 2, g0)) { ok = false; break; }
        }
        if (!ok) break;
        if (np >= 2 && !pv(gb - 2, g0)) { ok = false; break; }
        if (!pv(gb - 1, g0)) { ok = false; break; }
      }
      mma_commit(c.bar(B_FINAL));
      wait_bar(c, c.bar(B_FINAL), 0, false);
    }
  } else {
    // ------------------------------------------- softmax + epilogue warps ---
    const int h = threadIdx.x & 127;     // head = TMEM lane
    const int grp = threadIdx.x >> 7;    // column group
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t x_row_local = x_s + h * 128;
    const uint32_t x_row_remote = mapa_shared(x_s, peer) + h * 128;
    const uint32_t xfull_remote0 = mapa_shared(c.bar(B_XFULL0), peer);
    const uint32_t xempty_remote0 = mapa_shared(c.bar(B_XEMPTY0), peer);
    const uint32_t p_row = p_s + (h >> 3) * 1024 + (h & 7) * 128;
    const int swz = h & 7;
    float *pm = reinterpret_cast<float *>(smem + kOffPM);  // [page parity][group][row]
    float *pl = reinterpret_cast<float *>(smem + kOffPL);  // [group][row]
    const uint32_t s_col = kTmemS + 32 * grp;   // this group's score columns
    const uint32_t o_col = kTmemO + 128 * grp;  // this group's accumulator columns
    uint32_t gb = 0, ic_sm = 0;
    bool ok = true;
    // own partial scores (this group's 32 columns) of the page being
    // exchanged, rounded to bf16 pairs
    uint32_t own_cur[16], own_nxt[16];

    // Load this group's partial scores of page g from TMEM, round them to bf16
    // (the sum both CTAs form is then the same), send them to the peer.
    auto send = [&](uint32_t g, uint32_t (&own)[16]) -> bool {
      const int s = g & 1;
      if (!wait_bar_warp(c, c.bar(B_SFULL0 + s), (g >> 1) & 1, false)) return false;
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + s_col + 64 * s, r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(B_SFREE0 + s));
#pragma unroll
      for (int i = 0; i < 16; ++i)
        own[i] = pack_hi_pair(rne_bf16_hi(u2f(r[2 * i])), rne_bf16_hi(u2f(r[2 * i + 1])));
      if (g >= 2 && !wait_bar_warp(c, c.bar(B_XEMPTY0 + s), ((g >> 1) - 1) & 1, true)) return false;
      // asynchronous stores into the peer's buffer; their bytes complete the
      // peer's x_full barrier (armed by the peer for kXBytes)
      const uint32_t dst = x_row_remote + s * kXBytes;
      const uint32_t bar = xfull_remote0 + 8 * s;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_async_v4(dst + (((4 * grp + q) ^ swz) << 4), own[4 * q], own[4 * q + 1],
                    own[4 * q + 2], own[4 * q + 3], bar);
      return true;
    };

    for (int it = i0; it < i1 && ok; ++it) {
      const WorkItem wi = items[it];
      float m_ref = -INFINITY, l = 0.f;
      const uint32_t g0 = gb;
      {
        // stage this item's query slab in TMEM (A operand of QK): group g
        // writes slab elements [128g, 128g+128); the previous item's QKs are
        // complete (its epilogue waited for them)
        const long long qrow = ((long long)wi.b * a.q_len + wi.j) * a.n_h + h;
        const bool in = qrow < a.q_rows;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            a.q_full + (in ? qrow : 0) * MLA_ROW + col0 + 128 * grp);
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = in ? __ldg(src + ch * 8 + v) : make_uint4(0u, 0u, 0u, 0u);
            r[4 * v] = x.x;
            r[4 * v + 1] = x.y;
            r[4 * v + 2] = x.z;
            r[4 * v + 3] = x.w;
          }
          tmem_st32(tmem + lane_off + kTmemQ + 64 * grp + 32 * ch, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(B_QFULL));
      }
      // page ids, 32 at a time: lane i holds the id of page (chunk base + i);
      // the next chunk is fetched a whole chunk ahead
      const int32_t *row_pages = a.block_table + (size_t)wi.b * a.max_pages;
      auto fetch_ids = [&](int base_pg) -> int {
        const int p = base_pg + lane;
        return (p < wi.page_end && p < a.max_pages) ? row_pages[p] : -1;
      };
      int ids_cur = fetch_ids(wi.page_begin);
      int ids_nxt = fetch_ids(wi.page_begin + 32);
      if (!send(gb, own_cur)) { ok = false; break; }
      for (int pg = wi.page_begin; pg < wi.page_end; ++pg, ++gb) {
        const int s = gb & 1;
        const int rel = (pg - wi.page_begin) & 31;
        const int page = __shfl_sync(0xffffffffu, ids_cur, rel);
        if (rel == 31) {
          ids_cur = ids_nxt;
          ids_nxt = fetch_ids(pg + 33);
        }
        if (pg + 1 < wi.page_end) {
          // next page's scores go out before this page's softmax
          if (!send(gb + 1, own_nxt)) { ok = false; break; }
        }
        // this page's scores from the peer
        if (!wait_bar_warp(c, c.bar(B_XFULL0 + s), (gb >> 1) & 1, true)) { ok = false; break; }
        uint32_t peer[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = *reinterpret_cast<const uint4 *>(
              smem + (x_row_local + s * kXBytes - base) + (((4 * grp + q) ^ swz) << 4));
          peer[4 * q] = v.x;
          peer[4 * q + 1] = v.y;
          peer[4 * q + 2] = v.z;
          peer[4 * q + 3] = v.w;
        }
        __syncwarp();
        if (lane == 0) {
          // re-arm this buffer for page gb + 2 (the peer cannot send it before
          // all eight warps acknowledge page gb), then acknowledge page gb
          if (warp == 0) mbar_arrive_expect_tx(c.bar(B_XFULL0 + s), kXBytes);
          mbar_arrive_remote_relaxed(xempty_remote0 + 8 * s);
        }

        // scores of this group's 32 tokens, mask, partial max
        const bool valid = page >= 0 && page < a.num_pages;
        const int tok0 = pg * 64 + 32 * grp;
        const int nvis = valid ? min(32, max(0, wi.qpos - tok0 + 1)) : 0;  // visible prefix
        float sc[32];
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // both CTAs add the same two bf16-rounded partials: identical scores
          const float v0 = (u2f(own_cur[i] << 16) + u2f(peer[i] << 16)) * a.scale_log2;
          const float v1 = (u2f(own_cur[i] & 0xFFFF0000u) + u2f(peer[i] & 0xFFFF0000u)) * a.scale_log2;
          sc[2 * i] = 2 * i < nvis ? v0 : -INFINITY;
          sc[2 * i + 1] = 2 * i + 1 < nvis ? v1 : -INFINITY;
          mx4[i & 3] = fmaxf(mx4[i & 3], fmaxf(sc[2 * i], sc[2 * i + 1]));
        }
        // page max of the row = max over both groups
        float mblk = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        pm[(s * 2 + grp) * 128 + h] = mblk;
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(B_PMAX0 + s));
        if (!wait_bar_warp(c, c.bar(B_PMAX0 + s), (gb >> 1) & 1, false)) { ok = false; break; }
        mblk = fmaxf(mblk, pm[(s * 2 + (grp ^ 1)) * 128 + h]);
        float alpha = 1.f;
        bool resc = false;
        if (mblk > m_ref + kRescaleThreshold || (m_ref == -INFINITY && mblk > -INFINITY)) {
          if (m_ref > -INFINITY) {
            alpha = ex2_approx(m_ref - mblk);
            resc = true;
          }
          m_ref = mblk;
        }
        uint32_t pk[16];
        float ls4[4] = {0.f, 0.f, 0.f, 0.f};
        if (m_ref == -INFINITY) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t p0 = rne_bf16_hi(ex2_approx(sc[2 * i] - m_ref));
            const uint32_t p1 = rne_bf16_hi(ex2_approx(sc[2 * i + 1] - m_ref));
            pk[i] = pack_hi_pair(p0, p1);
            ls4[i & 3] += u2f(p0) + u2f(p1);  // the sum of the weights P*V uses
          }
        }
        l = l * alpha + ((ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));
#pragma unroll
        for (int i = 0; i < 16; ++i) own_cur[i] = own_nxt[i];

        // the previous page's P*V has finished: P buffer free, O stable
        if (gb > g0) {
          if (!wait_bar_warp(c, c.bar(B_PFREE), (gb - 1) & 1, false)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t r[32];
              tmem_ld32(tmem + lane_off + o_col + 32 * ch, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = f2u(u2f(r[e]) * alpha);
              tmem_st32(tmem + lane_off + o_col + 32 * ch, r);
            }
            tmem_wait_st();
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(smem + (p_row - base) + (((4 * grp + q) ^ swz) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(B_PFULL));
      }
      if (!ok) break;

      // epilogue: wait for the last P*V, combine the two groups' row sums,
      // then write o (or a partial result)
      if (!wait_bar_warp(c, c.bar(B_PFREE), (gb - 1) & 1, false)) { ok = false; break; }
      tc_fence_after();
      // (the partner group has read its last page maxes: it arrived p_full)
      pl[grp * 128 + h] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(B_EPI));
      if (!wait_bar_warp(c, c.bar(B_EPI), ic_sm & 1, false)) { ok = false; break; }
      ++ic_sm;
      const float lt = l + pl[(grp ^ 1) * 128 + h];
      const bool write = h < a.n_h;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const size_t row = ((size_t)wi.b * a.q_len + wi.j) * a.n_h + h;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + o_col + 32 * ch, r);
        tmem_wait_ld();
        if (!write) continue;
        const int d0 = col0 + 128 * grp + 32 * ch;
        if (wi.slot < 0) {
          uint4 *dst = reinterpret_cast<uint4 *>(a.o_latent + row * MLA_D_C + d0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(u2f(r[8 * q]) * inv, u2f(r[8 * q + 1]) * inv),
                                pack_bf16x2(u2f(r[8 * q + 2]) * inv, u2f(r[8 * q + 3]) * inv),
                                pack_bf16x2(u2f(r[8 * q + 4]) * inv, u2f(r[8 * q + 5]) * inv),
                                pack_bf16x2(u2f(r[8 * q + 6]) * inv, u2f(r[8 * q + 7]) * inv));
        } else {
          float4 *dst = reinterpret_cast<float4 *>(
              a.ws_o + ((size_t)wi.slot * a.n_h + h) * MLA_D_C + d0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(u2f(r[4 * q]) * inv, u2f(r[4 * q + 1]) * inv,
                                 u2f(r[4 * q + 2]) * inv, u2f(r[4 * q + 3]) * inv);
        }
      }
      tc_fence_before();
      // the next item writes the row-max/sum slots only after its first
      // page's scores exist, i.e. after every warp has staged its query
      // rows, i.e. after both groups left this epilogue
      if (write && rank == 0 && grp == 0) {
        const float lse = lt > 0.f ? (m_ref + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        if (wi.slot < 0) {
          if (a.lse != nullptr) a.lse[row] = lse;
        } else {
          a.ws_lse[(size_t)wi.slot * a.n_h + h] = lse;
        }
      }
    }
  }

  __syncthreads();
  __syncwarp();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  __syncwarp();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
}

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

// Row-major bf16 matrix [rows][576] viewed as 64-column x box_rows tiles with
// the 128-byte swizzle.
mla_status_t make_row_map(CUtensorMap *tm, const void *base, uint64_t rows, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)MLA_ROW, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)MLA_ROW * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

}  // namespace

mla_status_t launch_decode_tc(const DecodeArgs &a, cudaStream_t stream) {
  const PlanHeader *ph = a.plan_host;
  if (ph->num_items == 0 || ph->num_ctas == 0) return MLA_OK;
  CUtensorMap tm_cache, tm_q;
  mla_status_t st = make_row_map(&tm_cache, a.cache, (uint64_t)a.num_pages * MLA_PAGE, 64);
  if (st != MLA_OK) return st;
  st = make_row_map(&tm_q, a.q_full, (uint64_t)a.batch * a.q_len * a.n_h, 128);
  if (st != MLA_OK) return st;
  TcArgs t;
  t.plan = a.plan_dev;
  t.q_full = a.q_full;
  t.q_rows = (long long)a.batch * a.q_len * a.n_h;
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
  MLA_CUDA_TRY(cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemBytes));
  decode_tc_kernel<<<2 * ph->num_ctas, kThreads, kSmemBytes, stream>>>(tm_cache, tm_q, t);
  MLA_LAUNCH_CHECK("decode_tc_kernel");
  return MLA_OK;
}

}  // namespace mla

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
// Warp roles (192 threads): warps 0-3 softmax + epilogue (thread = head = TMEM
// lane), warp 4 TMA producer, warp 5 MMA issuer (and TMEM owner).
// Pipeline per page g: TMA(g) -> QK(g) -> [exchange, softmax](g) -> PV(g), with
// QK(g+1) issued before PV(g) and two smem stages / two TMEM score buffers.
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

constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kMaxBoxes = 5;                          // 64-column boxes per slab (CTA 1)
constexpr uint32_t kBoxQ = 128 * 128;                 // 128 query rows x 64 bf16
constexpr uint32_t kBoxT = 64 * 128;                  // 64 tokens x 64 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffT = kOffQ + kMaxBoxes * kBoxQ;   // 81920
constexpr uint32_t kStageBytes = kMaxBoxes * kBoxT;     // 40960
constexpr uint32_t kOffP = kOffT + 2 * kStageBytes;     // 163840
constexpr uint32_t kOffX = kOffP + 128 * 128;           // 180224: P is 128 x 64 bf16
constexpr uint32_t kOffBar = kOffX + 128 * 256;         // 212992: exchange is 128 x 64 fp32
constexpr uint32_t kSmemUsed = kOffBar + 256;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;      // slack for 1024-byte alignment

// barrier slots (8 bytes each) in the barrier area
enum {
  B_TFULL0, B_TFULL1, B_TEMPTY0, B_TEMPTY1, B_QFULL, B_QEMPTY, B_SFULL0, B_SFULL1,
  B_SFREE0, B_SFREE1, B_PFULL, B_PFREE, B_XFULL, B_XEMPTY, B_FINAL, B_COUNT
};
constexpr uint32_t kOffTmemPtr = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemPtr + 4;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;      // columns [0, 256): latent accumulator
constexpr uint32_t kTmemS = 256;    // columns [256, 384): two 64-column score buffers
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct TcArgs {
  const unsigned char *plan;
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

// Same, for a whole warp: every lane polls, the warp proceeds only if all did.
__device__ __forceinline__ bool wait_bar_warp(const Ctx &c, uint32_t bar, uint32_t parity,
                                              bool cluster) {
  const bool ok = wait_bar(c, bar, parity, cluster);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_cache,
                 const __grid_constant__ CUtensorMap tm_q, const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (base - raw);

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
    mbar_init(c.bar(B_TFULL0), 1);
    mbar_init(c.bar(B_TFULL1), 1);
    mbar_init(c.bar(B_TEMPTY0), 1);
    mbar_init(c.bar(B_TEMPTY1), 1);
    mbar_init(c.bar(B_QFULL), 1);
    mbar_init(c.bar(B_QEMPTY), 1);
    mbar_init(c.bar(B_SFULL0), 1);
    mbar_init(c.bar(B_SFULL1), 1);
    mbar_init(c.bar(B_SFREE0), 4);
    mbar_init(c.bar(B_SFREE1), 4);
    mbar_init(c.bar(B_PFULL), 4);
    mbar_init(c.bar(B_PFREE), 1);
    mbar_init(c.bar(B_XFULL), 4);    // the peer's four softmax warps
    mbar_init(c.bar(B_XEMPTY), 4);
    mbar_init(c.bar(B_FINAL), 1);
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

  const uint32_t q_s = base + kOffQ, t_s = base + kOffT, p_s = base + kOffP, x_s = base + kOffX;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(&tm_q);
      uint32_t gb = 0, ic = 0, q_armed = 0, armed[2] = {0, 0};
      bool ok = true;
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        if (ic > 0 && !wait_bar(c, c.bar(B_QEMPTY), (ic - 1) & 1, false)) { ok = false; break; }
        mbar_arrive_expect_tx(c.bar(B_QFULL), nbox * kBoxQ);
        ++q_armed;
        const int qrow = (wi.b * a.q_len + wi.j) * a.n_h;
        for (int x = 0; x < nbox; ++x)
          tma_load_2d(q_s + x * kBoxQ, &tm_q, col0 + 64 * x, qrow, c.bar(B_QFULL));
        for (int pg = wi.page_begin; pg < wi.page_end; ++pg, ++gb) {
          const int s = gb & 1;
          if (gb >= 2 && !wait_bar(c, c.bar(B_TEMPTY0 + s), ((gb >> 1) - 1) & 1, false)) {
            ok = false;
            break;
          }
          int page = pg < a.max_pages ? a.block_table[(size_t)wi.b * a.max_pages + pg] : -1;
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
      for (int s = 0; s < 2; ++s)
        if (armed[s]) wait_bar(c, c.bar(B_TFULL0 + s), (armed[s] - 1) & 1, false);
      if (q_armed) wait_bar(c, c.bar(B_QFULL), (q_armed - 1) & 1, false);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
      const int nks = nbox * 4;
      uint32_t gb = 0, ic = 0;
      bool ok = true;
      auto pv = [&](uint32_t g, uint32_t g0) -> bool {
        if (!wait_bar(c, c.bar(B_PFULL), g & 1, false)) return false;
        tc_fence_after();
        const uint32_t st = t_s + (g & 1) * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = smem_desc(p_s + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(st + kk * 2048, 8192, 1024, kSwizzle128B);
          mma_f16_ss(tmem + kTmemO, ad, bd, idesc_pv, (g != g0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(c.bar(B_TEMPTY0 + (g & 1)));
        mma_commit(c.bar(B_PFREE));
        return true;
      };
      for (int it = i0; it < i1 && ok; ++it, ++ic) {
        const WorkItem wi = items[it];
        if (!wait_bar(c, c.bar(B_QFULL), ic & 1, false)) { ok = false; break; }
        tc_fence_after();
        const uint32_t g0 = gb;
        const int np = wi.page_end - wi.page_begin;
        for (int k = 0; k < np; ++k, ++gb) {
          const int s = gb & 1;
          if (!wait_bar(c, c.bar(B_TFULL0 + s), (gb >> 1) & 1, false)) { ok = false; break; }
          if (gb >= 2 && !wait_bar(c, c.bar(B_SFREE0 + s), ((gb >> 1) - 1) & 1, false)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = t_s + s * kStageBytes;
          for (int ks = 0; ks < nks; ++ks) {
            const int x = ks >> 2, kk = ks & 3;
            const uint64_t ad = smem_desc(q_s + x * kBoxQ + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(st + x * kBoxT + kk * 32, 16, 1024, kSwizzle128B);
            mma_f16_ss(tmem + kTmemS + 64 * s, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
          }
          mma_commit(c.bar(B_SFULL0 + s));
          if (k == np - 1) mma_commit(c.bar(B_QEMPTY));
          if (k > 0 && !pv(gb - 1, g0)) { ok = false; break; }
        }
        if (!ok) break;
        if (!pv(gb - 1, g0)) { ok = false; break; }
      }
      mma_commit(c.bar(B_FINAL));
      wait_bar(c, c.bar(B_FINAL), 0, false);
    }
  } else {
    // ------------------------------------------- softmax + epilogue warps ---
    const int h = threadIdx.x;  // head = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t x_row_local = x_s + h * 256;
    const uint32_t x_row_remote = mapa_shared(x_s, peer) + h * 256;
    const uint32_t xfull_remote = mapa_shared(c.bar(B_XFULL), peer);
    const uint32_t xempty_remote = mapa_shared(c.bar(B_XEMPTY), peer);
    const uint32_t p_row = p_s + (h >> 3) * 1024 + (h & 7) * 128;
    const int swz = h & 7;
    uint32_t gb = 0;
    bool ok = true;
    for (int it = i0; it < i1 && ok; ++it) {
      const WorkItem wi = items[it];
      float m_ref = -INFINITY, l = 0.f;
      const uint32_t g0 = gb;
      for (int pg = wi.page_begin; pg < wi.page_end; ++pg, ++gb) {
        const int s = gb & 1;
        if (!wait_bar_warp(c, c.bar(B_SFULL0 + s), (gb >> 1) & 1, false)) { ok = false; break; }
        tc_fence_after();
        uint32_t own[64];
        {
          uint32_t (&o0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&own[0]);
          uint32_t (&o1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&own[32]);
          tmem_ld32(tmem + lane_off + kTmemS + 64 * s, o0);
          tmem_ld32(tmem + lane_off + kTmemS + 64 * s + 32, o1);
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(B_SFREE0 + s));

        // exchange partial scores with the peer CTA
        if (gb > 0 && !wait_bar_warp(c, c.bar(B_XEMPTY), (gb - 1) & 1, true)) { ok = false; break; }
#pragma unroll
        for (int q = 0; q < 16; ++q)
          st_cluster_v4(x_row_remote + ((q ^ swz) << 4), u2f(own[4 * q]), u2f(own[4 * q + 1]),
                        u2f(own[4 * q + 2]), u2f(own[4 * q + 3]));
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(xfull_remote);
        if (!wait_bar_warp(c, c.bar(B_XFULL), gb & 1, true)) { ok = false; break; }
        float sc[64];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 v = *reinterpret_cast<const float4 *>(
              smem + (x_row_local - base) + ((q ^ swz) << 4));
          sc[4 * q] = u2f(own[4 * q]) + v.x;
          sc[4 * q + 1] = u2f(own[4 * q + 1]) + v.y;
          sc[4 * q + 2] = u2f(own[4 * q + 2]) + v.z;
          sc[4 * q + 3] = u2f(own[4 * q + 3]) + v.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(xempty_remote);

        // mask, running max, probabilities
        int page = pg < a.max_pages ? a.block_table[(size_t)wi.b * a.max_pages + pg] : -1;
        const bool valid = page >= 0 && page < a.num_pages;
        const int tok0 = pg * 64;
        float mblk = -INFINITY;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const bool vis = valid && (tok0 + i <= wi.qpos);
          sc[i] = vis ? sc[i] * a.scale_log2 : -INFINITY;
          mblk = fmaxf(mblk, sc[i]);
        }
        float alpha = 1.f;
        bool resc = false;
        if (mblk > m_ref + kRescaleThreshold || (m_ref == -INFINITY && mblk > -INFINITY)) {
          if (m_ref > -INFINITY) {
            alpha = exp2f(m_ref - mblk);
            resc = true;
          }
          m_ref = mblk;
        }
        uint32_t pk[32];
        float lsum = 0.f;
        if (m_ref == -INFINITY) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t b2 = pack_bf16x2(exp2f(sc[2 * i] - m_ref), exp2f(sc[2 * i + 1] - m_ref));
            pk[i] = b2;
            lsum += bf16_bits_to_f32(b2 & 0xFFFFu) + bf16_bits_to_f32(b2 >> 16);
          }
        }
        l = l * alpha + lsum;

        // the previous page's P*V has finished: P buffer free, O stable
        if (gb > g0) {
          if (!wait_bar_warp(c, c.bar(B_PFREE), (gb - 1) & 1, false)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
            for (int ch = 0; ch < 8; ++ch) {
              uint32_t r[32];
              tmem_ld32(tmem + lane_off + kTmemO + 32 * ch, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = f2u(u2f(r[e]) * alpha);
              tmem_st32(tmem + lane_off + kTmemO + 32 * ch, r);
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
        if (lane == 0) mbar_arrive(c.bar(B_PFULL));
      }
      if (!ok) break;

      // epilogue: wait for the last P*V, then write o (or a partial result)
      if (!wait_bar_warp(c, c.bar(B_PFREE), (gb - 1) & 1, false)) { ok = false; break; }
      tc_fence_after();
      const bool write = h < a.n_h;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t row = ((size_t)wi.b * a.q_len + wi.j) * a.n_h + h;
#pragma unroll 1
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + kTmemO + 32 * ch, r);
        tmem_wait_ld();
        if (!write) continue;
        const int d0 = col0 + 32 * ch;
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
      if (write && rank == 0) {
        const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
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

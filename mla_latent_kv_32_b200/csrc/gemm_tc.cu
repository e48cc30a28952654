// Batched bf16 GEMM on the sm_100a tensor cores (tcgen05, TMA, TMEM), fp32
// accumulation, for the absorbed-MLA contractions around the attention:
//   W^UK folded into the query:   q~[t][h][c] = sum_d q^C[t][h][d] W^UK[h][d][c]
//   W^UV applied to the output:   u[t][h][d]  = sum_c o[t][h][c]  W^UV[h][d][c]
//   and the decode layer's projections (W^DQ, [W^UQ|W^QR], [W^DKV|W^KR], W^O)
// ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide", "The Matrix
// Absorption Trick" parts 2-3, "Core Architecture & Mathematics" 1-2).
//
// Every use has few tokens and a large weight, so the weight is the M side
// (tiles of 128 rows, the tensor core's native height) and the tokens are the
// N side (16..256 per tile):
//   C[z][m][n] = sum_k A[z][m][k] * B[z][n][k]
// A (the weight) is K-major or MN-major in global memory, B (the activations)
// is K-major; both arrive through 3-D TMA tensor maps (z = head or split) in
// 64-element k-chunks with the 128-byte swizzle. One CTA computes one
// 128 x BN tile: warp 0 lane 0 issues TMA into a ring of up to 4 stages, warp
// 1 lane 0 issues the MMAs into a TMEM accumulator of BN columns (shared memory
// and TMEM are sized to the tile, so several CTAs share an SM when the tiles
// are small), all four warps then read it back
// (thread = row m) and write C through arbitrary strides, as bf16 or fp32
// (fp32 outputs may be split over K and reduced with atomic adds).
//
// A launch may carry a side job in extra CTAs that run alongside the tiles:
// the q^R RoPE/pack of mla_absorb_q (q_full[t][h][512:576] = RoPE(q^R[t][h],
// pos[t]), interleaved pairs, fp32 table, no fused multiply-add, RNE to bf16;
// "Deconstructing DeepSeek V4 Pro", rotational embedding), which writes
// columns the GEMM tiles do not touch.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "append.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kMaxStages = 8;          // ring depth when one CTA per SM covers the grid
constexpr int kSharedStages = 4;       // ring depth when CTAs share SMs
constexpr uint32_t kSmemLimit = 232448;  // dynamic shared memory per CTA (227 KB)
constexpr uint32_t kAStage = 128 * 128;        // 128 rows x 64 k (bf16) = 16 KB
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr int kMaxPartSplits = 8;      // fp32 split-K into partial-sum tiles: at most this many

struct GemmTcArgs {
  int M, N, K;          // per batch
  int BN;               // tile width in n (multiple of 16, <= 256)
  int stages;           // ring depth (1..kMaxStages)
  uint32_t stage_bytes; // A chunk + B chunk, rounded to 1 KB
  uint32_t tmem_cols;   // accumulator columns allocated (power of two >= BN, >= 32)
  int k_chunks;         // 64-element k-chunks per split
  int splits;           // split-K factor (fp32 output only)
  int batch;
  int a_mn;             // A is MN-major (m contiguous)
  void *C;
  long long sCz, sCm, sCn;
  int c_fp32;
  float *ws;            // bf16 output split over K: fp32 sums at ((z*N + n)*M + m)
  uint32_t *status;
  int tile_z;           // z extent of the GEMM tiles; CTAs beyond it run the side job
  int b_shared;         // every batch z reads the same B (its tensor map has one z slice)
  float *part;          // fp32 output split over K: split s writes its partial tile at
                        // ((s * batch + z) * N + n) * M + m; a second kernel sums them
  // side job (rope_q_pe == nullptr: none)
  const uint16_t *rope_q_pe;
  int rope_ld_qp;
  const int32_t *rope_pos;
  const float *rope_table;
  int rope_max_pos, rope_T, rope_n_h;
  uint16_t *rope_q_full;
  AppendJob app;        // second side job (n_tokens == 0: none)
};

// Side job: each thread rotates the 4 pairs of one 16-byte chunk of q^R
// (8 chunks per token-head), kSideBatch chunks per pass at a stride of all
// side threads. A pass issues every load of its chunks (values, positions)
// before the table loads that depend on them, so a thread waits two memory
// round trips per pass, not two per chunk.
constexpr int kSideBatch = 4;

__device__ void rope_side_job(const GemmTcArgs &g, int cta, int ctas) {
  const long long chunks = (long long)g.rope_T * g.rope_n_h * 8;
  const long long stride = (long long)ctas * blockDim.x;
  for (long long c0 = (long long)cta * blockDim.x + threadIdx.x; c0 < chunks;
       c0 += kSideBatch * stride) {
    uint4 kv[kSideBatch];
    int p[kSideBatch];
#pragma unroll
    for (int u = 0; u < kSideBatch; ++u) {
      const long long c = c0 + u * stride;
      p[u] = -1;
      if (c >= chunks) continue;
      const long long th = c >> 3;
      const int t = (int)(th / g.rope_n_h), h = (int)(th % g.rope_n_h);
      kv[u] = __ldg(reinterpret_cast<const uint4 *>(g.rope_q_pe + (size_t)t * g.rope_ld_qp +
                                                    h * MLA_D_R) + (c & 7));
      if (g.rope_pos != nullptr) p[u] = __ldg(g.rope_pos + t);
    }
    float4 cs0[kSideBatch], cs1[kSideBatch];
#pragma unroll
    for (int u = 0; u < kSideBatch; ++u) {
      const long long c = c0 + u * stride;
      if (c >= chunks || g.rope_pos == nullptr || p[u] < 0 || p[u] >= g.rope_max_pos) continue;
      const float *row = g.rope_table + (size_t)p[u] * 64 + (c & 7) * 8;
      cs0[u] = __ldg(reinterpret_cast<const float4 *>(row));
      cs1[u] = __ldg(reinterpret_cast<const float4 *>(row + 4));
    }
#pragma unroll
    for (int u = 0; u < kSideBatch; ++u) {
      const long long c = c0 + u * stride;
      if (c >= chunks) continue;
      const long long th = c >> 3;
      const int t = (int)(th / g.rope_n_h), h = (int)(th % g.rope_n_h);
      uint4 *dst = reinterpret_cast<uint4 *>(g.rope_q_full + ((size_t)t * g.rope_n_h + h) *
                                                                 MLA_ROW + MLA_D_C) + (c & 7);
      if (g.rope_pos == nullptr) {
        *dst = kv[u];
        continue;
      }
      if (p[u] < 0 || p[u] >= g.rope_max_pos) {
        if ((c & 7) == 0) report(g.status, MLA_DEV_BAD_POSITION);
        *dst = make_uint4(0, 0, 0, 0);
        continue;
      }
      const uint32_t wv[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      const float cosv[4] = {cs0[u].x, cs0[u].z, cs1[u].x, cs1[u].z};
      const float sinv[4] = {cs0[u].y, cs0[u].w, cs1[u].y, cs1[u].w};
      uint32_t out[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float y0, y1;
        rope_pair_rn(bf16_bits_to_f32(wv[i] & 0xFFFFu), bf16_bits_to_f32(wv[i] >> 16), cosv[i],
                     sinv[i], y0, y1);
        out[i] = pack_bf16x2(y0, y1);
      }
      *dst = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

__device__ __noinline__ bool wait_bar_g(uint32_t bar, uint32_t parity, uint32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0 && globaltimer_ns() - t0 > kTimeoutNs) {
      report(status, MLA_DEV_TIMEOUT);
      return false;
    }
  }
}

// kTwoM: a CTA covers 256 rows of A with two 128-row accumulators (the
// instances keep the one-accumulator loops free of the second's branches).
template <bool kTwoM>
__global__ void __launch_bounds__(128, 4)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const GemmTcArgs g) {
  if ((int)blockIdx.z >= g.tile_z) {
    // side-job CTAs: no shared memory, barriers or tensor memory
    const int per_z = gridDim.x * gridDim.y;
    const int cta = ((int)blockIdx.z - g.tile_z) * per_z + blockIdx.y * gridDim.x + blockIdx.x;
    const int ctas = ((int)gridDim.z - g.tile_z) * per_z;
    if (g.rope_q_pe != nullptr) rope_side_job(g, cta, ctas);
    // the step's cache append: one warp per token
    const int warps = ctas * (blockDim.x >> 5);
    for (int t = cta * (blockDim.x >> 5) + (threadIdx.x >> 5); t < g.app.n_tokens; t += warps) {
      if (g.app.cache8 != nullptr)
        append_token_fp8_warp(g.app.cache8, g.app.scales8, g.app.num_pages, g.app.block_table,
                              g.app.batch, g.app.max_pages, g.app.seq_idx, g.app.pos, g.app.c_kv,
                              g.app.ld_c, g.app.k_pe, g.app.ld_k, g.rope_table, g.rope_max_pos, t,
                              threadIdx.x & 31, g.status);
      else
        append_token_warp(g.app.cache, g.app.num_pages, g.app.block_table, g.app.batch,
                          g.app.max_pages, g.app.seq_idx, g.app.pos, g.app.c_kv, g.app.ld_c,
                          g.app.k_pe, g.app.ld_k, g.rope_table, g.rope_max_pos, t,
                          threadIdx.x & 31, g.status);
    }
    return;
  }
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * g.BN;
  const int m0 = blockIdx.y * (kTwoM ? 256 : 128);
  constexpr uint32_t a_bytes = kTwoM ? 2 * kAStage : kAStage;
  const int z = blockIdx.z / g.splits;
  const int split = blockIdx.z % g.splits;
  const int kc0 = split * g.k_chunks;
  const int kc1 = min(kc0 + g.k_chunks, (g.K + 63) / 64);
  const int stages = g.stages;
  const uint32_t bar_full = base + stages * g.stage_bytes, bar_empty = bar_full + 8 * kMaxStages;
  const uint32_t bar_done = bar_empty + 8 * kMaxStages, tptr = bar_done + 8;
  const uint32_t b_bytes = (uint32_t)g.BN * 128;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_done, 1);
    fence_mbar_init_cluster();
  }
  if (warp == 1) tmem_alloc(tptr, g.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + (tptr - base));

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    int armed[kMaxStages] = {};
    for (int kc = kc0, i = 0; kc < kc1; ++kc, ++i) {
      const int s = i % stages;
      if (i >= stages && !wait_bar_g(bar_empty + 8 * s, ((i / stages) - 1) & 1, g.status))
        break;
      const uint32_t a_s = base + s * g.stage_bytes, b_s = a_s + a_bytes;
      mbar_arrive_expect_tx(bar_full + 8 * s, a_bytes + b_bytes);
      ++armed[s];
      if (g.a_mn) {
        // two 64-row (m) boxes of 64 k-rows each
        tma_load_3d(a_s, &tm_a, m0, kc * 64, z, bar_full + 8 * s);
        tma_load_3d(a_s + 8192, &tm_a, m0 + 64, kc * 64, z, bar_full + 8 * s);
      } else {
        tma_load_3d(a_s, &tm_a, kc * 64, m0, z, bar_full + 8 * s);
        if (kTwoM) tma_load_3d(a_s + kAStage, &tm_a, kc * 64, m0 + 128, z, bar_full + 8 * s);
      }
      tma_load_3d(b_s, &tm_b, kc * 64, n0, g.b_shared ? 0 : z, bar_full + 8 * s);
    }
    for (int s = 0; s < stages; ++s)
      if (armed[s]) wait_bar_g(bar_full + 8 * s, (armed[s] - 1) & 1, g.status);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(128, g.BN, g.a_mn, 0);
    for (int kc = kc0, i = 0; kc < kc1; ++kc, ++i) {
      const int s = i % stages;
      if (!wait_bar_g(bar_full + 8 * s, (i / stages) & 1, g.status)) break;
      tc_fence_after();
      const uint32_t a_s = base + s * g.stage_bytes, b_s = a_s + a_bytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = g.a_mn ? smem_desc(a_s + kk * 2048, 8192, 1024, kSwizzle128B)
                                   : smem_desc(a_s + kk * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd = smem_desc(b_s + kk * 32, 16, 1024, kSwizzle128B);
        mma_f16_ss(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        if (kTwoM)
          mma_f16_ss(tmem + g.BN, smem_desc(a_s + kAStage + kk * 32, 16, 1024, kSwizzle128B), bd,
                     idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar_empty + 8 * s);
    }
    mma_commit(bar_done);
  }
  __syncwarp();
  // epilogue: thread = row m of the tile
  const bool done = wait_bar_g(bar_done, 0, g.status);
  tc_fence_after();
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
#pragma unroll
  for (int pass = 0; pass < (kTwoM ? 2 : 1); ++pass)
  for (int ch = 0; ch * 32 < g.BN; ++ch) {
    const int m = m0 + 128 * pass + threadIdx.x;
    uint32_t r[32];
    tmem_ld32(tmem + lane_off + pass * g.BN + 32 * ch, r);
    tmem_wait_ld();
    if (!done || kc1 <= kc0 || m >= g.M) continue;
    if (g.part != nullptr) {
      // this split's partial tile
      float *dst = g.part + ((long long)split * g.batch + z) * g.N * g.M + m;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int n = n0 + 32 * ch + e;
        if (n >= g.N) break;
        dst[(long long)n * g.M] = __uint_as_float(r[e]);
      }
      continue;
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int n = n0 + 32 * ch + e;
      if (n >= g.N) break;
      const float v = __uint_as_float(r[e]);
      if (g.ws != nullptr) {
        atomicAdd(g.ws + ((long long)z * g.N + n) * g.M + m, v);
        continue;
      }
      const long long off = (long long)z * g.sCz + (long long)m * g.sCm + (long long)n * g.sCn;
      if (g.c_fp32) {
        if (g.splits > 1)
          atomicAdd(reinterpret_cast<float *>(g.C) + off, v);
        else
          reinterpret_cast<float *>(g.C)[off] = v;
      } else {
        reinterpret_cast<uint16_t *>(g.C)[off] = (uint16_t)f32_to_bf16_bits(v);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, g.tmem_cols);
  }
}

// C[z][m][n] (bf16, strided) = the fp32 split-K sums ws[(z*N + n)*M + m].
__global__ void __launch_bounds__(256)
split_to_bf16_kernel(const float *__restrict__ ws, int M, int N, int batch, uint16_t *C,
                     long long sCz, long long sCm, long long sCn) {
  const long long total = (long long)M * N * batch;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i % M);
    const long long zn = i / M;
    const int n = (int)(zn % N), z = (int)(zn / N);
    C[(long long)z * sCz + (long long)m * sCm + (long long)n * sCn] =
        (uint16_t)f32_to_bf16_bits(ws[i]);
  }
}

// C[z][m][n] (float32, strided) = the sum over the splits of
// part[((s * batch + z) * N + n) * M + m].
__global__ void __launch_bounds__(256)
part_reduce_kernel(const float *__restrict__ part, int splits, int M, int N, int batch, float *C,
                   long long sCz, long long sCm, long long sCn) {
  const long long total = (long long)M * N * batch;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int sp = 0; sp < splits; ++sp) acc += __ldg(part + sp * total + i);
    const int m = (int)(i % M);
    const long long zn = i / M;
    const int n = (int)(zn % N), z = (int)(zn / N);
    C[(long long)z * sCz + (long long)m * sCm + (long long)n * sCn] = acc;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 tensor: dim0 contiguous (d0 elements), dim1 stride s1 elements,
// dim2 stride s2 elements; box {64, box1, 1} with the 128-byte swizzle.
mla_status_t make_map3(CUtensorMap *tm, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t s1, uint64_t s2, uint32_t box1) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (((s1 * 2) & 15) || ((s2 * 2) & 15))
    return fail(MLA_ERR_INVALID_ARGUMENT, "GEMM operand strides must be multiples of 16 bytes");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1 * 2, s2 * 2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

}  // namespace

GemmPlan plan_gemm(int M, int N, int K, int batch, bool a_mn, bool c_fp32, bool fp32_part,
                   bool atomic_split, int sms) {
  GemmPlan pl;
  pl.BN = N >= 256 ? 256 : ((N + 15) / 16) * 16;
  pl.ntile = (N + pl.BN - 1) / pl.BN;
  const int kchunks = (K + 63) / 64;
  const bool big_m = !a_mn && M >= 1024;
  pl.splits = 1;
  pl.part = false;
  if (c_fp32 && fp32_part) {
    // fp32 output with a workspace: 256-row tiles (two accumulators, so each
    // CTA reads the B tile for twice the rows), split over K into partial-sum
    // tiles until the grid fills one wave (at most kMaxPartSplits; W^O at 256
    // tokens: 113.7 -> 95 us)
    pl.two_m = big_m;
    pl.mtile = (M + (pl.two_m ? 255 : 127)) / (pl.two_m ? 256 : 128);
    const long long tiles = (long long)pl.ntile * pl.mtile * batch;
    if (tiles < sms) {
      const int s0 = (int)std::min<long long>(std::min<long long>(sms / tiles, kMaxPartSplits),
                                              kchunks / 2);
      if (s0 >= 2) {
        const int per = (kchunks + s0 - 1) / s0;
        pl.splits = (kchunks + per - 1) / per;   // no empty split
        pl.part = pl.splits > 1;
      }
    }
  } else {
    // otherwise a small tile grid splits over K with atomic adds on 128-row
    // tiles (the fp32 output, or a bf16 output's fp32 workspace); a grid that
    // does not split takes 256-row tiles
    const long long tiles1 = (long long)pl.ntile * ((M + 127) / 128) * batch;
    if (atomic_split)
      while (pl.splits < 32 && tiles1 * pl.splits * 2 <= 296 && kchunks / (pl.splits * 2) >= 4)
        pl.splits *= 2;
    pl.two_m = big_m && pl.splits == 1;
    pl.mtile = (M + (pl.two_m ? 255 : 127)) / (pl.two_m ? 256 : 128);
  }
  pl.k_chunks = (kchunks + pl.splits - 1) / pl.splits;
  pl.part_bytes =
      pl.part ? ((size_t)pl.splits * M * N * batch * sizeof(float) + 255) & ~(size_t)255 : 0;
  return pl;
}

mla_status_t launch_gemm_tc(const GemmTcDesc &d, cudaStream_t stream) {
  if (d.M == 0 || d.N == 0 || d.batch == 0) return MLA_OK;
  if (d.K <= 0 || d.K % 16 != 0) return fail(MLA_ERR_UNSUPPORTED, "GEMM K must be a multiple of 16");
  CUtensorMap tm_a, tm_b;
  const int BN = d.N >= 256 ? 256 : ((d.N + 15) / 16) * 16;
  mla_status_t st;
  if (d.a_mn)  // A element (z, m, k) at A + z*sAz + k*sAk + m (m contiguous)
    st = make_map3(&tm_a, d.A, d.M, d.K, d.batch, d.sAk, d.sAz, 64);
  else         // A element (z, m, k) at A + z*sAz + m*sAm + k
    st = make_map3(&tm_a, d.A, d.K, d.M, d.batch, d.sAm, d.sAz, 128);
  if (st != MLA_OK) return st;
  const bool b_shared = d.sBz == 0;
  st = make_map3(&tm_b, d.B, d.K, d.N, b_shared ? 1 : d.batch, d.sBn,
                 b_shared ? (uint64_t)d.sBn * d.N : d.sBz, BN);
  if (st != MLA_OK) return st;
  GemmTcArgs g;
  g.M = d.M;
  g.N = d.N;
  g.K = d.K;
  g.BN = BN;
  int sms = 0;
  st = device_info(&sms, nullptr, nullptr);
  if (st != MLA_OK) return st;
  const GemmPlan pl = plan_gemm(d.M, d.N, d.K, d.batch, d.a_mn, d.c_fp32 != 0,
                                d.c_fp32 && d.part_ws != nullptr,
                                (d.c_fp32 && d.allow_split) || (!d.c_fp32 && d.split_ws != nullptr),
                                sms);
  if (pl.part && d.part_ws_bytes < pl.part_bytes)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "GEMM workspace %zu B < %zu B", d.part_ws_bytes,
                pl.part_bytes);
  const int kchunks = (d.K + 63) / 64;
  const bool two_m = pl.two_m;
  const int ntile = pl.ntile, mtile = pl.mtile;
  const int splits = pl.splits;
  const bool ws_split = splits > 1 && !d.c_fp32;
  g.part = pl.part ? d.part_ws : nullptr;
  g.splits = splits;
  g.k_chunks = (kchunks + splits - 1) / splits;
  g.stage_bytes = (two_m ? 2 : 1) * kAStage + (((uint32_t)BN * 128 + 1023u) & ~1023u);
  // A grid that fits one CTA per SM keeps every k-chunk of a tile in flight
  // (up to kMaxStages, within the shared memory), so a tile waits one load
  // round trip rather than one per ring cycle; denser grids keep a shallower
  // ring and several CTAs per SM.
  const uint32_t bar_bytes = 8 * (2 * kMaxStages + 2);
  const int fit = (int)((kSmemLimit - 1024 - bar_bytes) / g.stage_bytes);
  const long long tile_ctas = (long long)ntile * mtile * d.batch * splits;
  const int depth = tile_ctas <= sms ? std::min(kMaxStages, fit) : std::min(kSharedStages, fit);
  g.stages = std::min(g.k_chunks, depth);
  g.tmem_cols = 32;
  while (g.tmem_cols < (uint32_t)(two_m ? 2 * BN : BN)) g.tmem_cols *= 2;
  const uint32_t smem_bytes = g.stages * g.stage_bytes + bar_bytes + 1024;
  g.batch = d.batch;
  g.a_mn = d.a_mn;
  g.C = d.C;
  g.sCz = d.sCz;
  g.sCm = d.sCm;
  g.sCn = d.sCn;
  g.c_fp32 = d.c_fp32;
  g.ws = ws_split ? d.split_ws : nullptr;
  g.status = d.status;
  g.tile_z = d.batch * splits;
  g.b_shared = b_shared ? 1 : 0;
  g.rope_q_pe = d.rope_q_pe;
  g.rope_ld_qp = d.rope_ld_qp;
  g.rope_pos = d.rope_pos;
  g.rope_table = d.rope_table;
  g.rope_max_pos = d.rope_max_pos;
  g.rope_T = d.rope_T;
  g.rope_n_h = d.rope_n_h;
  g.rope_q_full = d.rope_q_full;
  g.app = d.app;
  // side-job CTAs: whole z-slices of the grid, ~64 CTAs of 128 threads
  int side_z = 0;
  long long want = 0;
  if (d.rope_q_pe != nullptr && d.rope_T > 0)
    want = std::min<long long>(64, ((long long)d.rope_T * d.rope_n_h * 8 + 127) / 128);
  if (d.app.n_tokens > 0) want = std::max<long long>(want, std::min(64, (d.app.n_tokens + 3) / 4));
  if (want > 0) side_z = (int)((want + ntile * mtile - 1) / (ntile * mtile));
  if (ws_split) {
    MLA_CUDA_TRY(cudaMemsetAsync(d.split_ws, 0, (size_t)d.M * d.N * d.batch * sizeof(float),
                                 stream));
  } else if (splits > 1 && !pl.part) {
    if (!d.c_contiguous)
      return fail(MLA_ERR_UNSUPPORTED, "split-K needs a contiguous fp32 output");
    MLA_CUDA_TRY(cudaMemsetAsync(d.C, 0, d.c_bytes, stream));
  }
  auto kernel = two_m ? gemm_tc_kernel<true> : gemm_tc_kernel<false>;
  MLA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_bytes));
  dim3 grid(ntile, mtile, d.batch * splits + side_z);
  kernel<<<grid, 128, smem_bytes, stream>>>(tm_a, tm_b, g);
  MLA_LAUNCH_CHECK("gemm_tc_kernel");
  if (pl.part) {
    const long long total = (long long)d.M * d.N * d.batch;
    const int blocks = (int)std::min<long long>(4 * sms, (total + 255) / 256);
    part_reduce_kernel<<<blocks, 256, 0, stream>>>(d.part_ws, splits, d.M, d.N, d.batch,
                                                    static_cast<float *>(d.C), d.sCz, d.sCm,
                                                    d.sCn);
    MLA_LAUNCH_CHECK("part_reduce_kernel");
  }
  if (ws_split) {
    const long long total = (long long)d.M * d.N * d.batch;
    const int blocks = (int)std::min<long long>(1184, (total + 255) / 256);
    split_to_bf16_kernel<<<blocks, 256, 0, stream>>>(d.split_ws, d.M, d.N, d.batch,
                                                      static_cast<uint16_t *>(d.C), d.sCz, d.sCm,
                                                      d.sCn);
    MLA_LAUNCH_CHECK("split_to_bf16_kernel");
  }
  return MLA_OK;
}

}  // namespace mla

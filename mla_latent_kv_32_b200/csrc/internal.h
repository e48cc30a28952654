// Internal launchers shared between the translation units of the library.
#pragma once

#include "common.cuh"
#include "plan.h"

namespace mla {

// The cache append of a decode step, run as a side job of another launch
// (the absorption GEMM): n_tokens == 0 means none. Same arguments as
// mla_cache_append.
struct AppendJob {
  uint16_t *cache;      // bf16 cache, or NULL with the FP8 cache below
  uint8_t *cache8;      // FP8 cache rows (640 bytes) and their scales, or NULL
  float *scales8;
  int num_pages;
  const int32_t *block_table;
  int batch, max_pages;
  const int32_t *seq_idx, *pos;
  const uint16_t *c_kv;
  int ld_c;
  const uint16_t *k_pe;
  int ld_k;
  int n_tokens;
};

// Tensor-core GEMM: C[z][m][n] = sum_k A[z][m][k] * B[z][n][k].
// A element (z,m,k): K-major at A + z*sAz + m*sAm + k, or (a_mn) MN-major at
// A + z*sAz + k*sAk + m. B element (z,n,k) at B + z*sBz + n*sBn + k.
// All strides in elements, multiples of 8 (16 bytes); K % 16 == 0.
struct GemmTcDesc {
  const uint16_t *A;
  long long sAz, sAm, sAk;
  int a_mn;
  const uint16_t *B;
  long long sBz, sBn;
  void *C;
  long long sCz, sCm, sCn;
  int c_fp32;
  int M, N, K, batch;
  int allow_split;       // fp32 output may be split over K (atomic adds, zeroed first)
  int c_contiguous;      // C occupies c_bytes contiguous bytes (needed for the split)
  size_t c_bytes;
  uint32_t *status;
  // bf16 output with a split over K: fp32 partial sums accumulate in
  // split_ws (M*N*batch floats, element (z, n, m) at (z*N + n)*M + m), then
  // are rounded into C. NULL: bf16 outputs are never split.
  float *split_ws;
  // fp32 output with a split over K through a caller workspace: each split
  // writes its partial tile (no atomics) and a second kernel sums them.
  float *part_ws;
  size_t part_ws_bytes;
  // Optional side job run by extra CTAs of the same launch (concurrently with
  // the GEMM tiles): q_full[t][h][512:576] = RoPE(q_pe[t][h][:], pos[t]) (a
  // copy when pos == NULL). Off when rope_q_pe == NULL.
  const uint16_t *rope_q_pe;
  int rope_ld_qp;
  const int32_t *rope_pos;
  const float *rope_table;
  int rope_max_pos, rope_T, rope_n_h;
  uint16_t *rope_q_full;
  // Optional second side job in the same extra CTAs: the step's cache append
  // (uses rope_table / rope_max_pos).
  AppendJob app;
};
mla_status_t launch_gemm_tc(const GemmTcDesc &d, cudaStream_t stream);

// Tile shape and K split launch_gemm_tc takes for a problem (gemm_tc.cu).
struct GemmPlan {
  int BN, two_m, ntile, mtile, splits, k_chunks;
  bool part;          // fp32 partial-sum tiles in a workspace
  size_t part_bytes;  // the workspace those need
};
GemmPlan plan_gemm(int M, int N, int K, int batch, bool a_mn, bool c_fp32, bool fp32_part,
                   bool atomic_split, int sms);

mla_status_t launch_cache_append(uint16_t *cache, int num_pages, const int32_t *block_table,
                                 int batch, int max_pages, const int32_t *seq_idx,
                                 const int32_t *pos, const uint16_t *c_kv, int ld_c,
                                 const uint16_t *k_pe, int ld_k, const float *rope_table,
                                 int max_pos, int n_tokens, uint32_t *status,
                                 cudaStream_t stream);

// FP8 cache: bytes per token row ([512 E4M3 | 64 bf16]) and the append.
constexpr int kFp8RowBytes = MLA_D_C + 2 * MLA_D_R;   // 640
mla_status_t launch_cache_append_fp8(uint8_t *cache, float *scales, int num_pages,
                                     const int32_t *block_table, int batch, int max_pages,
                                     const int32_t *seq_idx, const int32_t *pos,
                                     const uint16_t *c_kv, int ld_c, const uint16_t *k_pe, int ld_k,
                                     const float *rope_table, int max_pos, int n_tokens,
                                     uint32_t *status, cudaStream_t stream);

struct DecodeArgs {
  const uint16_t *q_full;
  const uint16_t *cache;
  int num_pages;
  const int32_t *block_table;
  int max_pages;
  int batch, q_len, n_h;
  float scale_log2;  // scale * log2(e)
  const PlanHeader *plan_host;
  const unsigned char *plan_dev;
  float *ws_o;       // [num_partials][n_h][512]
  float *ws_lse;     // [num_partials][n_h]
  uint16_t *o_latent;
  float *lse;
  uint32_t *status;
  const float *fp8_scales;  // FP8 cache only: [num_pages][64] per-token scales
};
mla_status_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream);
mla_status_t launch_decode_fp8(const DecodeArgs &a, cudaStream_t stream);
mla_status_t launch_decode_pair(const DecodeArgs &a, cudaStream_t stream);
mla_status_t set_decode_wait(double seconds, int suppress_arrive);  // mla_debug_decode_wait
mla_status_t launch_combine(const DecodeArgs &a, cudaStream_t stream);

// The kernels behind each entry point (ops.cu).
mla_status_t launch_absorb_q(const uint16_t *q_nope, int ld_qn, const uint16_t *q_pe, int ld_qp,
                             const int32_t *pos, const float *rope_table, int max_pos,
                             const uint16_t *w_uk, int T, int n_h, uint16_t *q_full,
                             uint32_t *status, cudaStream_t stream,
                             const AppendJob *app = nullptr);
mla_status_t launch_out_absorb(const uint16_t *o_latent, const uint16_t *w_uv, int T, int n_h,
                               uint16_t *u, int ld_u, cudaStream_t stream);
mla_status_t launch_projection(const uint16_t *X, int ld_x, const uint16_t *W, int ld_w, void *C,
                               int ld_c, int c_fp32, int M, int N, int K, float *ws,
                               size_t ws_bytes, cudaStream_t stream);
mla_status_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

}  // namespace mla

// Folded weights: the per-head products that the absorption lets one compute
// once, offline, instead of applying two matrices per token
// ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide", "The Matrix
// Absorption Trick", parts 2-3, where W^UV "can be pre-multiplied" into the
// output projection; "Deconstructing DeepSeek V4 Pro ...", "Practical
// Deployment & Systems Engineering Takeaways", which pre-computes the query
// and key up-projections' product during static compilation):
//
//   W~QK[h*512 + c][i] = sum_d W^UQ[h*128 + d][i] * W^UK[h][d][c]
//       (q~_h = W~QK_h x: the latent query straight from the query input x,
//        which is c^Q, or the hidden state when there is no query latent)
//   W~O[f][h*512 + c]  = sum_d W^O[f][h*128 + d] * W^UV[h][d][c]
//       (out = W~O [o_1; ...; o_H]: the output projection straight from the
//        latent attention outputs)
//
// Both folds run on the tcgen05 GEMM, batched over heads. The query fold needs
// W^UK with d contiguous, so W^UK is first transposed per head into a caller
// workspace. The folded absorption is the same GEMM over K = the query input
// width, with the q^R RoPE pack as its side job.
#include "internal.h"

namespace mla {
namespace {

// dst[h][c][d] = src[h][d][c]   (d < 128, c < 512), through a 32 x 33 tile
__global__ void __launch_bounds__(256)
transpose_head_kernel(const uint16_t *__restrict__ src, uint16_t *__restrict__ dst) {
  __shared__ uint16_t tile[32][33];
  const int h = blockIdx.z;
  const int c0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
  const uint16_t *s = src + (size_t)h * MLA_D_NOPE * MLA_D_C;
  uint16_t *t = dst + (size_t)h * MLA_D_NOPE * MLA_D_C;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
  for (int r = ty; r < 32; r += 8) tile[r][tx] = s[(size_t)(d0 + r) * MLA_D_C + c0 + tx];
  __syncthreads();
  for (int r = ty; r < 32; r += 8) t[(size_t)(c0 + r) * MLA_D_NOPE + d0 + tx] = tile[tx][r];
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

size_t mla_fold_qk_workspace_bytes(int n_h) {
  if (n_h <= 0) return 0;
  return (size_t)n_h * MLA_D_NOPE * MLA_D_C * sizeof(uint16_t);
}

mla_status_t mla_fold_qk(const mla_bf16_t *w_uq, int ld_uq, int q_in, const mla_bf16_t *w_uk,
                         int n_h, mla_bf16_t *w_qk, void *workspace, size_t workspace_bytes,
                         mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(n_h >= 0 && q_in >= 0, "negative size");
  if (n_h == 0 || q_in == 0) return MLA_OK;
  if (n_h > 128 || q_in % 64 != 0)
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (<= 128), q_in = %d (multiple of 64)", n_h, q_in);
  MLA_CHECK_ARG(w_uq && w_uk && w_qk && workspace, "NULL device pointer");
  MLA_CHECK_ARG(aligned16(w_uq) && aligned16(w_uk) && aligned16(w_qk) && aligned16(workspace),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_uq >= q_in && ld_uq % 8 == 0, "ld_uq too small or unaligned");
  if (workspace_bytes < mla_fold_qk_workspace_bytes(n_h))
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu B < %zu B", workspace_bytes,
                mla_fold_qk_workspace_bytes(n_h));
  int major = 0;
  mla_status_t st = device_info(nullptr, &major, nullptr);
  if (st != MLA_OK) return st;
  if (major != 10) return fail(MLA_ERR_UNSUPPORTED, "this library is built for sm_100a");
  cudaStream_t s = (cudaStream_t)stream;
  uint16_t *ukt = static_cast<uint16_t *>(workspace);
  transpose_head_kernel<<<dim3(MLA_D_C / 32, MLA_D_NOPE / 32, n_h), 256, 0, s>>>(w_uk, ukt);
  MLA_LAUNCH_CHECK("transpose_head_kernel");
  // C[h][i][c] = sum_d A[h][i][d] * B[h][c][d]; A = W^UQ rows h*128.. read
  // MN-major (i contiguous), B = W^UK^T (d contiguous)
  GemmTcDesc d = {};
  d.A = w_uq; d.sAz = (long long)MLA_D_NOPE * ld_uq; d.sAk = ld_uq; d.a_mn = 1;
  d.B = ukt; d.sBz = (long long)MLA_D_C * MLA_D_NOPE; d.sBn = MLA_D_NOPE;
  d.C = w_qk; d.sCz = (long long)MLA_D_C * q_in; d.sCm = 1; d.sCn = q_in;
  d.c_fp32 = 0; d.M = q_in; d.N = MLA_D_C; d.K = MLA_D_NOPE; d.batch = n_h;
  return launch_gemm_tc(d, s);
}

mla_status_t mla_fold_o(const mla_bf16_t *w_o, int ld_o, int d_model, const mla_bf16_t *w_uv,
                        int n_h, mla_bf16_t *w_o_folded, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(n_h >= 0 && d_model >= 0, "negative size");
  if (n_h == 0 || d_model == 0) return MLA_OK;
  if (n_h > 128) return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (<= 128)", n_h);
  MLA_CHECK_ARG(w_o && w_uv && w_o_folded, "NULL device pointer");
  MLA_CHECK_ARG(aligned16(w_o) && aligned16(w_uv) && aligned16(w_o_folded),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_o >= n_h * MLA_D_V && ld_o % 8 == 0, "ld_o too small or unaligned");
  int major = 0;
  mla_status_t st = device_info(nullptr, &major, nullptr);
  if (st != MLA_OK) return st;
  if (major != 10) return fail(MLA_ERR_UNSUPPORTED, "this library is built for sm_100a");
  // C[h][c][f] = sum_d A[h][c][d] * B[h][f][d]; A = W^UV[h] read MN-major (c
  // contiguous), B = the head's 128 columns of W^O (d contiguous)
  GemmTcDesc d = {};
  d.A = w_uv; d.sAz = (long long)MLA_D_V * MLA_D_C; d.sAk = MLA_D_C; d.a_mn = 1;
  d.B = w_o; d.sBz = MLA_D_V; d.sBn = ld_o;
  d.C = w_o_folded; d.sCz = MLA_D_C; d.sCm = 1; d.sCn = (long long)n_h * MLA_D_C;
  d.c_fp32 = 0; d.M = MLA_D_C; d.N = d_model; d.K = MLA_D_V; d.batch = n_h;
  return launch_gemm_tc(d, (cudaStream_t)stream);
}

mla_status_t mla_absorb_q_folded(const mla_bf16_t *x, int ld_x, int k_in, const mla_bf16_t *q_pe,
                                 int ld_qp, const mla_bf16_t *w_qk, const int32_t *pos,
                                 const float *rope_table, int max_pos, int T, int n_h,
                                 mla_bf16_t *q_full, uint32_t *status, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(T >= 0 && k_in >= 0, "negative size");
  if (T == 0) return MLA_OK;
  if (!(n_h >= 16 && n_h <= 128 && n_h % 16 == 0) || k_in % 64 != 0 || k_in == 0)
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (16..128 step 16), k_in = %d (multiple of 64)",
                n_h, k_in);
  MLA_CHECK_ARG(x && q_pe && w_qk && q_full, "NULL device pointer");
  MLA_CHECK_ARG(pos == nullptr || (rope_table != nullptr && max_pos > 0),
                "pos given without a RoPE table");
  MLA_CHECK_ARG(aligned16(x) && aligned16(q_pe) && aligned16(w_qk) && aligned16(q_full) &&
                    (rope_table == nullptr || aligned16(rope_table)),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_x >= k_in && ld_x % 8 == 0, "ld_x too small or unaligned");
  MLA_CHECK_ARG(ld_qp >= n_h * MLA_D_R && ld_qp % 8 == 0, "ld_qp too small or unaligned");
  int major = 0;
  mla_status_t st = device_info(nullptr, &major, nullptr);
  if (st != MLA_OK) return st;
  if (major != 10) return fail(MLA_ERR_UNSUPPORTED, "this library is built for sm_100a");
  // q_full[t][h][c] = sum_i W~QK[h*512 + c][i] * x[t][i]: batched over heads,
  // every head reading the same x; the q^R pack runs as the side job
  GemmTcDesc d = {};
  d.A = w_qk; d.sAz = (long long)MLA_D_C * k_in; d.sAm = k_in; d.a_mn = 0;
  d.B = x; d.sBz = 0; d.sBn = ld_x;
  d.C = q_full; d.sCz = MLA_ROW; d.sCm = 1; d.sCn = (long long)n_h * MLA_ROW;
  d.c_fp32 = 0; d.M = MLA_D_C; d.N = T; d.K = k_in; d.batch = n_h;
  d.status = status;
  d.rope_q_pe = q_pe; d.rope_ld_qp = ld_qp; d.rope_pos = pos; d.rope_table = rope_table;
  d.rope_max_pos = max_pos; d.rope_T = T; d.rope_n_h = n_h; d.rope_q_full = q_full;
  return launch_gemm_tc(d, (cudaStream_t)stream);
}

}  // extern "C"

// The kernels behind each entry point of the C ABI.
#include "internal.h"

namespace mla {

// q_full[t][h][c] = sum_d q_nope[t][h][d] * w_uk[h][d][c]   (batched over heads;
// m = latent column c, n = token t, k = d; W^UK read as its transpose), and in
// the same launch q_full[t][h][512:576] = RoPE(q_pe[t][h], pos[t])
mla_status_t launch_absorb_q(const uint16_t *q_nope, int ld_qn, const uint16_t *q_pe, int ld_qp,
                             const int32_t *pos, const float *rope_table, int max_pos,
                             const uint16_t *w_uk, int T, int n_h, uint16_t *q_full,
                             uint32_t *status, cudaStream_t stream, const AppendJob *app) {
  GemmTcDesc d = {};
  d.A = w_uk; d.sAz = (long long)MLA_D_NOPE * MLA_D_C; d.sAk = MLA_D_C; d.a_mn = 1;
  d.B = q_nope; d.sBz = MLA_D_NOPE; d.sBn = ld_qn;
  d.C = q_full; d.sCz = MLA_ROW; d.sCm = 1; d.sCn = (long long)n_h * MLA_ROW;
  d.c_fp32 = 0; d.M = MLA_D_C; d.N = T; d.K = MLA_D_NOPE; d.batch = n_h;
  d.status = status;
  d.rope_q_pe = q_pe; d.rope_ld_qp = ld_qp; d.rope_pos = pos; d.rope_table = rope_table;
  d.rope_max_pos = max_pos; d.rope_T = T; d.rope_n_h = n_h; d.rope_q_full = q_full;
  if (app != nullptr) d.app = *app;
  return launch_gemm_tc(d, stream);
}

// u[t][h*128 + d] = sum_c o[t][h][c] * w_uv[h][d][c]   (batched over heads;
// m = d, n = token t, k = c)
mla_status_t launch_out_absorb(const uint16_t *o_latent, const uint16_t *w_uv, int T, int n_h,
                               uint16_t *u, int ld_u, cudaStream_t stream) {
  GemmTcDesc d = {};
  d.A = w_uv; d.sAz = (long long)MLA_D_V * MLA_D_C; d.sAm = MLA_D_C; d.a_mn = 0;
  d.B = o_latent; d.sBz = MLA_D_C; d.sBn = (long long)n_h * MLA_D_C;
  d.C = u; d.sCz = MLA_D_V; d.sCm = 1; d.sCn = ld_u;
  d.c_fp32 = 0; d.M = MLA_D_V; d.N = T; d.K = MLA_D_C; d.batch = n_h;
  return launch_gemm_tc(d, stream);
}

// C[t][f] = sum_k X[t][k] * W[f][k]   (m = output feature f, n = token t)
mla_status_t launch_projection(const uint16_t *X, int ld_x, const uint16_t *W, int ld_w, void *C,
                               int ld_c, int c_fp32, int M, int N, int K, float *ws,
                               size_t ws_bytes, cudaStream_t stream) {
  GemmTcDesc d = {};
  d.A = W; d.sAz = 0; d.sAm = ld_w; d.a_mn = 0;
  d.B = X; d.sBz = 0; d.sBn = ld_x;
  d.C = C; d.sCz = 0; d.sCm = 1; d.sCn = ld_c;
  d.c_fp32 = c_fp32; d.M = N; d.N = M; d.K = K; d.batch = 1;
  d.allow_split = c_fp32;
  d.c_contiguous = 1;
  d.c_bytes = (size_t)M * ld_c * (c_fp32 ? 4 : 2);
  d.split_ws = c_fp32 ? nullptr : ws;
  d.part_ws = c_fp32 ? ws : nullptr;
  d.part_ws_bytes = c_fp32 ? ws_bytes : 0;
  return launch_gemm_tc(d, stream);
}

mla_status_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  return launch_decode_pair(a, stream);
}

}  // namespace mla

// The kernels behind each entry point of the C ABI.
#include "internal.h"

namespace mla {

// q_full[t][h][c] = sum_d q_nope[t][h][d] * w_uk[h][d][c]   (batched over heads)
mla_status_t launch_absorb_q(const uint16_t *q_nope, int ld_qn, const uint16_t *w_uk, int T,
                             int n_h, uint16_t *q_full, cudaStream_t stream) {
  GemmArgs g;
  g.A = q_nope; g.sAz = MLA_D_NOPE; g.sAm = ld_qn; g.sAk = 1;
  g.B = w_uk; g.sBz = (long long)MLA_D_NOPE * MLA_D_C; g.sBn = 1; g.sBk = MLA_D_C;
  g.C = q_full; g.sCz = MLA_ROW; g.sCm = (long long)n_h * MLA_ROW; g.sCn = 1;
  g.c_fp32 = 0; g.M = T; g.N = MLA_D_C; g.K = MLA_D_NOPE; g.batch = n_h;
  return launch_gemm_simt(g, stream);
}

// u[t][h*128 + d] = sum_c o[t][h][c] * w_uv[h][d][c]   (batched over heads)
mla_status_t launch_out_absorb(const uint16_t *o_latent, const uint16_t *w_uv, int T, int n_h,
                               uint16_t *u, int ld_u, cudaStream_t stream) {
  GemmArgs g;
  g.A = o_latent; g.sAz = MLA_D_C; g.sAm = (long long)n_h * MLA_D_C; g.sAk = 1;
  g.B = w_uv; g.sBz = (long long)MLA_D_V * MLA_D_C; g.sBn = MLA_D_C; g.sBk = 1;
  g.C = u; g.sCz = MLA_D_V; g.sCm = ld_u; g.sCn = 1;
  g.c_fp32 = 0; g.M = T; g.N = MLA_D_V; g.K = MLA_D_C; g.batch = n_h;
  return launch_gemm_simt(g, stream);
}

// C[m][n] = sum_k X[m][k] * W[n][k]
mla_status_t launch_projection(const uint16_t *X, int ld_x, const uint16_t *W, int ld_w, void *C,
                               int ld_c, int c_fp32, int M, int N, int K, cudaStream_t stream) {
  GemmArgs g;
  g.A = X; g.sAz = 0; g.sAm = ld_x; g.sAk = 1;
  g.B = W; g.sBz = 0; g.sBn = ld_w; g.sBk = 1;
  g.C = C; g.sCz = 0; g.sCm = ld_c; g.sCn = 1;
  g.c_fp32 = c_fp32; g.M = M; g.N = N; g.K = K; g.batch = 1;
  return launch_gemm_simt(g, stream);
}

mla_status_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  return launch_decode_tc(a, stream);
}

}  // namespace mla

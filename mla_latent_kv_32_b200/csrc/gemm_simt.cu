// Strided, batched bf16 GEMM on CUDA cores with fp32 accumulation, and the
// q^R RoPE/pack step of mla_absorb_q.
//
// The GEMM serves the small per-head contractions of the absorbed form (W^UK
// folded into the query, W^UV applied to the latent output) and the decode
// layer's projections whenever the tensor-core GEMM does not cover a shape.
// Tile 64x64, k-step 32, 256 threads with a 4x4 register tile each.
#include "internal.h"

namespace mla {
namespace {

constexpr int BM = 64, BN = 64, BK = 32;

template <bool kF32Out>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int z = blockIdx.z;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const uint16_t *A = g.A + (long long)z * g.sAz;
  const uint16_t *B = g.B + (long long)z * g.sBz;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int mm = i / BK, kk = i % BK;
      const int m = m0 + mm, k = k0 + kk;
      float va = 0.f;
      if (m < g.M && k < g.K) va = bf16_bits_to_f32(A[(long long)m * g.sAm + (long long)k * g.sAk]);
      As[kk][mm] = va;
      const int n = n0 + mm;
      float vb = 0.f;
      if (n < g.N && k < g.K) vb = bf16_bits_to_f32(B[(long long)n * g.sBn + (long long)k * g.sBk]);
      Bs[kk][mm] = vb;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) b[i] = Bs[kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      const long long off = (long long)z * g.sCz + (long long)m * g.sCm + (long long)n * g.sCn;
      if (kF32Out)
        reinterpret_cast<float *>(g.C)[off] = acc[i][j];
      else
        reinterpret_cast<uint16_t *>(g.C)[off] = (uint16_t)f32_to_bf16_bits(acc[i][j]);
    }
  }
}

// One warp per (token, head): lanes 0..7 each rotate 4 pairs of q^R.
__global__ void __launch_bounds__(256)
q_rope_pack_kernel(const uint16_t *__restrict__ q_pe, int ld_qp, const int32_t *__restrict__ pos,
                   const float *__restrict__ rope_table, int max_pos, int T, int n_h,
                   uint16_t *__restrict__ q_full, uint32_t *status) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= T * n_h || lane >= 8) return;
  const int t = w / n_h, h = w % n_h;
  const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(q_pe + (size_t)t * ld_qp + h * MLA_D_R) + lane);
  uint4 *dst = reinterpret_cast<uint4 *>(q_full + ((size_t)t * n_h + h) * MLA_ROW + MLA_D_C);
  if (pos == nullptr) {
    dst[lane] = kv;
    return;
  }
  const int p = __ldg(pos + t);
  if (p < 0 || p >= max_pos) {
    if (lane == 0) report(status, MLA_DEV_BAD_POSITION);
    dst[lane] = make_uint4(0, 0, 0, 0);
    return;
  }
  const float4 cs0 = __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8));
  const float4 cs1 = __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8 + 4));
  const uint32_t wv[4] = {kv.x, kv.y, kv.z, kv.w};
  const float cosv[4] = {cs0.x, cs0.z, cs1.x, cs1.z};
  const float sinv[4] = {cs0.y, cs0.w, cs1.y, cs1.w};
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float y0, y1;
    rope_pair_rn(bf16_bits_to_f32(wv[i] & 0xFFFFu), bf16_bits_to_f32(wv[i] >> 16), cosv[i],
                 sinv[i], y0, y1);
    out[i] = pack_bf16x2(y0, y1);
  }
  dst[lane] = make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace

mla_status_t launch_gemm_simt(const GemmArgs &g, cudaStream_t stream) {
  if (g.M == 0 || g.N == 0 || g.batch == 0) return MLA_OK;
  dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM, g.batch);
  if (g.c_fp32)
    gemm_simt_kernel<true><<<grid, 256, 0, stream>>>(g);
  else
    gemm_simt_kernel<false><<<grid, 256, 0, stream>>>(g);
  MLA_LAUNCH_CHECK("gemm_simt_kernel");
  return MLA_OK;
}

mla_status_t launch_q_rope_pack(const uint16_t *q_pe, int ld_qp, const int32_t *pos,
                                const float *rope_table, int max_pos, int T, int n_h,
                                uint16_t *q_full, uint32_t *status, cudaStream_t stream) {
  const int warps = T * n_h;
  if (warps == 0) return MLA_OK;
  q_rope_pack_kernel<<<(warps + 7) / 8, 256, 0, stream>>>(q_pe, ld_qp, pos, rope_table, max_pos,
                                                          T, n_h, q_full, status);
  MLA_LAUNCH_CHECK("q_rope_pack_kernel");
  return MLA_OK;
}

}  // namespace mla

// mla_cache_append: decoupled RoPE on k^R and scatter of the new rows into the
// paged latent cache ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide",
// "3. The Decoupled RoPE Key" and "Step 3": the new latent and rotated key are
// appended before attention).
//
// One warp per token. The 512 latent values move as 64 x 16-byte chunks (two
// per lane); lanes 0..7 each rotate 4 interleaved pairs of k^R (8 values,
// one 16-byte store). The row lands in slot pos % 64 of page
// block_table[b][pos / 64]: 1152 contiguous bytes.
#include "internal.h"

namespace mla {
namespace {

constexpr int kWarpsPerCta = 8;

__global__ void __launch_bounds__(kWarpsPerCta * 32)
cache_append_kernel(uint16_t *__restrict__ cache, int num_pages,
                    const int32_t *__restrict__ block_table, int batch, int max_pages,
                    const int32_t *__restrict__ seq_idx, const int32_t *__restrict__ pos,
                    const uint16_t *__restrict__ c_kv, int ld_c,
                    const uint16_t *__restrict__ k_pe, int ld_k,
                    const float *__restrict__ rope_table, int max_pos, int n_tokens,
                    uint32_t *status) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  const int b = __ldg(seq_idx + t);
  const int p = __ldg(pos + t);
  if (p < 0 || p >= max_pos || (p >> 6) >= max_pages) {
    if (lane == 0) report(status, MLA_DEV_BAD_POSITION);
    return;
  }
  if (b < 0 || b >= batch) {
    if (lane == 0) report(status, MLA_DEV_BAD_PAGE);
    return;
  }
  const int page = __ldg(block_table + (size_t)b * max_pages + (p >> 6));
  if (page < 0 || page >= num_pages) {
    if (lane == 0) report(status, MLA_DEV_BAD_PAGE);
    return;
  }
  uint16_t *dst = cache + ((size_t)page * MLA_PAGE + (p & 63)) * MLA_ROW;

  // latent: 1024 bytes = 64 chunks of 16 bytes
  const uint4 *src_c = reinterpret_cast<const uint4 *>(c_kv + (size_t)t * ld_c);
  uint4 *dst_c = reinterpret_cast<uint4 *>(dst);
  uint4 v0 = __ldg(src_c + lane);
  uint4 v1 = __ldg(src_c + lane + 32);
  dst_c[lane] = v0;
  dst_c[lane + 32] = v1;

  // RoPE key: lanes 0..7 rotate pairs 4*lane .. 4*lane+3
  if (lane < 8) {
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(k_pe + (size_t)t * ld_k) + lane);
    const float4 cs0 = __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8));
    const float4 cs1 = __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8 + 4));
    const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
    const float cosv[4] = {cs0.x, cs0.z, cs1.x, cs1.z};
    const float sinv[4] = {cs0.y, cs0.w, cs1.y, cs1.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float x0 = bf16_bits_to_f32(w[i] & 0xFFFFu);
      float x1 = bf16_bits_to_f32(w[i] >> 16);
      float y0, y1;
      rope_pair_rn(x0, x1, cosv[i], sinv[i], y0, y1);
      out[i] = pack_bf16x2(y0, y1);
    }
    reinterpret_cast<uint4 *>(dst + MLA_D_C)[lane] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace

mla_status_t launch_cache_append(uint16_t *cache, int num_pages, const int32_t *block_table,
                                 int batch, int max_pages, const int32_t *seq_idx,
                                 const int32_t *pos, const uint16_t *c_kv, int ld_c,
                                 const uint16_t *k_pe, int ld_k, const float *rope_table,
                                 int max_pos, int n_tokens, uint32_t *status,
                                 cudaStream_t stream) {
  const int grid = (n_tokens + kWarpsPerCta - 1) / kWarpsPerCta;
  cache_append_kernel<<<grid, kWarpsPerCta * 32, 0, stream>>>(
      cache, num_pages, block_table, batch, max_pages, seq_idx, pos, c_kv, ld_c, k_pe, ld_k,
      rope_table, max_pos, n_tokens, status);
  MLA_LAUNCH_CHECK("cache_append_kernel");
  return MLA_OK;
}

}  // namespace mla

// One warp appends one token to the bf16 paged cache: the row
// [c_kv[t][0:512] | RoPE(k_pe[t][0:64], pos[t])] lands in page
// block_table[seq_idx[t]][pos[t] / 64], slot pos[t] % 64 ("DeepSeek-V3 MLA:
// Multi-Head Latent Attention Guide", "3. The Decoupled RoPE Key" and "Step
// 3": the new latent and rotated key are appended before attention). The
// rotation is float32 with each product and sum rounded once, then bf16.
// Used by the append kernel and by the absorption launch's side job.
#pragma once

#include "common.cuh"

namespace mla {

__device__ __forceinline__ void append_token_warp(
    uint16_t *__restrict__ cache, int num_pages, const int32_t *__restrict__ block_table,
    int batch, int max_pages, const int32_t *__restrict__ seq_idx,
    const int32_t *__restrict__ pos, const uint16_t *__restrict__ c_kv, int ld_c,
    const uint16_t *__restrict__ k_pe, int ld_k, const float *__restrict__ rope_table,
    int max_pos, int t, int lane, uint32_t *status) {
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
  const uint4 v0 = __ldg(src_c + lane);
  const uint4 v1 = __ldg(src_c + lane + 32);
  dst_c[lane] = v0;
  dst_c[lane + 32] = v1;

  // RoPE key: lanes 0..7 rotate pairs 4*lane .. 4*lane+3
  if (lane < 8) {
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(k_pe + (size_t)t * ld_k) + lane);
    const float4 cs0 =
        __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8));
    const float4 cs1 =
        __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8 + 4));
    const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
    const float cosv[4] = {cs0.x, cs0.z, cs1.x, cs1.z};
    const float sinv[4] = {cs0.y, cs0.w, cs1.y, cs1.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float y0, y1;
      rope_pair_rn(bf16_bits_to_f32(w[i] & 0xFFFFu), bf16_bits_to_f32(w[i] >> 16), cosv[i],
                   sinv[i], y0, y1);
      out[i] = pack_bf16x2(y0, y1);
    }
    reinterpret_cast<uint4 *>(dst + MLA_D_C)[lane] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace mla

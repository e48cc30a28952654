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

// One warp appends one token to the FP8 paged cache. Row: [512 E4M3 latent
// codes | k^R as bf16 (128 B)] = 640 bytes, plus one float32 scale per token:
// the least power of two 2^k with max|c| / 2^k <= 448 (1 for an all-zero
// latent). codes = E4M3(c / 2^k), round to nearest even, saturating; c / 2^k
// is exact (ldexpf). Lane l quantizes latent values [16 l, 16 l + 16); lanes
// 0..7 rotate k^R as the bf16 cache does ("Deconstructing DeepSeek V4 Pro ...",
// "Practical Deployment & Systems Engineering Takeaways": c^KV tolerates
// E4M3). Used by the FP8 append kernel and by the absorption launch's side job.
__device__ __forceinline__ void append_token_fp8_warp(
    uint8_t *__restrict__ cache, float *__restrict__ scales, int num_pages,
    const int32_t *__restrict__ block_table, int batch, int max_pages,
    const int32_t *__restrict__ seq_idx, const int32_t *__restrict__ pos,
    const uint16_t *__restrict__ c_kv, int ld_c, const uint16_t *__restrict__ k_pe, int ld_k,
    const float *__restrict__ rope_table, int max_pos, int t, int lane, uint32_t *status) {
  constexpr int kRowBytes = MLA_D_C + 2 * MLA_D_R;   // 640
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
  const size_t slot = (size_t)page * MLA_PAGE + (p & 63);
  uint8_t *dst = cache + slot * kRowBytes;

  const uint4 *src_c = reinterpret_cast<const uint4 *>(c_kv + (size_t)t * ld_c);
  const uint4 v0 = __ldg(src_c + 2 * lane), v1 = __ldg(src_c + 2 * lane + 1);
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float x[16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    x[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    amax = fmaxf(amax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  int k = 0;
  if (amax > 0.f) {
    int e;
    const float m = frexpf(amax, &e);   // amax = m 2^e, m in [0.5, 1)
    k = m <= 0.875f ? e - 9 : e - 8;    // 448 = 0.875 * 2^9
  }
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo, hi;
    const float a0 = ldexpf(x[4 * i], -k), a1 = ldexpf(x[4 * i + 1], -k);
    const float a2 = ldexpf(x[4 * i + 2], -k), a3 = ldexpf(x[4 * i + 3], -k);
    asm("{\n\t.reg .b16 r;\n\tcvt.rn.satfinite.e4m3x2.f32 r, %1, %2;\n\tcvt.u32.u16 %0, r;\n\t}"
        : "=r"(lo) : "f"(a1), "f"(a0));
    asm("{\n\t.reg .b16 r;\n\tcvt.rn.satfinite.e4m3x2.f32 r, %1, %2;\n\tcvt.u32.u16 %0, r;\n\t}"
        : "=r"(hi) : "f"(a3), "f"(a2));
    q[i] = lo | (hi << 16);
  }
  reinterpret_cast<uint4 *>(dst)[lane] = make_uint4(q[0], q[1], q[2], q[3]);
  if (lane == 0) scales[slot] = ldexpf(1.f, k);

  if (lane < 8) {
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(k_pe + (size_t)t * ld_k) + lane);
    const float4 cs0 = __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8));
    const float4 cs1 = __ldg(reinterpret_cast<const float4 *>(rope_table + (size_t)p * 64 + lane * 8 + 4));
    const uint32_t wk[4] = {kv.x, kv.y, kv.z, kv.w};
    const float cosv[4] = {cs0.x, cs0.z, cs1.x, cs1.z};
    const float sinv[4] = {cs0.y, cs0.w, cs1.y, cs1.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float y0, y1;
      rope_pair_rn(bf16_bits_to_f32(wk[i] & 0xFFFFu), bf16_bits_to_f32(wk[i] >> 16), cosv[i],
                   sinv[i], y0, y1);
      out[i] = pack_bf16x2(y0, y1);
    }
    reinterpret_cast<uint4 *>(dst + MLA_D_C)[lane] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace mla

// mla_cache_append: decoupled RoPE on k^R and scatter of the new rows into the
// paged latent cache ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide",
// "3. The Decoupled RoPE Key" and "Step 3": the new latent and rotated key are
// appended before attention).
//
// One warp per token. The 512 latent values move as 64 x 16-byte chunks (two
// per lane); lanes 0..7 each rotate 4 interleaved pairs of k^R (8 values,
// one 16-byte store). The row lands in slot pos % 64 of page
// block_table[b][pos / 64]: 1152 contiguous bytes.
#include "append.cuh"
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
  const int t = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  append_token_warp(cache, num_pages, block_table, batch, max_pages, seq_idx, pos, c_kv, ld_c,
                    k_pe, ld_k, rope_table, max_pos, t, threadIdx.x & 31, status);
}

// FP8 cache row: [512 E4M3 latent codes | k^R as bf16 (128 B)] = 640 bytes,
// plus one float32 scale per token: the least power of two 2^k with
// max|c| / 2^k <= 448 (1 for an all-zero latent). codes = E4M3(c / 2^k),
// round to nearest even, saturating; c / 2^k is exact (ldexpf). Lane l
// quantizes latent values [16 l, 16 l + 16); lanes 0..7 rotate k^R as the bf16
// cache does.
__global__ void __launch_bounds__(kWarpsPerCta * 32)
cache_append_fp8_kernel(uint8_t *__restrict__ cache, float *__restrict__ scales, int num_pages,
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
  const size_t slot = (size_t)page * MLA_PAGE + (p & 63);
  uint8_t *dst = cache + slot * kFp8RowBytes;

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

}  // namespace

mla_status_t launch_cache_append_fp8(uint8_t *cache, float *scales, int num_pages,
                                     const int32_t *block_table, int batch, int max_pages,
                                     const int32_t *seq_idx, const int32_t *pos,
                                     const uint16_t *c_kv, int ld_c, const uint16_t *k_pe, int ld_k,
                                     const float *rope_table, int max_pos, int n_tokens,
                                     uint32_t *status, cudaStream_t stream) {
  const int grid = (n_tokens + kWarpsPerCta - 1) / kWarpsPerCta;
  cache_append_fp8_kernel<<<grid, kWarpsPerCta * 32, 0, stream>>>(
      cache, scales, num_pages, block_table, batch, max_pages, seq_idx, pos, c_kv, ld_c, k_pe,
      ld_k, rope_table, max_pos, n_tokens, status);
  MLA_LAUNCH_CHECK("cache_append_fp8_kernel");
  return MLA_OK;
}

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

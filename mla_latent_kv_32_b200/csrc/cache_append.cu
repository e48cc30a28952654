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

// FP8 cache (see append_token_fp8_warp).
__global__ void __launch_bounds__(kWarpsPerCta * 32)
cache_append_fp8_kernel(uint8_t *__restrict__ cache, float *__restrict__ scales, int num_pages,
                        const int32_t *__restrict__ block_table, int batch, int max_pages,
                        const int32_t *__restrict__ seq_idx, const int32_t *__restrict__ pos,
                        const uint16_t *__restrict__ c_kv, int ld_c,
                        const uint16_t *__restrict__ k_pe, int ld_k,
                        const float *__restrict__ rope_table, int max_pos, int n_tokens,
                        uint32_t *status) {
  const int t = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  append_token_fp8_warp(cache, scales, num_pages, block_table, batch, max_pages, seq_idx, pos,
                        c_kv, ld_c, k_pe, ld_k, rope_table, max_pos, t, threadIdx.x & 31, status);
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

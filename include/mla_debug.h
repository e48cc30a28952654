/*
 * mla_debug.h -- diagnostic entry points of the MLA decode library.
 *
 * Not part of the decode path. They exist so that tests can compare two
 * independent GPU implementations of the same operation, and exercise the
 * device-side failure detection without faulting the GPU.
 */
#ifndef MLA_DEBUG_H_
#define MLA_DEBUG_H_

#include "mla.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * mla_decode_attention_cudacore -- device. Same contract and arguments as
 * mla_decode_attention ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide",
 * "The Matrix Absorption Trick", parts 2-4), computed by a plain CUDA-core
 * kernel (fp32 FMA; one CTA per work item and 16 heads) instead of the
 * tensor-core kernel. Same plan and workspace; same error behaviour.
 * Orders of magnitude slower; for differential testing only.
 */
mla_status_t mla_decode_attention_cudacore(const mla_bf16_t *q_full, const mla_bf16_t *cache,
                                           int num_pages, const int32_t *block_table,
                                           int max_pages, int batch, int q_len, int n_h,
                                           float scale, const void *plan_host,
                                           const void *plan_dev, void *workspace,
                                           size_t workspace_bytes, mla_bf16_t *o_latent,
                                           float *lse, uint32_t *status, mla_stream_t stream);

/*
 * mla_debug_decode_wait -- host. Failure-detection switch of the tensor-core
 * decode kernel for the calls that follow (process-wide; not thread-safe).
 *   wait_cap_seconds: bound of every wait of the decode kernel on a barrier
 *                     (default 1.0; must be > 0 and <= 10).
 *   suppress_arrive:  1 = the producer of each CTA pair skips its first
 *                     arrival on the first stage barrier, so the MMA issuer's
 *                     wait on it can only end by running out; 0 = normal.
 * When a wait runs out the kernel sets MLA_DEV_TIMEOUT in the status word,
 * stops issuing work, lets what it issued complete and exits; the context
 * stays usable. The pages describe no failure handling; this is the build's
 * own test hook. Returns INVALID_ARGUMENT for a cap outside (0, 10].
 */
mla_status_t mla_debug_decode_wait(double wait_cap_seconds, int suppress_arrive);

/*
 * mla_debug_gemm_plan -- host, no device needed. The tile plan the
 * tensor-core GEMM takes for a problem, so that tests can check the planner
 * on the CPU. C[z][m][n] = sum_k A[z][m][k] B[z][n][k] with M weight rows, N
 * tokens, K the reduction, `batch` problems; a_mn: A is MN-major; c_fp32: the
 * output is float32; fp32_part: an fp32 output with a partial-sum workspace
 * (mla_gemm_bf16_ws); atomic_split: a split over K may accumulate with atomic
 * adds; sms: the SM count to plan for.
 *   out[0] N tile (BN), out[1] 128-row accumulators per CTA (1 or 2),
 *   out[2] N tiles, out[3] M tiles, out[4] splits over K, out[5] 64-wide
 *   k-chunks per split, out[6] 1 when the splits write partial tiles,
 *   out[7] the partial-tile workspace bytes (low 31 bits are enough for the
 *   checked shapes; larger values saturate at 2^31 - 1).
 * Returns INVALID_ARGUMENT for non-positive sizes or a NULL `out`.
 */
mla_status_t mla_debug_gemm_plan(int M, int N, int K, int batch, int a_mn, int c_fp32,
                                 int fp32_part, int atomic_split, int sms, int32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DEBUG_H_ */

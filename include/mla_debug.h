/*
 * mla_debug.h -- diagnostic entry points of the MLA decode library.
 *
 * Not part of the decode path. They exist so that tests can compare two
 * independent GPU implementations of the same operation.
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

#ifdef __cplusplus
}
#endif

#endif /* MLA_DEBUG_H_ */

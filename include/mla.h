/*
 * mla.h -- C ABI of the absorbed Multi-Head Latent Attention (MLA) decode
 * library for NVIDIA B200 (sm_100a).
 *
 * The library computes one decode step of MLA with weight absorption over a
 * paged latent cache, as described on the MLA pages:
 *   - the cache holds, per token, the 512-dim latent c^KV and the 64-dim
 *     decoupled RoPE key k^R ("DeepSeek-V3 MLA: Multi-Head Latent Attention
 *     Guide", section "4. Cache Footprint Math");
 *   - W^UK is folded into the query, q~_i = (W^UK_i)^T q^C_i, and the scores
 *     are taken directly on the latents, score_j = q~_i . c_j + q^R_i . k^R_j
 *     (same page, "The Matrix Absorption Trick", part 2);
 *   - the softmax-weighted latents o_i = sum_j a_ij c_j are expanded once
 *     through W^UV, u_i = W^UV_i o_i (same page, part 3).
 *
 * Conventions shared by every call:
 *   - All tensors are caller-owned. Pointers documented as "device" must be
 *     device memory of the current CUDA device; "host" pointers are host
 *     memory. The library allocates no device memory in any call.
 *   - bf16 tensors are passed as uint16_t bit patterns (mla_bf16_t).
 *   - Every device call is asynchronous on the given stream (a cudaStream_t
 *     passed as void*; NULL = the legacy default stream) and never
 *     synchronises, except mla_read_status.
 *   - Every call returns an mla_status_t; no C++ exception crosses the ABI.
 *     On an error nothing is launched (argument errors) and a message is
 *     available from mla_last_error() on the calling thread.
 *   - Kernels that find bad data (a page id outside the pool, a position
 *     outside the RoPE table, an expired bounded wait) skip the affected
 *     work and OR an MLA_DEV_* bit into the optional device status word
 *     `status` (a uint32_t in device memory, may be NULL). They never trap.
 *   - Device pointers must be 16-byte aligned unless stated otherwise; row
 *     strides (in elements) must keep every row 16-byte aligned.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mla_bf16_t;   /* bf16 bit pattern */
typedef void *mla_stream_t;    /* cudaStream_t */

/* Fixed widths of the method (DeepSeek-V2/V3 MLA). */
#define MLA_D_C 512    /* latent width of c^KV */
#define MLA_D_R 64     /* decoupled RoPE width of k^R, q^R */
#define MLA_D_NOPE 128 /* per-head content query/key width d_h */
#define MLA_D_V 128    /* per-head value width */
#define MLA_ROW 576    /* cached elements per token: [c^KV | k^R] */
#define MLA_PAGE 64    /* tokens per cache page */
#define MLA_MAX_Q_LEN 1024 /* query tokens per sequence in one call (MTP verify, prefill chunk) */

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARGUMENT = 1,    /* null/misaligned pointer, bad size or stride */
  MLA_ERR_UNSUPPORTED = 2,         /* shape outside the supported set, or not sm_100 */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* plan or workspace buffer smaller than required */
  MLA_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed */
  MLA_ERR_DEVICE = 5               /* mla_read_status found device status bits set */
} mla_status_t;

/* Device status bits (OR-ed into the caller's status word). */
#define MLA_DEV_BAD_PAGE 0x1u     /* page id or sequence index out of range: work skipped */
#define MLA_DEV_BAD_POSITION 0x2u /* position outside the RoPE table or the page table */
#define MLA_DEV_TIMEOUT 0x4u      /* a bounded wait expired: the kernel abandoned its work */
#define MLA_DEV_BAD_PLAN 0x8u     /* a work item disagrees with the sequence lengths */
#define MLA_DEV_RANGE 0x10u       /* FP8 decode: a latent query value that is not finite in
                                     fp16 (|x| >= 65520, inf, NaN), or a token scale above 2^7 */

/* Message of the last failed call on this thread ("" if none). */
const char *mla_last_error(void);

/* Library ABI version (increments on any signature change). */
int mla_version(void);

/*
 * mla_rope_table -- host. Fills table[max_pos][32][2] (float32) with
 * (cos, sin) of theta_j = pos / base^(2j/64), j = 0..31, computed in double
 * precision and rounded once to float. Interleaved pairs (2j, 2j+1) are
 * rotated by theta_j ("Deconstructing DeepSeek V4 Pro ...", section "Hands-On
 * PyTorch Implementation", apply_rope).
 *   table: host, caller-owned, max_pos * 64 floats.
 * Errors: INVALID_ARGUMENT if table is NULL, max_pos <= 0 or base <= 1.
 */
mla_status_t mla_rope_table(float *table, int max_pos, double base);

/*
 * mla_cache_append -- device. Appends n_tokens new tokens to the paged cache:
 * for token t (sequence seq_idx[t], position pos[t]) the row
 *   [c_kv[t][0:512] | RoPE(k_pe[t][0:64], pos[t])]
 * is written to page block_table[seq_idx[t] * max_pages + pos[t] / 64],
 * slot pos[t] % 64. The decoupled RoPE key is rotated before it is cached
 * ("DeepSeek-V3 MLA ... Guide", "3. The Decoupled RoPE Key"; "Step 3" appends
 * the new latent and rotated key to the cache before attention).
 * The rotation is float32 with no fused multiply-add: for pair j,
 *   y0 = x0*cos - x1*sin, y1 = x1*cos + x0*sin, each product and sum rounded
 * once, then rounded to bf16 (nearest even), so the stored code is a fixed
 * function of the inputs and the table.
 *   cache:       device bf16 [num_pages][64][576], updated in place.
 *   block_table: device int32 [batch][max_pages], page ids.
 *   seq_idx,pos: device int32 [n_tokens].
 *   c_kv:        device bf16, row t at c_kv + t*ld_c (512 elements).
 *   k_pe:        device bf16, row t at k_pe + t*ld_k (64 elements, pre-RoPE).
 *   rope_table:  device float32 [max_pos][32][2] (see mla_rope_table).
 *   status:      device uint32 or NULL.
 * A token with seq_idx outside [0,batch), pos outside [0,max_pos) or
 * pos/64 >= max_pages, or whose page id is outside [0,num_pages), is skipped
 * and sets MLA_DEV_BAD_PAGE / MLA_DEV_BAD_POSITION.
 */
mla_status_t mla_cache_append(mla_bf16_t *cache, int num_pages,
                              const int32_t *block_table, int batch, int max_pages,
                              const int32_t *seq_idx, const int32_t *pos,
                              const mla_bf16_t *c_kv, int ld_c,
                              const mla_bf16_t *k_pe, int ld_k,
                              const float *rope_table, int max_pos, int n_tokens,
                              uint32_t *status, mla_stream_t stream);

/*
 * mla_absorb_q -- device. Folds W^UK into the content query and packs the
 * query row the attention kernel reads:
 *   q_full[t][h][0:512]   = sum_d q_nope[t][h][d] * w_uk[h][d][:]
 *   q_full[t][h][512:576] = RoPE(q_pe[t][h][:], pos[t])   (or a copy if pos == NULL)
 * ("DeepSeek-V3 MLA ... Guide", "The Matrix Absorption Trick", part 2:
 * q~ = (W^UK_i)^T q^C_i, computed once per query token).
 *   q_nope: device bf16, element (t,h,d) at q_nope + t*ld_qn + h*128 + d.
 *   q_pe:   device bf16, element (t,h,r) at q_pe + t*ld_qp + h*64 + r (pre-RoPE).
 *   w_uk:   device bf16 [n_h][128][512] (the view(n_h, d_h, d_c) of W^UK).
 *   pos:    device int32 [T] absolute positions, or NULL.
 *   rope_table: device float32 [max_pos][32][2] (unused when pos == NULL).
 *   q_full: device bf16 [T][n_h][576], written.
 * fp32 accumulation, one bf16 rounding per output element.
 * Supported: 1 <= n_h <= 128, n_h % 16 == 0.
 */
mla_status_t mla_absorb_q(const mla_bf16_t *q_nope, int ld_qn,
                          const mla_bf16_t *q_pe, int ld_qp,
                          const mla_bf16_t *w_uk, const int32_t *pos,
                          const float *rope_table, int max_pos, int T, int n_h,
                          mla_bf16_t *q_full, uint32_t *status, mla_stream_t stream);

/*
 * mla_append_absorb_q -- device. mla_cache_append and mla_absorb_q of one
 * decode step in one launch (the append runs in extra CTAs of the absorption
 * GEMM, beside the q^R RoPE pack): the same results as the two calls in that
 * order ("DeepSeek-V3 MLA ... Guide", "Step 3": append the new rows, absorb
 * the query). The cache arguments are those of mla_cache_append (positions
 * tok_pos, n_tokens rows), the query arguments those of mla_absorb_q
 * (positions q_pos, may be NULL); the RoPE table is shared and required.
 * The appended rows are not read by this call. Errors: as the two calls.
 */
mla_status_t mla_append_absorb_q(mla_bf16_t *cache, int num_pages, const int32_t *block_table,
                                 int batch, int max_pages, const int32_t *seq_idx,
                                 const int32_t *tok_pos, const mla_bf16_t *c_kv, int ld_c,
                                 const mla_bf16_t *k_pe, int ld_k, int n_tokens,
                                 const mla_bf16_t *q_nope, int ld_qn, const mla_bf16_t *q_pe,
                                 int ld_qp, const mla_bf16_t *w_uk, const int32_t *q_pos,
                                 const float *rope_table, int max_pos, int T, int n_h,
                                 mla_bf16_t *q_full, uint32_t *status, mla_stream_t stream);

/*
 * Decode plan. The split of each sequence's pages into work items is made on
 * the host from the sequence lengths (split-KV: long sequences are cut into
 * several items whose partial results are merged by a log-sum-exp combine).
 * The plan is a flat byte buffer; its size depends only on (batch, q_len,
 * num_ctas) and is returned by mla_plan_bytes. mla_plan_upload copies the
 * host plan to a caller-owned device buffer; mla_decode_attention takes both
 * copies (the host one for the launch shape, the device one for the kernels).
 */
typedef struct mla_plan_info {
  int num_items;        /* work items in the plan */
  int num_ctas;         /* concurrent work lists (CTA clusters) the plan targets */
  int num_partials;     /* partial-result slots used by split items */
  int num_combine;      /* (sequence, query) pairs that need the combine pass */
  size_t plan_bytes;    /* bytes of the plan actually used */
  size_t workspace_bytes; /* device scratch mla_decode_attention needs */
} mla_plan_info_t;

/* Upper bound of the plan size for these sizes (host, no side effects). */
size_t mla_plan_bytes(int batch, int q_len, int num_ctas);

/*
 * mla_decode_plan -- host.
 *   seq_lens: host int32 [batch], total tokens of each sequence including the
 *             q_len new ones (1 <= q_len <= seq_lens[b]).
 *   q_len:    query tokens per sequence, 1..MLA_MAX_Q_LEN; query j of
 *             sequence b sits at position seq_lens[b] - q_len + j and sees the
 *             keys at positions <= its own: the causal mask between the tokens
 *             of a multi-token-prediction verify step ("DeepSeek-V3 & MLA in
 *             2026 ...", section 5) or of a chunked-prefill chunk (the causal
 *             forward of "DeepSeek-V3 MLA ... Guide", Step 2, restricted to the
 *             chunk's queries, computed in the absorbed form).
 *   num_ctas: work lists to balance over; 0 = derive from the current
 *             device's SM count.
 *   max_split: 1 = every (sequence, query) is one item (no combine pass);
 *             0 = cut the pages of all sequences into num_ctas equal ranges
 *             (long sequences become several items merged by the combine);
 *             negative = build both and keep the one with the smaller
 *             estimated time.
 *   plan:     host buffer of plan_bytes (>= mla_plan_bytes(batch, q_len, num_ctas)).
 *   info:     out, may be NULL.
 * Errors: INVALID_ARGUMENT (bad lengths, q_len < 1), UNSUPPORTED (q_len >
 * MLA_MAX_Q_LEN or n_h outside 16..128 step 16), WORKSPACE_TOO_SMALL (plan
 * buffer).
 */
mla_status_t mla_decode_plan(const int32_t *seq_lens, int batch, int q_len, int n_h,
                             int num_ctas, int max_split, void *plan, size_t plan_bytes,
                             mla_plan_info_t *info);

/*
 * mla_plan_used_bytes -- host. Bytes of a built plan that the kernels read
 * (header, work lists, items, combine items); 0 if plan_host is NULL or not
 * a plan.
 */
size_t mla_plan_used_bytes(const void *plan_host);

/*
 * mla_plan_upload -- device copy. Copies the used bytes of the host plan to
 * plan_dev (cudaMemcpyAsync on `stream`). The host plan must stay unchanged
 * until the copy has completed (it is read asynchronously when it lives in
 * page-locked memory).
 *   plan_dev: device, 16-byte aligned, >= mla_plan_used_bytes(plan_host).
 * Errors: INVALID_ARGUMENT (NULL, misaligned, not a plan),
 * WORKSPACE_TOO_SMALL (plan_dev_bytes too small), CUDA.
 */
mla_status_t mla_plan_upload(const void *plan_host, void *plan_dev, size_t plan_dev_bytes,
                             mla_stream_t stream);

/*
 * mla_decode_attention -- device. Absorbed attention over the paged cache:
 * for sequence b, query j (position p = L_b - q_len + j) and head h,
 *   s_i   = (q_full[b][j][h][0:512] . c_i + q_full[b][j][h][512:576] . k^R_i) * scale,
 *           for cached tokens i <= p (the new tokens are already appended);
 *   a     = softmax(s);  o_latent[b][j][h][:] = sum_i a_i c_i;
 *   lse[b][j][h] = log(sum_i exp(s_i)) (natural log), if lse != NULL.
 * ("DeepSeek-V3 MLA ... Guide", "The Matrix Absorption Trick" parts 2-4 and
 * "Step 3": scores on the 512-dim latents plus the RoPE term, softmax, latent
 * output.) Long sequences are split across CTA clusters per the plan and
 * merged by a log-sum-exp combine pass.
 *   q_full:      device bf16 [batch][q_len][n_h][576] (from mla_absorb_q).
 *   cache:       device bf16 [num_pages][64][576].
 *   block_table: device int32 [batch][max_pages].
 *   plan_host / plan_dev: the same plan bytes in host and device memory.
 *   workspace:   device scratch of >= info.workspace_bytes (16-byte aligned).
 *   o_latent:    device bf16 [batch][q_len][n_h][512], written.
 *   lse:         device float32 [batch][q_len][n_h] or NULL.
 * Cache slots past a sequence's length (inside its last page) must hold
 * finite values: they are read, and given weight zero.
 * Supported: n_h % 16 == 0, 16 <= n_h <= 128, 1 <= q_len <= MLA_MAX_Q_LEN (as
 * the plan).
 */
mla_status_t mla_decode_attention(const mla_bf16_t *q_full, const mla_bf16_t *cache,
                                  int num_pages, const int32_t *block_table, int max_pages,
                                  int batch, int q_len, int n_h, float scale,
                                  const void *plan_host, const void *plan_dev,
                                  void *workspace, size_t workspace_bytes,
                                  mla_bf16_t *o_latent, float *lse, uint32_t *status,
                                  mla_stream_t stream);

/*
 * mla_decode_attention_noalloc -- device. The same attention as
 * mla_decode_attention, for callers that cannot supply device memory of their
 * own at the time of the call: a serving engine that has reserved the GPU's
 * memory for its own cache pool, or a plugin running under another
 * framework's allocator. The pages describe no such variant; it exists only
 * for those callers.
 * Instead of a caller-supplied workspace, the split-KV partial results go to a
 * fixed 48 MiB array inside the library (allocated on every GPU that loads the
 * library, held until the process exits). The caller still passes all inputs
 * and outputs. The first call on each device looks up the array's address
 * (with that device current); make that first call before any stream capture.
 * The address is kept per device index for the life of the process: after a
 * cudaDeviceReset of that device it is stale.
 * Every call shares the array and it keeps the previous call's contents;
 * nothing in it needs to start at zero. Calls that can overlap on the GPU
 * (other streams or host threads) race on the array: serialise them.
 * No cudaMalloc, cudaFree or other allocating routine is called.
 * Errors: as mla_decode_attention; WORKSPACE_TOO_SMALL when the plan needs more
 * than 48 MiB of partial results (plan with fewer splits, e.g. max_split = 1).
 */
mla_status_t mla_decode_attention_noalloc(const mla_bf16_t *q_full, const mla_bf16_t *cache,
                                          int num_pages, const int32_t *block_table,
                                          int max_pages, int batch, int q_len, int n_h,
                                          float scale, const void *plan_host,
                                          const void *plan_dev, mla_bf16_t *o_latent,
                                          float *lse, uint32_t *status, mla_stream_t stream);

/*
 * FP8 latent cache ("Deconstructing DeepSeek V4 Pro ...", "Practical
 * Deployment & Systems Engineering Takeaways": the latent c^KV tolerates
 * E4M3; "DeepSeek-V3 MLA ... Guide", "4. Cache Footprint Math": an FP8
 * cache). Layout: cache8 [num_pages][64][640] bytes, a row being
 *   bytes [0, 512)   the 512 latent values as E4M3 codes, code = E4M3(c / s)
 *                    (round to nearest even, saturating at 448),
 *   bytes [512, 640) the rotated k^R as the same 64 bf16 codes the bf16 cache
 *                    stores (little-endian),
 * and scales [num_pages][64] float32: s = the least power of two 2^k with
 * max|c| / 2^k <= 448 (1 when the latent is all zero), so c / s and code * s
 * are exact. 640 + 4 bytes per token against 1152 for the bf16 cache.
 *
 * mla_cache_append_fp8 -- device. mla_cache_append for the FP8 cache: the
 * row and the scale of each new token are written to its page slot (same
 * placement, RoPE and error behaviour as mla_cache_append).
 *   cache: device, 16-byte aligned, updated in place. scales: device float32
 *   [num_pages][64], 16-byte aligned, updated in place.
 *
 * mla_decode_attention_fp8 -- device. mla_decode_attention over the FP8
 * cache: the same result for the dequantized rows (code * s, k^R); the same
 * plan, workspace, outputs and errors. The latent products run on fp16
 * operands: the dequantized values code * s exactly (for scales in
 * [2^-15, 2^7]; below 2^-15 the smallest codes round on the fp16 grid), the
 * query's latent columns as fp16 (exact for bf16 values in the fp16 normal
 * range), the probabilities rounded to fp16. The RoPE products stay bf16.
 * A latent query value that is not finite in fp16, or a scale above 2^7,
 * sets MLA_DEV_RANGE in *status (the outputs are then not meaningful).
 */
mla_status_t mla_cache_append_fp8(uint8_t *cache, float *scales, int num_pages,
                                  const int32_t *block_table, int batch, int max_pages,
                                  const int32_t *seq_idx, const int32_t *pos,
                                  const mla_bf16_t *c_kv, int ld_c, const mla_bf16_t *k_pe,
                                  int ld_k, const float *rope_table, int max_pos, int n_tokens,
                                  uint32_t *status, mla_stream_t stream);
/*
 * mla_append_fp8_absorb_q -- device. mla_cache_append_fp8 and mla_absorb_q of
 * one decode step in one launch, as mla_append_absorb_q is for the bf16
 * cache: the same results as the two calls in that order; the cache arguments
 * are those of mla_cache_append_fp8, the query arguments those of
 * mla_absorb_q. Errors: as the two calls.
 */
mla_status_t mla_append_fp8_absorb_q(uint8_t *cache, float *scales, int num_pages,
                                     const int32_t *block_table, int batch, int max_pages,
                                     const int32_t *seq_idx, const int32_t *tok_pos,
                                     const mla_bf16_t *c_kv, int ld_c, const mla_bf16_t *k_pe,
                                     int ld_k, int n_tokens, const mla_bf16_t *q_nope, int ld_qn,
                                     const mla_bf16_t *q_pe, int ld_qp, const mla_bf16_t *w_uk,
                                     const int32_t *q_pos, const float *rope_table, int max_pos,
                                     int T, int n_h, mla_bf16_t *q_full, uint32_t *status,
                                     mla_stream_t stream);
mla_status_t mla_decode_attention_fp8(const mla_bf16_t *q_full, const uint8_t *cache,
                                      const float *scales, int num_pages,
                                      const int32_t *block_table, int max_pages, int batch,
                                      int q_len, int n_h, float scale, const void *plan_host,
                                      const void *plan_dev, void *workspace,
                                      size_t workspace_bytes, mla_bf16_t *o_latent,
                                      float *lse, uint32_t *status, mla_stream_t stream);

/*
 * mla_out_absorb -- device. Expands the latent attention output through W^UV:
 *   u[t][h*128 + d] = sum_c o_latent[t][h][c] * w_uv[h][d][c]
 * ("DeepSeek-V3 MLA ... Guide", "The Matrix Absorption Trick", part 3:
 * u_i = W^UV_i o_i; "Step 3", einsum 'bnc,nhc->bnh').
 *   o_latent: device bf16 [T][n_h][512].
 *   w_uv:     device bf16 [n_h][128][512].
 *   u:        device bf16, row t at u + t*ld_u (n_h*128 elements), written.
 * fp32 accumulation, one bf16 rounding per output element.
 */
mla_status_t mla_out_absorb(const mla_bf16_t *o_latent, const mla_bf16_t *w_uv, int T,
                            int n_h, mla_bf16_t *u, int ld_u, mla_stream_t stream);

/*
 * mla_gemm_bf16 -- device. Plain projection GEMM used by the decode layer
 * (W^DQ, [W^UQ|W^QR], [W^DKV|W^KR], W^O; "DeepSeek-V3 MLA ... Guide",
 * "Core Architecture & Mathematics" sections 1-2, and the output projection):
 *   C[m][n] = sum_k X[m][k] * W[n][k]
 *   X: device bf16 [M][K], row stride ld_x.  W: device bf16 [N][K] (nn.Linear
 *   layout), row stride ld_w.  C: device, row stride ld_c, bf16 if c_fp32 == 0
 *   else float32. fp32 accumulation.
 */
mla_status_t mla_gemm_bf16(const mla_bf16_t *X, int ld_x, const mla_bf16_t *W, int ld_w,
                           void *C, int ld_c, int c_fp32, int M, int N, int K,
                           mla_stream_t stream);

/*
 * mla_gemm_bf16_ws -- device. mla_gemm_bf16 with a caller workspace: when
 * the output has few tiles and K is long (the down-projections from the
 * 7168-wide hidden state, the output projection), the reduction is split over
 * K across more CTAs. For a bf16 output the fp32 sums accumulate in the
 * workspace (zeroed by the call) and one more kernel rounds them to bf16 into
 * C; for an fp32 output each split writes its own partial tile into the
 * workspace (no atomics, so the result does not depend on the order the CTAs
 * finish in) and one more kernel adds them into C. Same result as
 * mla_gemm_bf16 up to the order of the fp32 additions.
 *   workspace: device, 16-byte aligned, >= mla_gemm_bf16_workspace_bytes(M,
 *              N, K) bytes (the larger of the two uses; it depends on the
 *              current device's SM count), or NULL (then exactly
 *              mla_gemm_bf16).
 * The workspace must not be in use by another call running at the same time.
 */
size_t mla_gemm_bf16_workspace_bytes(int M, int N, int K);
mla_status_t mla_gemm_bf16_ws(const mla_bf16_t *X, int ld_x, const mla_bf16_t *W, int ld_w,
                              void *C, int ld_c, int c_fp32, int M, int N, int K,
                              void *workspace, size_t workspace_bytes, mla_stream_t stream);

/*
 * Folded weights ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide", "The
 * Matrix Absorption Trick", parts 2-3: W^UK folded into the query side and
 * W^UV pre-multiplied into the output projection; "Deconstructing DeepSeek V4
 * Pro ...", "Practical Deployment & Systems Engineering Takeaways": the
 * query/key up-projection product pre-computed once). Computed once per
 * weight set; fp32 accumulation, one bf16 rounding per folded element.
 *
 * mla_fold_qk -- device.
 *   W~QK[h*512 + c][i] = sum_d w_uq[(h*128 + d)*ld_uq + i] * w_uk[h][d][c]
 *   w_uq: device bf16 [n_h*128][ld_uq] (W^UQ, or W_Q of a layer without a
 *         query latent), q_in input features (q_in % 64 == 0).
 *   w_uk: device bf16 [n_h][128][512].
 *   w_qk: device bf16 [n_h*512][q_in], written.
 *   workspace: device, >= mla_fold_qk_workspace_bytes(n_h) (holds W^UK with
 *              d contiguous), not in use by another call at the same time.
 * mla_fold_o -- device.
 *   W~O[f][h*512 + c] = sum_d w_o[f*ld_o + h*128 + d] * w_uv[h][d][c]
 *   w_o: device bf16 [d_model][ld_o] (W^O, n_h*128 input features).
 *   w_uv: device bf16 [n_h][128][512].  w_o_folded: device bf16 [d_model][n_h*512].
 *   The output projection then runs as mla_gemm_bf16 of o_latent viewed as
 *   [T][n_h*512] against W~O (K = n_h*512), with no mla_out_absorb.
 * mla_absorb_q_folded -- device. The query absorption from the folded weight:
 *   q_full[t][h][0:512]   = sum_i W~QK[h*512 + c][i] * x[t*ld_x + i]
 *   q_full[t][h][512:576] = RoPE(q_pe[t][h][:], pos[t])   (a copy if pos == NULL)
 *   x: device bf16, the query input (c^Q, or h without a query latent), k_in
 *      features (k_in % 64 == 0). Other arguments as mla_absorb_q.
 * Supported: n_h <= 128 (absorb: 16..128, multiple of 16).
 * Errors: INVALID_ARGUMENT, UNSUPPORTED, WORKSPACE_TOO_SMALL, CUDA.
 */
size_t mla_fold_qk_workspace_bytes(int n_h);
mla_status_t mla_fold_qk(const mla_bf16_t *w_uq, int ld_uq, int q_in, const mla_bf16_t *w_uk,
                         int n_h, mla_bf16_t *w_qk, void *workspace, size_t workspace_bytes,
                         mla_stream_t stream);
mla_status_t mla_fold_o(const mla_bf16_t *w_o, int ld_o, int d_model, const mla_bf16_t *w_uv,
                        int n_h, mla_bf16_t *w_o_folded, mla_stream_t stream);
mla_status_t mla_absorb_q_folded(const mla_bf16_t *x, int ld_x, int k_in, const mla_bf16_t *q_pe,
                                 int ld_qp, const mla_bf16_t *w_qk, const int32_t *pos,
                                 const float *rope_table, int max_pos, int T, int n_h,
                                 mla_bf16_t *q_full, uint32_t *status, mla_stream_t stream);

/*
 * mla_read_status -- host. Synchronises `stream`, copies the device status
 * word to *bits and, if clear != 0, zeroes it. Returns MLA_ERR_DEVICE if any
 * bit was set, MLA_OK otherwise.
 */
mla_status_t mla_read_status(uint32_t *status, uint32_t *bits, int clear,
                             mla_stream_t stream);

/* mla_check_status -- host. mla_read_status without clearing the word. */
mla_status_t mla_check_status(uint32_t *status, uint32_t *bits, mla_stream_t stream);

/*
 * mla_reset_status -- device. Zeroes the status word on `stream`
 * (cudaMemsetAsync); does not synchronise.
 */
mla_status_t mla_reset_status(uint32_t *status, mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */

// Absorbed MLA decode attention on CUDA cores (fp32 FMA, no tensor cores),
// and the log-sum-exp combine of split-KV partial results.
//
// This kernel is the plain GPU statement of the absorbed decode
// ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide", "The Matrix Absorption
// Trick", parts 2-4: scores on the cached latents plus the RoPE term, softmax,
// latent output). It serves as a second GPU implementation for differential
// tests of the tensor-core kernel; it is not the timed product path.
//
// One CTA = one work item x 16 heads. Per 64-token page: stage the page in
// shared memory, form 16 x 64 scores, update the running max / sum (base-2
// online softmax) and the 16 x 512 latent accumulators held in registers
// (thread -> one head x 32 latent dims).
#include <math.h>

#include "internal.h"

namespace mla {
namespace {

constexpr int kHeadsPerCta = 16;
constexpr int kThreads = 256;
constexpr int kTileStride = MLA_ROW + 8;  // 1168 B rows: conflict-free 16-byte accesses

struct SimtSmem {
  float q[kHeadsPerCta][MLA_ROW];
  uint16_t tile[MLA_PAGE][kTileStride];
  float p[kHeadsPerCta][MLA_PAGE];
  float alpha[kHeadsPerCta];
  float m[kHeadsPerCta];
  float l[kHeadsPerCta];
  int page_ok;
};

__global__ void __launch_bounds__(kThreads)
decode_simt_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem &sm = *reinterpret_cast<SimtSmem *>(smem_raw);
  const PlanHeader *ph = reinterpret_cast<const PlanHeader *>(a.plan_dev);
  const WorkItem it = reinterpret_cast<const WorkItem *>(a.plan_dev + ph->items_off)[blockIdx.x];
  const int h0 = blockIdx.y * kHeadsPerCta;
  const int tid = threadIdx.x;
  const int n_h = a.n_h;

  // query rows of heads h0..h0+15 (fp32)
  const uint16_t *qsrc = a.q_full + (((size_t)it.b * a.q_len + it.j) * n_h + h0) * MLA_ROW;
  for (int i = tid; i < kHeadsPerCta * MLA_ROW; i += kThreads)
    sm.q[i / MLA_ROW][i % MLA_ROW] = bf16_bits_to_f32(qsrc[i]);
  if (tid < kHeadsPerCta) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  const int my_h = tid >> 4;          // head (within the 16) of the accumulator
  const int my_d = (tid & 15) * 32;   // first latent dim of the accumulator
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;

  for (int pg = it.page_begin; pg < it.page_end; ++pg) {
    __syncthreads();  // previous page fully consumed
    if (tid == 0) {
      int page = -1;
      if (pg < a.max_pages) page = a.block_table[(size_t)it.b * a.max_pages + pg];
      const int ok = page >= 0 && page < a.num_pages;
      if (!ok) report(a.status, MLA_DEV_BAD_PAGE);
      sm.page_ok = ok ? page : -1;
    }
    __syncthreads();
    const int page = sm.page_ok;
    if (page < 0) continue;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.cache + (size_t)page * MLA_PAGE * MLA_ROW);
    for (int i = tid; i < MLA_PAGE * (MLA_ROW / 8); i += kThreads) {
      const int r = i / (MLA_ROW / 8), c = i % (MLA_ROW / 8);
      *reinterpret_cast<uint4 *>(&sm.tile[r][c * 8]) = __ldg(src + i);
    }
    __syncthreads();
    // scores: thread -> token r, heads 4*(tid/64) .. +3
    {
      const int r = tid & 63;
      const int hq = (tid >> 6) * 4;
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c = 0; c < MLA_ROW; c += 8) {
        const uint4 v = *reinterpret_cast<const uint4 *>(&sm.tile[r][c]);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = bf16_bits_to_f32(w[e] & 0xFFFFu), x1 = bf16_bits_to_f32(w[e] >> 16);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            s[k] = fmaf(sm.q[hq + k][c + 2 * e], x0, s[k]);
            s[k] = fmaf(sm.q[hq + k][c + 2 * e + 1], x1, s[k]);
          }
        }
      }
      const int tok = pg * MLA_PAGE + r;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        sm.p[hq + k][r] = tok <= it.qpos ? s[k] * a.scale_log2 : -INFINITY;
    }
    __syncthreads();
    // online softmax (base 2), one thread per head
    if (tid < kHeadsPerCta) {
      float mx = sm.m[tid];
      for (int r = 0; r < MLA_PAGE; ++r) mx = fmaxf(mx, sm.p[tid][r]);
      const float al = exp2f(sm.m[tid] - mx);  // m = -inf on the first page -> 0
      float sum = 0.f;
      for (int r = 0; r < MLA_PAGE; ++r) {
        const float e = exp2f(sm.p[tid][r] - mx);
        sm.p[tid][r] = e;
        sum += e;
      }
      sm.l[tid] = sm.l[tid] * al + sum;
      sm.m[tid] = mx;
      sm.alpha[tid] = al;
    }
    __syncthreads();
    {
      const float al = sm.alpha[my_h];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] *= al;
      for (int r = 0; r < MLA_PAGE; ++r) {
        const float pr = sm.p[my_h][r];
        const uint4 *row = reinterpret_cast<const uint4 *>(&sm.tile[r][my_d]);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 v = row[q4];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[q4 * 8 + 2 * e] = fmaf(pr, bf16_bits_to_f32(w[e] & 0xFFFFu), acc[q4 * 8 + 2 * e]);
            acc[q4 * 8 + 2 * e + 1] = fmaf(pr, bf16_bits_to_f32(w[e] >> 16), acc[q4 * 8 + 2 * e + 1]);
          }
        }
      }
    }
  }
  __syncthreads();
  const int h = h0 + my_h;
  const float l = sm.l[my_h];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float lse = l > 0.f ? (sm.m[my_h] + log2f(l)) * 0.69314718055994531f : -INFINITY;
  if (it.slot < 0) {
    uint16_t *dst = a.o_latent + (((size_t)it.b * a.q_len + it.j) * n_h + h) * MLA_D_C + my_d;
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<uint4 *>(dst)[i] =
          make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    if (a.lse != nullptr && (tid & 15) == 0)
      a.lse[((size_t)it.b * a.q_len + it.j) * n_h + h] = lse;
  } else {
    float *dst = a.ws_o + ((size_t)it.slot * n_h + h) * MLA_D_C + my_d;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      reinterpret_cast<float4 *>(dst)[i] =
          make_float4(acc[4 * i] * inv, acc[4 * i + 1] * inv, acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
    if ((tid & 15) == 0) a.ws_lse[(size_t)it.slot * n_h + h] = lse;
  }
}

// Log-sum-exp merge of the parts of one (sequence, query): one CTA of 128
// threads per (combine item, head), 4 latent dims per thread. Parts are read
// eight at a time (their lse and float4 slices issued before any is used), so
// a thread keeps eight loads in flight instead of waiting on one per part.
constexpr int kCombineBatch = 8;

__global__ void __launch_bounds__(128)
combine_kernel(DecodeArgs a) {
  const PlanHeader *ph = reinterpret_cast<const PlanHeader *>(a.plan_dev);
  const CombineItem ci = reinterpret_cast<const CombineItem *>(a.plan_dev + ph->combine_off)[blockIdx.x];
  const int h = blockIdx.y;
  const int n_h = a.n_h;
  const float *lse_base = a.ws_lse + (size_t)ci.first_slot * n_h + h;
  float mx = -INFINITY;
  for (int s0 = 0; s0 < ci.n_parts; s0 += kCombineBatch) {
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u)
      if (s0 + u < ci.n_parts) mx = fmaxf(mx, __ldg(lse_base + (size_t)(s0 + u) * n_h));
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  for (int s0 = 0; s0 < ci.n_parts; s0 += kCombineBatch) {
    float ls[kCombineBatch];
    float4 v[kCombineBatch];
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) {
      if (s0 + u >= ci.n_parts) continue;
      const size_t slot = (size_t)(ci.first_slot + s0 + u);
      ls[u] = __ldg(lse_base + (size_t)(s0 + u) * n_h);
      v[u] = __ldg(reinterpret_cast<const float4 *>(a.ws_o + (slot * n_h + h) * MLA_D_C) +
                   threadIdx.x);
    }
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) {
      if (s0 + u >= ci.n_parts) continue;
      const float w = (ls[u] == -INFINITY) ? 0.f : expf(ls[u] - mx);
      wsum += w;
      acc.x = fmaf(w, v[u].x, acc.x);
      acc.y = fmaf(w, v[u].y, acc.y);
      acc.z = fmaf(w, v[u].z, acc.z);
      acc.w = fmaf(w, v[u].w, acc.w);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const size_t row = ((size_t)ci.b * a.q_len + ci.j) * n_h + h;
  uint2 out;
  out.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  out.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2 *>(a.o_latent + row * MLA_D_C)[threadIdx.x] = out;
  if (a.lse != nullptr && threadIdx.x == 0)
    a.lse[row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace

mla_status_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream) {
  const int n_items = a.plan_host->num_items;
  if (n_items == 0) return MLA_OK;
  const size_t smem = sizeof(SimtSmem);
  MLA_CUDA_TRY(cudaFuncSetAttribute(decode_simt_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid(n_items, a.n_h / kHeadsPerCta);
  decode_simt_kernel<<<grid, kThreads, smem, stream>>>(a);
  MLA_LAUNCH_CHECK("decode_simt_kernel");
  return MLA_OK;
}

mla_status_t launch_combine(const DecodeArgs &a, cudaStream_t stream) {
  const int n = a.plan_host->num_combine;
  if (n == 0) return MLA_OK;
  dim3 grid(n, a.n_h);
  combine_kernel<<<grid, 128, 0, stream>>>(a);
  MLA_LAUNCH_CHECK("combine_kernel");
  return MLA_OK;
}

}  // namespace mla

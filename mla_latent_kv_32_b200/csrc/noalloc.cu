// mla_decode_attention_noalloc: the decode attention call for callers that
// cannot hand the library a workspace.
//
// Some callers cannot allocate device memory of their own when they call us:
// serving engines that reserve nearly all GPU memory up front for their own
// cache pool and hand out nothing else, and plugins running inside another
// framework's runtime, whose allocator they do not own and whose memory
// accounting an extra cudaMalloc would bypass. For them the split-KV partial
// results live in one fixed array in this library's own device memory instead
// of in a caller-supplied workspace.
//
// The array (kNoAllocScratchBytes, 48 MiB) exists on every GPU that loads the
// library and stays allocated until the process exits. Its device address is
// looked up once per device, on the first call made on that device, with that
// device current; make that first call before any stream capture begins. The
// address is kept per device index for the life of the process, so it goes
// stale if that device is reset (cudaDeviceReset) and the library used again.
//
// All calls share the array and it keeps whatever the previous call left in
// it. Nothing in it has to start at zero: every partial-result slot a call
// reads is written earlier in the same call. Two calls that may run at the
// same time on the GPU (different streams, different host threads) race on
// the array and corrupt each other's results; serialise them.
#include <mutex>

#include "internal.h"

namespace mla {
namespace {

constexpr size_t kNoAllocScratchBytes = 48ull << 20;
constexpr int kMaxDevices = 64;

// File-scope scratch. In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

mla_status_t scratch_address(void **out) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(MLA_ERR_CUDA, "cudaGetSymbolAddress of the scratch array on device %d: %s", dev,
                  cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" mla_status_t mla_decode_attention_noalloc(
    const mla_bf16_t *q_full, const mla_bf16_t *cache, int num_pages,
    const int32_t *block_table, int max_pages, int batch, int q_len, int n_h, float scale,
    const void *plan_host, const void *plan_dev, mla_bf16_t *o_latent, float *lse,
    uint32_t *status, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(plan_host != nullptr, "plan_host is NULL");
  const PlanHeader *ph = static_cast<const PlanHeader *>(plan_host);
  MLA_CHECK_ARG(ph->magic == kPlanMagic && ph->version == kPlanVersion, "not a decode plan");
  const size_t need = workspace_bytes(ph->num_partials, ph->n_h);
  if (need > kNoAllocScratchBytes)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL,
                "the plan needs %zu bytes of partial-result scratch but the built-in array "
                "holds %zu bytes; build the plan with fewer splits (e.g. max_split = 1) or "
                "use mla_decode_attention with a workspace",
                need, kNoAllocScratchBytes);
  void *scratch = nullptr;
  if (ph->num_partials > 0) {
    mla_status_t st = scratch_address(&scratch);
    if (st != MLA_OK) return st;
  }
  return mla_decode_attention(q_full, cache, num_pages, block_table, max_pages, batch, q_len, n_h,
                              scale, plan_host, plan_dev, scratch,
                              scratch ? kNoAllocScratchBytes : 0, o_latent, lse, status, stream);
}

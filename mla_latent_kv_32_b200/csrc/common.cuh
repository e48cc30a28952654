// Shared host/device helpers of the MLA decode library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "mla.h"

namespace mla {

// ------------------------------------------------------------------ host ---

// Records a message for mla_last_error() on this thread and returns `st`.
mla_status_t fail(mla_status_t st, const char *fmt, ...);
// Clears the per-thread message (called at the start of every entry point).
void clear_error();

#define MLA_CHECK_ARG(cond, ...)                                   \
  do {                                                             \
    if (!(cond)) return ::mla::fail(MLA_ERR_INVALID_ARGUMENT, __VA_ARGS__); \
  } while (0)

#define MLA_CUDA_TRY(expr)                                                   \
  do {                                                                       \
    cudaError_t e_ = (expr);                                                 \
    if (e_ != cudaSuccess)                                                   \
      return ::mla::fail(MLA_ERR_CUDA, "%s: %s (%s:%d)", #expr,              \
                         cudaGetErrorString(e_), __FILE__, __LINE__);        \
  } while (0)

// Launch-error check after a <<<>>> or cudaLaunchKernelEx.
#define MLA_LAUNCH_CHECK(what)                                               \
  do {                                                                       \
    cudaError_t e_ = cudaGetLastError();                                     \
    if (e_ != cudaSuccess)                                                   \
      return ::mla::fail(MLA_ERR_CUDA, "launch of %s failed: %s", what,      \
                         cudaGetErrorString(e_));                            \
  } while (0)

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SM count and compute capability of the current device (cached per device).
mla_status_t device_info(int *num_sms, int *cc_major, int *cc_minor);

// ---------------------------------------------------------------- device ---

__device__ __forceinline__ void report(uint32_t *status, uint32_t bit) {
  if (status != nullptr) atomicOr(status, bit);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
  return __uint_as_float(b16 << 16);
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return static_cast<uint32_t>(*reinterpret_cast<uint16_t *>(&h));
}

// Two floats -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return f32_to_bf16_bits(lo) | (f32_to_bf16_bits(hi) << 16);
}

// Rotation of one interleaved pair in float32 with each product and each sum
// rounded once (no fused multiply-add):
//   y0 = x0*c - x1*s,  y1 = x1*c + x0*s
__device__ __forceinline__ void rope_pair_rn(float x0, float x1, float c, float s,
                                             float &y0, float &y1) {
  y0 = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
  y1 = __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
}

}  // namespace mla

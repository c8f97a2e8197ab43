// Shared device helpers for liblcvq (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lcvq.h"

namespace lcvq {

constexpr int kWarp = 32;
constexpr int kNumSMsB200 = 148;

// Workspace header: the first 256 bytes of every workspace.
//   err   - first device-side error code (0 = none), set with atomicCAS
//   site  - which wait gave up (a small integer naming the wait)
//   wait_limit - bounded waits give up after this many clock cycles
//           (0 = kDefaultWaitLimit); a caller may lower it
struct WsHeader {
  unsigned int err;
  unsigned int site;
  long long wait_limit;
  unsigned int pad[60];
};
constexpr size_t kWsHeaderBytes = 256;
constexpr long long kDefaultWaitLimit = 1LL << 32;  // clock cycles (~2 s)

// the wait limit of the workspace whose header err_word points to
__device__ __forceinline__ long long wait_limit(const unsigned int* err_word) {
  if (err_word == nullptr) return kDefaultWaitLimit;
  const long long v = *reinterpret_cast<const volatile long long*>(err_word + 2);
  return v > 0 ? v : kDefaultWaitLimit;
}

__device__ __forceinline__ void record_error(unsigned int* err_word, unsigned int code,
                                             unsigned int site) {
  if (err_word != nullptr) {
    if (atomicCAS(err_word, 0u, code) == 0u) err_word[1] = site;
  }
}

// ---- bf16 <-> fp32 (round to nearest even) ----
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return uint32_t(f32_to_bf16(lo)) | (uint32_t(f32_to_bf16(hi)) << 16);
}

// ---- the 2-bit code of one proxy weight: clamp(rint(w), 0, 3); NaN -> 0 ----
__device__ __forceinline__ uint32_t code_of(float w) {
  // fmaxf returns the non-NaN operand, so NaN maps to 0; rintf rounds half to even.
  return static_cast<uint32_t>(fminf(fmaxf(rintf(w), 0.0f), 3.0f));
}
// STE pass region 0 <= w <= 3 (false for NaN).
__device__ __forceinline__ uint32_t in_mask(float w) { return (w >= 0.0f) & (w <= 3.0f); }

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- loads of data that an earlier kernel on the stream may have written ----
// Kernels launched with programmatic dependent launch can become resident
// before their producer has written, so such data is not constant over the
// kernel's lifetime and may not be read through the read-only path
// (ld.global.nc: __ldg, or what the compiler makes of const __restrict__
// pointers), which can return a line that an earlier kernel left in this SM's
// L1.  Ordinary global loads issued after griddepcontrol.wait see the
// producer's writes.  These are volatile so that they stay after that wait.
__device__ __forceinline__ uint4 ld_global_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_global_f32(const float* p) {
  float v;
  asm volatile("ld.global.f32 %0, [%1];\n" : "=f"(v) : "l"(p));
  return v;
}

}  // namespace lcvq

// Helpers of the decode-GEMV kernels (gemv.cu, gemv_tc.cu):
// the legacy tensor-core MMA they use for few tokens, shared-memory vector
// loads, cp.async copies, programmatic dependent launch controls, and the K
// chunking of the code stream.
#pragma once

#include <stdint.h>

namespace lcvq {

// D += A B for one m16n8k16 tile: bf16 in, fp32 accumulate
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A B for one m16n8k32 tile: A unsigned bytes, B signed bytes, exact
// int32 accumulate (the int8 path: codes times the digits of X')
__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The four u8 registers of one 32-bit word of 2-bit codes for the int8 MMA:
// register p holds the codes of positions p, p + 4, p + 8, p + 12 (byte i =
// position 4 i + p), the order of the int8 digit planes of X'.
__device__ __forceinline__ void dec_word_u8(uint32_t w, uint32_t (&r)[4]) {
  r[0] = w & 0x03030303u;
  r[1] = (w >> 2) & 0x03030303u;
  r[2] = (w >> 4) & 0x03030303u;
  r[3] = (w >> 6) & 0x03030303u;
}

// One chunk class's part of Y on the int8 path, added to the running sum of
// the classes (in class order): the exact integer sums of the codes times the
// hi and lo digits, (256 hi + lo), scaled by the class's 1 / s (a power of two)
__device__ __forceinline__ float i8_add_class(float sum, int hi, int lo, float inv_s) {
  return fmaf(fmaf(256.f, static_cast<float>(hi), static_cast<float>(lo)), inv_s, sum);
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

// A "unit" is 128 codes of a row (32 bytes); a chunk is kAhead units.
constexpr int kUnit = 128;
constexpr int kAhead = 4;

__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// 16-byte global -> shared copy through L2 only (zero-filled when !valid),
// and its commit / wait groups
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace lcvq

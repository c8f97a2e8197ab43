// The d = 8 decode W~ = A z + B as a small product on the tensor cores
// (mma.sync m16n8k16), shared by the materializing decode and the decode-form
// GEMM's decoder warps.
//
// 16 vectors are the rows of the MMA's A operand and the 8 output coordinates
// its columns,
//     W~[v][i] = B[i] + sum_k Aop[v][k] Bop[k][i],
// with k running over (code j, part):  k = 2t -> code t, hi;  k = 2t + 1 ->
// code t + 4, hi;  k = 2t + 8 -> code t, lo;  k = 2t + 9 -> code t + 4, lo
// (t = 0..3).  Aop[v][k] is the code z_v[j] as a bf16 (exact) and Bop[k][i] the
// hi or lo bf16 part of A[i][j] (hi = bf16(A), lo = bf16(A - hi): A to 2^-17),
// so the products are exact in fp32 and the accumulator starts at B[i]; a
// vector of zero codes gives B exactly.  A code becomes its bf16 value by one
// byte permute from two constant tables.  Lane (g, t) of the fragments needs
// codes t and t + 4 of vectors g and g + 8 (bits 2t and 2t + 8 of each 16-bit
// vector code) and gets back coordinates 2t, 2t + 1 of both vectors.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace lcvq {
namespace dec8 {

constexpr uint32_t kBf16CodeLo = 0x40008000u;  // low bytes of bf16 0, 1, 2, 3: 00 80 00 40
constexpr uint32_t kBf16CodeHi = 0x40403F00u;  // high bytes: 00 3F 40 40

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// bf16 pair (code t, code t + 4) of the vector whose 16-bit code starts at bit
// sh - 2t of `word`
__device__ __forceinline__ uint32_t code_pair_bf16(uint32_t word, uint32_t sh) {
  const uint32_t y = (word >> sh) & 0x0303u;  // code t at bits 0-1, code t + 4 at bits 8-9
  return prmt(kBf16CodeLo, kBf16CodeHi, y * 0x11u + 0x4040u);
}
// D = Aop Bop + C with the A registers repeated (k 8..15 are the lo parts of
// the same codes) and C = (B[2t], B[2t+1]) in both rows
__device__ __forceinline__ void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0,
                                    uint32_t b1, float c0, float c1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%4,%5}, "
      "{%6,%7}, {%8,%9,%8,%9};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0), "r"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// lane (g, t)'s B operand (column n = g: output coordinate g) and accumulator
// start, from A (8 x 8 row-major) and B (8)
__device__ __forceinline__ void operands(const float* A, const float* B, int g, int t,
                                         uint32_t& b0, uint32_t& b1, float& c0, float& c1) {
  const float x0 = A[g * 8 + t], x1 = A[g * 8 + t + 4];
  const uint16_t h0 = f32_to_bf16(x0), h1 = f32_to_bf16(x1);
  b0 = uint32_t(h0) | (uint32_t(h1) << 16);
  b1 = pack_bf16x2(x0 - bf16_to_f32(h0), x1 - bf16_to_f32(h1));
  c0 = B[2 * t];
  c1 = B[2 * t + 1];
}

}  // namespace dec8
}  // namespace lcvq

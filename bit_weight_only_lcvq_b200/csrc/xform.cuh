// The X-transform of one 16-element block of activations (xform.cu), and the
// fixed order of the corr sum.  See xform.cu for the
// algebra (the algebraic form of the forward, LC-QAT technical summary,
// Methodology 3) and the decoder order of X''.
//
// The per-row constant corr = s' - 3/2 sum bf16(X') - 128 sum X'' is summed in
// one fixed order everywhere: the K positions are cut into chunks of 512 (32
// blocks); a chunk's block values (fp32, from xform_block) are widened to fp64
// and summed by a warp-shuffle tree (lane l = block l of the chunk, lanes past
// the end of K contribute 0); chunk c's sum is added to the running sum of
// class c mod 8 in increasing c; the 8 class sums are added in class order;
// corr = fp32(s_b - 1.5 s_xr - 128 s_xpp).
#pragma once

#include "common.cuh"

namespace lcvq {

// X' of one 16-element block of activations, in fp32: x16 as two 16-byte
// words of bf16; sA: A (D x D, row-major, fp32); sBp: B' = B + 3/2 A 1.
//   xp[v d + j] = sum_i x[v d + i] A[i][j]   (fused multiply-adds in i order)
//   sb          = sum_{v, i} x[v d + i] B'[i]  (s' of the block, in v, i order)
template <int D>
__device__ __forceinline__ void xprime_block(const uint4& u0, const uint4& u1,
                                             const float* __restrict__ sA,
                                             const float* __restrict__ sBp, float (&xp)[16],
                                             float& sb) {
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
  float x[16];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    x[2 * q] = bf16_lo(w[q]);
    x[2 * q + 1] = bf16_hi(w[q]);
  }
  sb = 0.f;
#pragma unroll
  for (int v = 0; v < 16 / D; ++v) {
#pragma unroll
    for (int j = 0; j < D; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) acc = fmaf(x[v * D + i], sA[i * D + j], acc);
      xp[v * D + j] = acc;
    }
#pragma unroll
    for (int i = 0; i < D; ++i) sb = fmaf(x[v * D + i], sBp[i], sb);
  }
}

// One 16-element block of the bf16 transform.  Writes the block's X'' in
// decoder order (o[c] = bf16x2 of positions c and c + 8, each scaled by
// 4^-(c mod 3)) and the block's parts of the per-row constant:
//   sb   = sum x^T B'           (s')
//   sxr  = sum bf16(X')         (X'r)
//   sxpp = sum X''
template <int D>
__device__ __forceinline__ void xform_block(const uint4& u0, const uint4& u1,
                                            const float* __restrict__ sA,
                                            const float* __restrict__ sBp, uint32_t (&o)[8],
                                            float& sb, float& sxr, float& sxpp) {
  float xrd[16];  // X', then bf16(X') as fp32
  xprime_block<D>(u0, u1, sA, sBp, xrd, sb);
  sxr = 0.f;
#pragma unroll
  for (int v = 0; v < 16 / D; ++v)
#pragma unroll
    for (int j = 0; j < D; ++j) {
      xrd[v * D + j] = bf16_to_f32(f32_to_bf16(xrd[v * D + j]));
      sxr += xrd[v * D + j];
    }
  sxpp = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float scale = (c % 3 == 0) ? 1.0f : ((c % 3 == 1) ? 0.25f : 0.0625f);
    const float lo = xrd[c] * scale;
    const float hi = xrd[c + 8] * scale;
    sxpp += lo + hi;
    o[c] = pack_bf16x2(lo, hi);  // exact: power-of-two scaling of bf16 values
  }
}

// B'[i] = B[i] + 3/2 sum_j A[i][j], summed in j order (thread i < D)
template <int D>
__device__ __forceinline__ float shifted_offset(const float* __restrict__ A_row, float b) {
  float rs = 0.f;
#pragma unroll
  for (int j = 0; j < D; ++j) rs += A_row[j];
  return b + 1.5f * rs;
}



// the warp-shuffle tree of one chunk's block values (result in lane 0)
__device__ __forceinline__ double chunk_tree_sum(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  return v;
}

constexpr int kCorrChunk = 512;  // positions per chunk of the corr sum
constexpr int kCorrClasses = 8;  // chunk classes (c mod 8)

}  // namespace lcvq

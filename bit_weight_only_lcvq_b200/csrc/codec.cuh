// The one-instruction decoder of 2-bit codes into bf16 pairs, shared by every
// kernel that multiplies raw codes on the tensor cores (the algebraic form of
// the forward: the X-transform folds A, B, the 128 offset and the powers of
// two into X'' and corr, see xform.cu).
//
// A 32-bit word holds 16 codes (format V1: code e at bits 2e, 2e + 1).  Pair c
// (c = 0..7) is the bf16x2 (128 + 4^p z_c, 128 + 4^p z_{c+8}), p = c mod 3: one
// LOP3 masks the two codes into mantissa bits 2p .. 2p + 1 of each half of
// 0x4300_4300 (bf16 128.0, 128.0).  Pairs 0..2 read the word itself, 3..5 the
// word shifted right by 6 and 6..7 by 12, so that code c lands at bit 2p.
#pragma once

#include <stdint.h>

namespace lcvq {

template <int C>
__device__ __forceinline__ uint32_t dec_pair(uint32_t w0, uint32_t w6, uint32_t w12) {
  constexpr int P = C % 3;
  const uint32_t src = (C < 3) ? w0 : ((C < 6) ? w6 : w12);
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n"  // (a & b) | c
      : "=r"(r)
      : "r"(src), "n"(0x00030003u << (2 * P)), "n"(0x43004300u));
  return r;
}

// dec_pair<c> for a c that is a compile-time constant after unrolling
__device__ __forceinline__ uint32_t dec_pair_rt(int c, uint32_t w0, uint32_t w6, uint32_t w12) {
  switch (c) {
    case 0: return dec_pair<0>(w0, w6, w12);
    case 1: return dec_pair<1>(w0, w6, w12);
    case 2: return dec_pair<2>(w0, w6, w12);
    case 3: return dec_pair<3>(w0, w6, w12);
    case 4: return dec_pair<4>(w0, w6, w12);
    case 5: return dec_pair<5>(w0, w6, w12);
    case 6: return dec_pair<6>(w0, w6, w12);
    default: return dec_pair<7>(w0, w6, w12);
  }
}

// all 8 pairs of one word, in decoder order
__device__ __forceinline__ void dec_word8(uint32_t w, uint32_t* o) {
  const uint32_t w6 = w >> 6, w12 = w >> 12;
  o[0] = dec_pair<0>(w, w6, w12);
  o[1] = dec_pair<1>(w, w6, w12);
  o[2] = dec_pair<2>(w, w6, w12);
  o[3] = dec_pair<3>(w, w6, w12);
  o[4] = dec_pair<4>(w, w6, w12);
  o[5] = dec_pair<5>(w, w6, w12);
  o[6] = dec_pair<6>(w, w6, w12);
  o[7] = dec_pair<7>(w, w6, w12);
}

// the same as two 16-byte chunks (pairs 0..3 and 4..7)
__device__ __forceinline__ void dec_word(uint32_t w, uint4& c0, uint4& c1) {
  uint32_t o[8];
  dec_word8(w, o);
  c0 = make_uint4(o[0], o[1], o[2], o[3]);
  c1 = make_uint4(o[4], o[5], o[6], o[7]);
}

}  // namespace lcvq

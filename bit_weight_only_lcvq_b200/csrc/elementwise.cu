// Code assignment + 2-bit packing, and decode (materialization of A z + B).
//
// Both are streaming, HBM-bound kernels:
//   assign_pack reads 4 B and writes 0.25 B (+0.125 B of mask) per weight;
//   decode reads 0.25 B and writes 2 B (bf16) or 4 B (fp32) per weight.
#include <math.h>

#include "common.cuh"
#include "decode_mma.cuh"
#include "internal.h"

namespace lcvq {

// ---------------------------------------------------------------------------
// assign + pack (LC-QAT technical summary, Methodology 1 and 3: proxy weights
// rounded and clamped to 2-bit integer codes).
//
// The matrix is handled as a flat array (rows are contiguous and d_in % 8 == 0,
// so the flat order is the row order).  A warp owns chunks of 128 weights:
// lane l loads the float4 of weights 4l..4l+3 (one 128-bit load, 512 B per warp
// instruction, fully coalesced), turns it into one byte of codes and a nibble
// of mask bits, and warp shuffles gather 4 lanes' bytes into one 32-bit store
// and 8 lanes' nibbles into one 32-bit mask store.
// ---------------------------------------------------------------------------
constexpr int kApUnroll = 4;  // chunks per warp iteration (independent loads in flight)

__device__ __forceinline__ void ap_codes(const float4 v, uint32_t& byte, uint32_t& nib) {
  byte = code_of(v.x) | (code_of(v.y) << 2) | (code_of(v.z) << 4) | (code_of(v.w) << 6);
  nib = in_mask(v.x) | (in_mask(v.y) << 1) | (in_mask(v.z) << 2) | (in_mask(v.w) << 3);
}

__global__ void __launch_bounds__(256) assign_pack_kernel(const float4* __restrict__ wp,
                                                          int64_t n_chunks, int tail_floats,
                                                          uint8_t* __restrict__ packed,
                                                          uint8_t* __restrict__ mask) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const unsigned full = 0xffffffffu;

  for (int64_t base = gw * kApUnroll; base < n_chunks; base += nw * kApUnroll) {
    float4 v[kApUnroll];
#pragma unroll
    for (int u = 0; u < kApUnroll; ++u) {
      const int64_t c = base + u;
      if (c < n_chunks) v[u] = __ldcs(wp + c * 32 + lane);
    }
#pragma unroll
    for (int u = 0; u < kApUnroll; ++u) {
      const int64_t c = base + u;
      if (c >= n_chunks) break;  // warp-uniform
      uint32_t b, nib;
      ap_codes(v[u], b, nib);
      const uint32_t b1 = __shfl_down_sync(full, b, 1);
      const uint32_t b2 = __shfl_down_sync(full, b, 2);
      const uint32_t b3 = __shfl_down_sync(full, b, 3);
      if ((lane & 3) == 0) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(packed + c * 32) + (lane >> 2);
        __stcs(dst, b | (b1 << 8) | (b2 << 16) | (b3 << 24));
      }
      if (mask != nullptr) {
        const uint32_t x = nib | (__shfl_down_sync(full, nib, 1) << 4);
        const uint32_t y = x | (__shfl_down_sync(full, x, 2) << 8);
        const uint32_t w = y | (__shfl_down_sync(full, y, 4) << 16);
        if ((lane & 7) == 0) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(mask + c * 16) + (lane >> 3);
          __stcs(dst, w);
        }
      }
    }
  }

  // Ragged tail (< 128 weights, a multiple of 8): the first warp of the grid.
  if (tail_floats > 0 && gw == 0) {
    const int64_t c = n_chunks;
    const bool valid = 4 * lane < tail_floats;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid) v = wp[c * 32 + lane];
    uint32_t b, nib;
    ap_codes(v, b, nib);
    if (valid) packed[c * 32 + lane] = static_cast<uint8_t>(b);
    const uint32_t x = nib | (__shfl_down_sync(full, nib, 1) << 4);
    if (mask != nullptr && valid && (lane & 1) == 0) mask[c * 16 + (lane >> 1)] = static_cast<uint8_t>(x);
  }
}

cudaError_t launch_assign_pack(const float* Wp, int64_t n_elems, uint8_t* packed,
                               uint8_t* mask_bits, cudaStream_t s, int* launches) {
  const int64_t n_chunks = n_elems / 128;
  const int tail = static_cast<int>(n_elems % 128);
  const int64_t warps_needed = ceil_div(n_chunks, kApUnroll) + (tail ? 1 : 0);
  int64_t blocks = ceil_div(warps_needed, 8);
  // one wave of resident blocks (the loop strides over the rest): a grid of
  // more blocks than fit at once would end in a partly empty second wave
  static const int resident = [] {  // thread-safe one-time initialisation
    int r = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, assign_pack_kernel, 256, 0) !=
            cudaSuccess ||
        r < 1)
      r = 1;
    return r;
  }();
  const int64_t cap = int64_t(kNumSMsB200) * resident;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  assign_pack_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<const float4*>(Wp), n_chunks, tail, packed, mask_bits);
  ++*launches;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// decode (Methodology 1: c = A z + B; Methodology 3: A W_z + B).
// One thread per 32-bit word of codes = 16 consecutive weights of one row
// (d in {1,2,4,8} divides 16, and d_in % 16 == 0, so a word holds whole
// vectors).  A and B sit in shared memory; fp32 FMA in a fixed order.
// ---------------------------------------------------------------------------
template <int D, bool kBf16>
__global__ void __launch_bounds__(256) decode_kernel(const uint32_t* __restrict__ codes,
                                                     int64_t n_words, const float* __restrict__ A,
                                                     const float* __restrict__ B,
                                                     void* __restrict__ W) {
  __shared__ float sA[D * D];
  __shared__ float sB[D];
  for (int i = threadIdx.x; i < D * D; i += blockDim.x) sA[i] = A[i];
  for (int i = threadIdx.x; i < D; i += blockDim.x) sB[i] = B[i];
  __syncthreads();
  for (int64_t w = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; w < n_words;
       w += int64_t(gridDim.x) * blockDim.x) {
    const uint32_t word = __ldcs(codes + w);
    float out[16];
#pragma unroll
    for (int v = 0; v < 16 / D; ++v) {
      float z[D];
#pragma unroll
      for (int j = 0; j < D; ++j) z[j] = static_cast<float>((word >> (2 * (v * D + j))) & 3u);
#pragma unroll
      for (int i = 0; i < D; ++i) {
        float acc = sB[i];
#pragma unroll
        for (int j = 0; j < D; ++j) acc = fmaf(sA[i * D + j], z[j], acc);
        out[v * D + i] = acc;
      }
    }
    if constexpr (kBf16) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(W) + w * 16);
      uint4 o0, o1;
      o0.x = pack_bf16x2(out[0], out[1]);
      o0.y = pack_bf16x2(out[2], out[3]);
      o0.z = pack_bf16x2(out[4], out[5]);
      o0.w = pack_bf16x2(out[6], out[7]);
      o1.x = pack_bf16x2(out[8], out[9]);
      o1.y = pack_bf16x2(out[10], out[11]);
      o1.z = pack_bf16x2(out[12], out[13]);
      o1.w = pack_bf16x2(out[14], out[15]);
      __stcs(dst, o0);
      __stcs(dst + 1, o1);
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(W) + w * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        __stcs(dst + q, make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]));
    }
  }
}

// d = 8, bf16 output: the decode as a small product on the tensor cores
// (decode_mma.cuh).  This costs about 4 instructions per weight, where the FMA
// form (8 FMAs and an int-to-float conversion per weight) is ALU-bound below
// the store bandwidth.
constexpr int kDec8Groups = 4;                 // MMAs (16 vectors each) per warp and iteration

__global__ void __launch_bounds__(256) decode8_mma_kernel(const uint32_t* __restrict__ words,
                                                          int64_t n_vec,
                                                          const float* __restrict__ A,
                                                          const float* __restrict__ B,
                                                          uint16_t* __restrict__ W) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // B operand: column n = g is output coordinate g; rows 2t, 2t + 1 (hi) and
  // 2t + 8, 2t + 9 (lo) are A[g][t] and A[g][t + 4]
  uint32_t b0, b1;
  float c0, c1;
  dec8::operands(A, B, g, t, b0, b1, c0, c1);
  const uint32_t sh = 16u * (g & 1) + 2u * t;  // vector g of a group is half g & 1 of its word
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  constexpr int kPer = 16 * kDec8Groups;      // vectors per warp iteration
  const int64_t n_full = n_vec / kPer;
  // lane's pointers for iteration v0: the words of vectors v0 + 16m + g (+ 8),
  // and the output word of vector v0 + g, coordinates 2t, 2t + 1
  auto wsrc = [&](int64_t it) { return words + it * (kPer / 2) + (g >> 1); };
  auto wdst = [&](int64_t it) {
    return reinterpret_cast<uint32_t*>(W) + (it * kPer + g) * 4 + t;
  };
  int64_t it = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  uint32_t nxt[kDec8Groups][2];
  if (it < n_full) {
    const uint32_t* src = wsrc(it);
#pragma unroll
    for (int m = 0; m < kDec8Groups; ++m) nxt[m][0] = __ldcs(src + 8 * m), nxt[m][1] = __ldcs(src + 8 * m + 4);
  }
  for (; it < n_full; it += warps) {
    uint32_t cur[kDec8Groups][2];
#pragma unroll
    for (int m = 0; m < kDec8Groups; ++m) cur[m][0] = nxt[m][0], cur[m][1] = nxt[m][1];
    if (it + warps < n_full) {
      const uint32_t* src = wsrc(it + warps);
#pragma unroll
      for (int m = 0; m < kDec8Groups; ++m) nxt[m][0] = __ldcs(src + 8 * m), nxt[m][1] = __ldcs(src + 8 * m + 4);
    }
    uint32_t* dst = wdst(it);
#pragma unroll
    for (int m = 0; m < kDec8Groups; ++m) {
      float d[4];
      dec8::mma(d, dec8::code_pair_bf16(cur[m][0], sh), dec8::code_pair_bf16(cur[m][1], sh), b0, b1, c0, c1);
      __stcs(dst + 64 * m, dec8::bf16x2_rn(d[0], d[1]));
      __stcs(dst + 64 * m + 32, dec8::bf16x2_rn(d[2], d[3]));
    }
  }
  // the ragged tail (fewer than kPer vectors) goes to the warp whose turn it is
  if (it == n_full && n_full * kPer < n_vec) {
    const int64_t v0 = n_full * kPer;
    for (int m = 0; m < kDec8Groups; ++m) {
      const int64_t v1 = v0 + 16 * m + g, v2 = v1 + 8;
      const uint32_t w1 = v1 < n_vec ? words[v1 >> 1] : 0u;
      const uint32_t w2 = v2 < n_vec ? words[v2 >> 1] : 0u;
      float d[4];
      dec8::mma(d, dec8::code_pair_bf16(w1, sh), dec8::code_pair_bf16(w2, sh), b0, b1, c0, c1);
      if (v1 < n_vec) reinterpret_cast<uint32_t*>(W)[v1 * 4 + t] = dec8::bf16x2_rn(d[0], d[1]);
      if (v2 < n_vec) reinterpret_cast<uint32_t*>(W)[v2 * 4 + t] = dec8::bf16x2_rn(d[2], d[3]);
    }
  }
}

template <int D>
static void decode_dispatch_bf(const uint32_t* codes, int64_t n_words, const float* A,
                               const float* B, void* W, bool bf16, unsigned blocks,
                               cudaStream_t s) {
  if (bf16)
    decode_kernel<D, true><<<blocks, 256, 0, s>>>(codes, n_words, A, B, W);
  else
    decode_kernel<D, false><<<blocks, 256, 0, s>>>(codes, n_words, A, B, W);
}

cudaError_t launch_decode(const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                          const float* A, const float* B, void* W, bool w_bf16, cudaStream_t s,
                          int* launches) {
  const int64_t n_words = d_out * (d_in / 16);
  int64_t blocks = ceil_div(n_words, 256);
  const int64_t cap = int64_t(kNumSMsB200) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(packed);
  if (d == 8 && w_bf16) {
    const int64_t n_vec = d_out * (d_in / 8);
    int64_t b8 = ceil_div(ceil_div(n_vec, 16 * kDec8Groups), 8);
    // a persistent grid of resident blocks: each warp keeps its next batch
    // of codes (128 bytes) in flight while it decodes and stores the current one
    static const int resident = [] {  // thread-safe one-time initialisation
      int r = 0;
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, decode8_mma_kernel, 256, 0);
      return r > 0 ? r : 1;
    }();
    const int64_t cap8 = int64_t(kNumSMsB200) * resident;
    if (b8 > cap8) b8 = cap8;
    if (b8 < 1) b8 = 1;
    decode8_mma_kernel<<<static_cast<unsigned>(b8), 256, 0, s>>>(codes, n_vec, A, B,
                                                                   static_cast<uint16_t*>(W));
    ++*launches;
    return cudaGetLastError();
  }
  switch (d) {
    case 1: decode_dispatch_bf<1>(codes, n_words, A, B, W, w_bf16, unsigned(blocks), s); break;
    case 2: decode_dispatch_bf<2>(codes, n_words, A, B, W, w_bf16, unsigned(blocks), s); break;
    case 4: decode_dispatch_bf<4>(codes, n_words, A, B, W, w_bf16, unsigned(blocks), s); break;
    default: decode_dispatch_bf<8>(codes, n_words, A, B, W, w_bf16, unsigned(blocks), s); break;
  }
  ++*launches;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// DGE rescale (LC-QAT technical summary, Methodology 3: a differentiable
// gradient estimator through the rounding instead of the STE).  The pages give
// no curve; the reading here is the tanh staircase
//   phi_k(w) = floor(w) + 1/2 + tanh(k (frac(w) - 1/2)) / (2 tanh(k/2))  on [0, 3]
// whose derivative k / (2 tanh(k/2)) sech^2(k (frac - 1/2)) replaces the STE's
// clamp mask (0 outside [0, 3]; k -> 0 gives the mask back).  The STE
// gradient inside the mask is A^T G, so dWp_DGE = dWp_STE * phi_k'(Wp).
// 12 bytes per weight (dWp read and written, Wp read), float4 at a time.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float dge_factor(float w, float k, float ck) {
  if (!(w >= 0.f && w <= 3.f)) return 0.f;
  const float f = w - fminf(floorf(w), 2.f);
  const float t = tanhf(k * (f - 0.5f));
  return ck * (1.f - t * t);
}

__global__ void __launch_bounds__(256) dge_scale_kernel(float4* __restrict__ dWp,
                                                        const float4* __restrict__ Wp,
                                                        int64_t n4, float k, float ck) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 w = __ldcs(Wp + i);
    float4 g = __ldcs(dWp + i);
    g.x *= dge_factor(w.x, k, ck);
    g.y *= dge_factor(w.y, k, ck);
    g.z *= dge_factor(w.z, k, ck);
    g.w *= dge_factor(w.w, k, ck);
    __stcs(dWp + i, g);
  }
}

cudaError_t launch_dge_scale(float* dWp, const float* Wp, int64_t n, float k, cudaStream_t s,
                             int* launches) {
  const int64_t n4 = n / 4;
  int64_t blocks = ceil_div(n4, 256);
  const int64_t cap = int64_t(kNumSMsB200) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const double kd = k;
  const float ck = static_cast<float>(kd / (2.0 * tanh(kd / 2.0)));
  dge_scale_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<float4*>(dWp), reinterpret_cast<const float4*>(Wp), n4, k, ck);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace lcvq

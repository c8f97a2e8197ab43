// Decode-GEMV for few tokens (M <= 32): Y = X W~ with W~ = A z + B streamed as
// packed 2-bit codes (LC-QAT technical summary, Methodology 3: the forward runs
// on INT2 x FP16 matmul operators).
//
// The kernel multiplies the transformed activations X'' (see xform.cu) with the
// raw codes on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   * weights are the 16-row A operand, tokens the 8-column B operand, so a
//     weight tile is decoded once and serves every token;
//   * codes go from HBM straight into registers (one 128-bit load per row and
//     lane per 256 codes) and are decoded by a single LOP3 per bf16 pair:
//     (word >> s) & 0x00030003 << 2p | 0x43004300 = bf16x2(128 + 4^p z_lo,
//     128 + 4^p z_hi); the power of two and the 128 offset are folded into X''
//     and the per-row constant `corr`, so decoding costs no float arithmetic;
//   * the MMA's logical k of each lane is mapped onto the lane's own code
//     words (the decoder order of X'' makes the B fragments contiguous loads);
//   * a CTA owns 16 R rows over the whole K (8 warps split K, fixed-order
//     shared-memory sum), so no partial sum leaves the CTA and the result is
//     deterministic;
//   * programmatic dependent launch: the code loads do not depend on the
//     X-transform, so they are issued before griddepcontrol.wait and stream
//     while the prologue runs.  The kernel touches nothing else before the
//     wait, and the X-transform waits for every earlier kernel before it lets
//     this one launch, so the early reads never race a producer of the codes.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace lcvq {

namespace {

constexpr int kGemvRows = 128;   // weight rows per CTA

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 (128 + 4^p z_c, 128 + 4^p z_{c+8}) of pair c of a 16-code word, given
// the word and its shifts by 6 and 12.
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

// same as dec_pair<C> for a C that is a compile-time constant after unrolling
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

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

// CTA: kWarps warps on 16 R weight rows over the whole K, so no partial sum
// leaves the CTA.  Warp w takes K slice w.  A "unit" is 128 codes of each of the
// CTA's rows: lane (g, t) holds 2 words of rows g and g + 8 of every row
// block (8 B each); a warp keeps up to kAhead units of loads in flight.
// Launch order with the X-transform (programmatic dependent launch): the code
// loads are issued before griddepcontrol.wait, so they overlap the prologue;
// X'' and corr are read only after it.
constexpr int kUnit = 128;  // codes per row per unit (32 B)
constexpr int kAhead = 4;

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];\n"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

template <int NT, int R, int kWarps>
__global__ void __launch_bounds__(kWarps * 32, (kWarps == 16 ? 1 : (NT <= 2 ? 2 : 1)))
    gemv_kernel(const uint16_t* __restrict__ Xpp, const float* __restrict__ corr, int M,
                const uint8_t* __restrict__ packed, int64_t N, int64_t K,
                uint16_t* __restrict__ Y) {
  constexpr int MP = NT * 8;
  constexpr int ROWS = 16 * R;
  constexpr bool kPrefX = NT == 1;  // keep the next unit's X'' fragments in flight
  __shared__ float part[kWarps][ROWS][MP + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row0 = int64_t(blockIdx.x) * ROWS;
  const int64_t Kb = K / 4;
  const int64_t nunits = ceil_div(K, kUnit);
  const int64_t u0 = nunits * warp / kWarps, u1 = nunits * (warp + 1) / kWarps;

  const uint8_t* rowp[R][2];
  bool rowok[R][2];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t row = row0 + r * 16 + g + 8 * h;
      rowok[r][h] = row < N;
      rowp[r][h] = packed + (rowok[r][h] ? row : 0) * Kb + 8 * t;
    }

  auto load_unit = [&](int64_t u, uint2 (&cw)[R][2]) {
    const bool kok = u < u1 && u * kUnit + 32 * t < K;  // K % 64 == 0: whole lane chunks
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        cw[r][h] = (kok && rowok[r][h]) ? ld_stream_v2(rowp[r][h] + u * 32) : make_uint2(0, 0);
  };

  uint2 ring[kAhead][R][2];
#pragma unroll
  for (int j = 0; j < kAhead; ++j) load_unit(u0 + j, ring[j]);

  griddep_wait();  // X'' and corr written by the X-transform are visible from here

  const uint16_t* xrow[NT];
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok = n * 8 + g;
    tokok[n] = tok < M;
    xrow[n] = Xpp + int64_t(tokok[n] ? tok : 0) * K + 32 * t;
  }

  float acc[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

  // X'' fragments of one unit: word q, token tile n -> two 16-byte halves
  auto load_x = [&](int64_t u, uint4 (&xb)[2][NT][2]) {
    const bool kok = u < u1 && u * kUnit + 32 * t < K;
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (kok && tokok[n]) {
          const uint4* src = reinterpret_cast<const uint4*>(xrow[n] + u * kUnit + 16 * q);
          xb[q][n][0] = __ldg(src);
          xb[q][n][1] = __ldg(src + 1);
        } else {
          xb[q][n][0] = make_uint4(0, 0, 0, 0);
          xb[q][n][1] = make_uint4(0, 0, 0, 0);
        }
      }
  };
  uint4 xcur[2][NT][2], xnxt[2][NT][2];
  load_x(u0, xcur);

  for (int64_t base = u0; base < u1; base += kAhead) {
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int64_t u = base + j;
      if (u >= u1) break;
      if constexpr (kPrefX) load_x(u + 1, xnxt);
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // word q of each row: 16 codes, 4 k16 tiles
        uint32_t w0[R][2], w6[R][2], w12[R][2];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            w0[r][h] = q == 0 ? ring[j][r][h].x : ring[j][r][h].y;
            w6[r][h] = w0[r][h] >> 6;
            w12[r][h] = w0[r][h] >> 12;
          }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {  // k16 tile: pairs 2jj, 2jj+1 of word q
          uint32_t a[R][2][2];
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              a[r][h][0] = dec_pair_rt(2 * jj, w0[r][h], w6[r][h], w12[r][h]);
              a[r][h][1] = dec_pair_rt(2 * jj + 1, w0[r][h], w6[r][h], w12[r][h]);
            }
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint32_t b0 = word_of(xcur[q][n][jj >> 1], (2 * jj) & 3);
            const uint32_t b1 = word_of(xcur[q][n][jj >> 1], (2 * jj + 1) & 3);
#pragma unroll
            for (int r = 0; r < R; ++r)
              mma_bf16_16816(acc[r][n], a[r][0][0], a[r][1][0], a[r][0][1], a[r][1][1], b0, b1);
          }
        }
      }
      load_unit(u + kAhead, ring[j]);  // refill the slot just consumed
      if constexpr (kPrefX) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            xcur[q][n][0] = xnxt[q][n][0];
            xcur[q][n][1] = xnxt[q][n][1];
          }
      } else {
        load_x(u + 1, xcur);
      }
    }
  }

  // every CTA has passed its main loop: the next kernel may start launching
  griddep_launch_dependents();

#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int lr = r * 16 + g;
      const int tk = n * 8 + 2 * t;
      part[warp][lr][tk] = acc[r][n][0];
      part[warp][lr][tk + 1] = acc[r][n][1];
      part[warp][lr + 8][tk] = acc[r][n][2];
      part[warp][lr + 8][tk + 1] = acc[r][n][3];
    }
  __syncthreads();
  // sum the 8 K slices in slice order, add the per-row constant, store
  for (int e = threadIdx.x; e < ROWS * M; e += kWarps * 32) {
    const int lr = e % ROWS, tok = e / ROWS;
    const int64_t grow = row0 + lr;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sum += part[w][lr][tok];
    if (grow < N) Y[int64_t(tok) * N + grow] = f32_to_bf16(sum + corr[tok]);
  }
}

template <int NT, int R, int kWarps>
cudaError_t launch_gemv_t(const uint16_t* Xpp, const float* corr, int M, const uint8_t* packed,
                          int64_t N, int64_t K, uint16_t* Y, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(N, 16 * R)), 1, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, R, kWarps>, Xpp, corr, M, packed, N, K, Y);
}

// ---------------------------------------------------------------------------
// Single-kernel decode-GEMV (X-transform fused).  A thread-block cluster of S
// CTAs (grid y) splits K; each CTA owns 128 weight rows and one K slice, and
//   1. issues the code loads of its slice (they do not depend on X),
//   2. waits for the producer of X (programmatic dependent launch), then
//      transforms its slice of X into X'' in shared memory -- the same
//      arithmetic as xform.cu: X' = bf16(group-wise X A), scaled by 4^-p, in
//      decoder order -- and the slice's parts of the per-row constant,
//   3. runs the decode + mma.sync main loop with B fragments from shared memory,
//   4. sums the S partial tiles and constant parts in a fixed order through
//      distributed shared memory and stores Y.
// One launch per call, and X'' never goes through global memory.
constexpr int kFuRows = 128;

__host__ __device__ inline size_t round16(size_t x) { return (x + 15) & ~size_t(15); }
// byte offsets of the regions of the fused kernel's dynamic shared memory
__host__ __device__ inline size_t fused_smem_layout(int MP, int64_t slice_max, size_t& off_part,
                                                    size_t& off_corr, size_t& off_item) {
  off_part = round16(size_t(MP) * size_t(slice_max + 16) * 2);
  off_corr = round16(off_part + size_t(kFuRows) * (MP + 1) * 4);
  off_item = round16(off_corr + size_t(MP) * 8);
  return off_item + size_t(3) * MP * size_t(slice_max / 8) * 4;
}

template <int NT, int D>
__global__ void __launch_bounds__(256, 2) gemv_fused_kernel(
    const uint16_t* __restrict__ X, const float* __restrict__ A, const float* __restrict__ B,
    int M, const uint8_t* __restrict__ packed, int64_t N, int64_t K, int64_t slice_max,
    uint16_t* __restrict__ Y) {
  constexpr int MP = NT * 8;
  extern __shared__ __align__(16) uint8_t fsm[];
  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.dim_blocks().y);
  const int rank = static_cast<int>(cluster.block_index().y);
  // shared memory: X'' slice [MP][slice_max + 16 pad] bf16 | part [128][MP+1] f32 |
  //                corr parts [MP] f64 | item sums [3][MP][slice_max/8] f32
  const int64_t xpitch = slice_max + 16;  // elements; 32 B pad against bank conflicts
  size_t off_part, off_corr, off_item;
  fused_smem_layout(MP, slice_max, off_part, off_corr, off_item);
  uint16_t* sX = reinterpret_cast<uint16_t*>(fsm);
  float* part = reinterpret_cast<float*>(fsm + off_part);
  double* scorr = reinterpret_cast<double*>(fsm + off_corr);
  float* sitem = reinterpret_cast<float*>(fsm + off_item);
  __shared__ float sA[D * D], sBp[D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row0 = int64_t(blockIdx.x) * kFuRows;
  const int64_t Kb = K / 4;
  const int64_t nunits = ceil_div(K, kUnit);
  const int64_t u0 = nunits * rank / S, u1 = nunits * (rank + 1) / S;
  const int64_t k0 = u0 * kUnit;
  const int64_t klen = (u1 * kUnit < K ? u1 * kUnit : K) - k0;  // multiple of 64

  // 1. codes of this warp's 16 rows over the slice, up to kAhead units in flight
  const uint8_t* rowp[2];
  bool rowok[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t row = row0 + warp * 16 + g + 8 * h;
    rowok[h] = row < N;
    rowp[h] = packed + (rowok[h] ? row : 0) * Kb + 8 * t;
  }
  auto load_unit = [&](int64_t u, uint2 (&cw)[2]) {
    const bool kok = u < u1 && u * kUnit + 32 * t < K;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      cw[h] = (kok && rowok[h]) ? ld_stream_v2(rowp[h] + u * 32) : make_uint2(0, 0);
  };
  uint2 ring[kAhead][2];
#pragma unroll
  for (int j = 0; j < kAhead; ++j) load_unit(u0 + j, ring[j]);

  griddep_wait();  // X (possibly the previous layer's output) is complete from here

  // 2. X'' of the slice and the slice's parts of the per-row constant
  if (threadIdx.x < D * D) sA[threadIdx.x] = A[threadIdx.x];
  __syncthreads();
  if (threadIdx.x < D) {
    float rs = 0.f;
    for (int j = 0; j < D; ++j) rs += sA[threadIdx.x * D + j];
    sBp[threadIdx.x] = B[threadIdx.x] + 1.5f * rs;
  }
  __syncthreads();
  const int nhalf = static_cast<int>(klen / 8);  // items per token: halves of 16-blocks
  const int nitems = M * nhalf;
  for (int it = threadIdx.x; it < nitems; it += 256) {
    const int tok = it / nhalf, hb = it % nhalf;
    const int blk = hb >> 1, h = hb & 1;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(X + int64_t(tok) * K + k0 + 16 * blk + 8 * h));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float x[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      x[2 * q] = bf16_lo(w[q]);
      x[2 * q + 1] = bf16_hi(w[q]);
    }
    float sb = 0.f, sxr = 0.f, sxpp = 0.f;
    uint16_t* dst = sX + int64_t(tok) * xpitch + 16 * blk;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 8 * h + j;         // physical position in the 16-block
      const int vb = (c / D) * D - 8 * h;  // first input of c's vector, within this half
      const int jj = c % D;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) acc = fmaf(x[vb + i], sA[i * D + jj], acc);
      const float xr = bf16_to_f32(f32_to_bf16(acc));
      const float scale = (j % 3 == 0) ? 1.0f : ((j % 3 == 1) ? 0.25f : 0.0625f);
      const float xpp = xr * scale;
      sxr += xr;
      sxpp += xpp;
      dst[2 * j + h] = f32_to_bf16(xpp);  // decoder order: pair j holds positions j, j + 8
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) sb = fmaf(x[i], sBp[(8 * h + i) % D], sb);
    sitem[(0 * MP + tok) * (slice_max / 8) + hb] = sb;
    sitem[(1 * MP + tok) * (slice_max / 8) + hb] = sxr;
    sitem[(2 * MP + tok) * (slice_max / 8) + hb] = sxpp;
  }
  __syncthreads();
  if (threadIdx.x < M) {  // fixed-order sums of this slice's parts, in fp64
    const int tok = threadIdx.x;
    double a = 0.0, b = 0.0, c = 0.0;
    for (int hb = 0; hb < nhalf; ++hb) {
      a += sitem[(0 * MP + tok) * (slice_max / 8) + hb];
      b += sitem[(1 * MP + tok) * (slice_max / 8) + hb];
      c += sitem[(2 * MP + tok) * (slice_max / 8) + hb];
    }
    scorr[tok] = a - 1.5 * b - 128.0 * c;
  }

  // 3. main loop over the slice: B fragments from shared memory
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
  const uint16_t* xrow[NT];
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok = n * 8 + g;
    tokok[n] = tok < M;
    xrow[n] = sX + int64_t(tokok[n] ? tok : 0) * xpitch + 32 * t;
  }
  for (int64_t base = u0; base < u1; base += kAhead) {
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int64_t u = base + j;
      if (u >= u1) break;
      const bool kok = u * kUnit + 32 * t < K;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint4 xb[NT][2];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          if (kok && tokok[n]) {
            const uint4* src = reinterpret_cast<const uint4*>(xrow[n] + (u - u0) * kUnit + 16 * q);
            xb[n][0] = src[0];
            xb[n][1] = src[1];
          } else {
            xb[n][0] = make_uint4(0, 0, 0, 0);
            xb[n][1] = make_uint4(0, 0, 0, 0);
          }
        }
        uint32_t w0[2], w6[2], w12[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          w0[h] = q == 0 ? ring[j][h].x : ring[j][h].y;
          w6[h] = w0[h] >> 6;
          w12[h] = w0[h] >> 12;
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const uint32_t a0 = dec_pair_rt(2 * jj, w0[0], w6[0], w12[0]);
          const uint32_t a1 = dec_pair_rt(2 * jj, w0[1], w6[1], w12[1]);
          const uint32_t a2 = dec_pair_rt(2 * jj + 1, w0[0], w6[0], w12[0]);
          const uint32_t a3 = dec_pair_rt(2 * jj + 1, w0[1], w6[1], w12[1]);
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint32_t b0 = word_of(xb[n][jj >> 1], (2 * jj) & 3);
            const uint32_t b1 = word_of(xb[n][jj >> 1], (2 * jj + 1) & 3);
            mma_bf16_16816(acc[n], a0, a1, a2, a3, b0, b1);
          }
        }
      }
      load_unit(u + kAhead, ring[j]);
    }
  }

  // 4. partial tile -> shared memory, then the fixed-order cluster sum
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int lr = warp * 16 + g;
    const int tk = n * 8 + 2 * t;
    part[lr * (MP + 1) + tk] = acc[n][0];
    part[lr * (MP + 1) + tk + 1] = acc[n][1];
    part[(lr + 8) * (MP + 1) + tk] = acc[n][2];
    part[(lr + 8) * (MP + 1) + tk + 1] = acc[n][3];
  }
  griddep_launch_dependents();
  cluster.sync();
  const int r0 = kFuRows * rank / S, r1 = kFuRows * (rank + 1) / S;
  const int nrows = r1 - r0;
  for (int e = threadIdx.x; e < nrows * M; e += 256) {
    const int lr = r0 + e % nrows, tok = e / nrows;
    const int64_t grow = row0 + lr;
    float sum = 0.f;
    double cs = 0.0;
    for (int s2 = 0; s2 < S; ++s2) {
      const float* rp = cluster.map_shared_rank(part, s2);
      const double* rc = cluster.map_shared_rank(scorr, s2);
      sum += rp[lr * (MP + 1) + tok];
      cs += rc[tok];
    }
    if (grow < N) Y[int64_t(tok) * N + grow] = f32_to_bf16(sum + static_cast<float>(cs));
  }
  cluster.sync();
}

template <int NT, int D>
cudaError_t launch_fused_t(const uint16_t* X, const float* A, const float* B, int M,
                           const uint8_t* packed, int64_t N, int64_t K, uint16_t* Y,
                           cudaStream_t s, int S, int64_t slice_max, size_t smem) {
  auto kern = gemv_fused_kernel<NT, D>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] {
    attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 100 * 1024);
  });
  if (attr != cudaSuccess) return attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(N, kFuRows)), static_cast<unsigned>(S), 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = 1;
  attrs[0].val.clusterDim.y = static_cast<unsigned>(S);
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, X, A, B, M, packed, N, K, slice_max, Y);
}

template <int NT>
cudaError_t launch_fused_d(int d, const uint16_t* X, const float* A, const float* B, int M,
                           const uint8_t* packed, int64_t N, int64_t K, uint16_t* Y,
                           cudaStream_t s, int S, int64_t slice_max, size_t smem) {
  switch (d) {
    case 1: return launch_fused_t<NT, 1>(X, A, B, M, packed, N, K, Y, s, S, slice_max, smem);
    case 2: return launch_fused_t<NT, 2>(X, A, B, M, packed, N, K, Y, s, S, slice_max, smem);
    case 4: return launch_fused_t<NT, 4>(X, A, B, M, packed, N, K, Y, s, S, slice_max, smem);
    default: return launch_fused_t<NT, 8>(X, A, B, M, packed, N, K, Y, s, S, slice_max, smem);
  }
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* Xpp, const float* corr, int64_t M, const uint8_t* packed,
                        int64_t d_out, int64_t d_in, uint16_t* Y, cudaStream_t s,
                        int* launches) {
  cudaError_t e;
  const int m = static_cast<int>(M);
  if (M <= 8)
    e = launch_gemv_t<1, 1, 8>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  else if (M <= 16)
    e = launch_gemv_t<2, 2, 8>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  else
    e = launch_gemv_t<4, 2, 8>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

bool launch_gemv_fused(const uint16_t* X, int64_t M, const uint8_t* packed, int64_t d_out,
                       int64_t d_in, int d, const float* A, const float* B, uint16_t* Y,
                       cudaStream_t s, int* launches, cudaError_t* err) {
  if (M < 1 || M > 32) return false;
  const int64_t tiles = ceil_div(d_out, kFuRows);
  const int64_t nunits = ceil_div(d_in, kUnit);
  int S = static_cast<int>(ceil_div(2 * kNumSMsB200, tiles));
  if (S > 8) S = 8;
  int p2 = 1;
  while (p2 * 2 <= S) p2 *= 2;
  S = p2;
  while (S > 1 && S > nunits) S /= 2;
  const int64_t slice_max = ceil_div(nunits, S) * kUnit;
  const int MP = M <= 8 ? 8 : (M <= 16 ? 16 : 32);
  size_t o1, o2, o3;
  const size_t smem = fused_smem_layout(MP, slice_max, o1, o2, o3);
  if (smem > 96 * 1024) return false;  // the two-kernel path takes larger slices
  const int m = static_cast<int>(M);
  if (MP == 8)
    *err = launch_fused_d<1>(d, X, A, B, m, packed, d_out, d_in, Y, s, S, slice_max, smem);
  else if (MP == 16)
    *err = launch_fused_d<2>(d, X, A, B, m, packed, d_out, d_in, Y, s, S, slice_max, smem);
  else
    *err = launch_fused_d<4>(d, X, A, B, m, packed, d_out, d_in, Y, s, S, slice_max, smem);
  ++*launches;
  if (*err == cudaSuccess) *err = cudaGetLastError();
  return true;
}

cudaError_t launch_gemm_xformed(const uint16_t* Xpp, const float* corr, int64_t M,
                                const uint8_t* packed, int64_t d_out, int64_t d_in, uint16_t* Y,
                                unsigned int* err, cudaStream_t s, int* launches) {
  if (M <= 32) return launch_gemv(Xpp, corr, M, packed, d_out, d_in, Y, s, launches);
  return launch_tc_forward(Xpp, true, corr, M, packed, d_out, d_in, 8, nullptr, nullptr, Y, err, s,
                           launches);
}

}  // namespace lcvq

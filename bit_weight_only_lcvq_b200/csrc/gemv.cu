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
//   * the 4 lanes of a quad cover 4 consecutive 16-code words, and the MMA's
//     logical k of each lane is mapped onto its own word (the decoder order of
//     X'' makes the B fragments contiguous 128-bit loads);
//   * K is split across a thread-block cluster along grid y; the partial
//     tiles are summed in a fixed order through distributed shared memory, so
//     no partial sum ever goes to HBM and the result is deterministic.
#include <cooperative_groups.h>

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

// CTA: 8 warps on a 128-row weight tile; warp w takes row half (w & 1) (4 row
// blocks of 16) and K slice (w >> 1) of the CTA's 4; the cluster (grid y)
// splits K S ways more.  A "unit" is 128 codes of each of the warp's 64 rows:
// lane (g, t) holds 2 words of rows g and g + 8 of every row block (8 B each),
// so one unit is 16 x 64-bit loads per lane, issued one unit ahead.
constexpr int kUnit = 128;  // codes per row per unit (32 B)
constexpr int kWarps = 8;
constexpr int kRB = 4;      // row blocks of 16 per warp

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];\n"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

template <int NT>
__global__ void __launch_bounds__(kWarps * 32, (NT <= 2 ? 2 : 1)) gemv_kernel(const uint16_t* __restrict__ Xpp,
                                                           const float* __restrict__ corr, int M,
                                                           const uint8_t* __restrict__ packed,
                                                           int64_t N, int64_t K,
                                                           uint16_t* __restrict__ Y) {
  constexpr int MP = NT * 8;
  __shared__ float part[kGemvRows][MP + 1];

  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.dim_blocks().y);
  const int rank = static_cast<int>(cluster.block_index().y);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rh = warp & 1, ks = warp >> 1;
  const int64_t tile_row0 = int64_t(blockIdx.x) * kGemvRows;
  const int64_t Kb = K / 4;
  const int64_t nunits = ceil_div(K, kUnit);
  const int nslices = 4 * S;
  const int gs = rank * 4 + ks;
  const int64_t u0 = nunits * gs / nslices, u1 = nunits * (gs + 1) / nslices;

  const uint8_t* rowp[kRB][2];
  bool rowok[kRB][2];
#pragma unroll
  for (int r = 0; r < kRB; ++r)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t row = tile_row0 + rh * 64 + r * 16 + g + 8 * h;
      rowok[r][h] = row < N;
      rowp[r][h] = packed + (rowok[r][h] ? row : 0) * Kb + 8 * t;
    }
  const uint16_t* xrow[NT];
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok = n * 8 + g;
    tokok[n] = tok < M;
    xrow[n] = Xpp + int64_t(tokok[n] ? tok : 0) * K + 32 * t;
  }

  float acc[kRB][NT][4];
#pragma unroll
  for (int r = 0; r < kRB; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

  auto load_codes = [&](int64_t u, uint2 (&cw)[kRB][2]) {
    const bool kok = u * kUnit + 32 * t < K;  // K % 64 == 0: whole 32-code lane chunks
#pragma unroll
    for (int r = 0; r < kRB; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        cw[r][h] = (kok && rowok[r][h]) ? ld_stream_v2(rowp[r][h] + u * 32) : make_uint2(0, 0);
  };

  uint2 cur[kRB][2], nxt[kRB][2];
  if (u0 < u1) load_codes(u0, cur);
  for (int64_t u = u0; u < u1; ++u) {
    if (u + 1 < u1) load_codes(u + 1, nxt);
    const bool kok = u * kUnit + 32 * t < K;
#pragma unroll
    for (int q = 0; q < 2; ++q) {  // word q of each row: 16 codes, 4 k16 tiles
      uint4 xb[NT][2];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (kok && tokok[n]) {
          const uint4* src = reinterpret_cast<const uint4*>(xrow[n] + u * kUnit + 16 * q);
          xb[n][0] = __ldg(src);
          xb[n][1] = __ldg(src + 1);
        } else {
          xb[n][0] = make_uint4(0, 0, 0, 0);
          xb[n][1] = make_uint4(0, 0, 0, 0);
        }
      }
      uint32_t w0[kRB][2], w6[kRB][2], w12[kRB][2];
#pragma unroll
      for (int r = 0; r < kRB; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          w0[r][h] = q == 0 ? cur[r][h].x : cur[r][h].y;
          w6[r][h] = w0[r][h] >> 6;
          w12[r][h] = w0[r][h] >> 12;
        }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {  // k16 tile: pairs 2jj, 2jj+1 of word q
        uint32_t a[kRB][2][2];
#pragma unroll
        for (int r = 0; r < kRB; ++r)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            a[r][h][0] = dec_pair_rt(2 * jj, w0[r][h], w6[r][h], w12[r][h]);
            a[r][h][1] = dec_pair_rt(2 * jj + 1, w0[r][h], w6[r][h], w12[r][h]);
          }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint32_t b0 = word_of(xb[n][jj >> 1], (2 * jj) & 3);
          const uint32_t b1 = word_of(xb[n][jj >> 1], (2 * jj + 1) & 3);
#pragma unroll
          for (int r = 0; r < kRB; ++r)
            mma_bf16_16816(acc[r][n], a[r][0][0], a[r][1][0], a[r][0][1], a[r][1][1], b0, b1);
        }
      }
    }
    if (u + 1 < u1) {
#pragma unroll
      for (int r = 0; r < kRB; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) cur[r][h] = nxt[r][h];
    }
  }

  // the CTA's 4 K slices, summed into shared memory in slice order
  for (int round = 0; round < 4; ++round) {
    if (ks == round) {
#pragma unroll
      for (int r = 0; r < kRB; ++r)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const int lr = rh * 64 + r * 16 + g;
          const int tk = n * 8 + 2 * t;
          if (round == 0) {
            part[lr][tk] = acc[r][n][0];
            part[lr][tk + 1] = acc[r][n][1];
            part[lr + 8][tk] = acc[r][n][2];
            part[lr + 8][tk + 1] = acc[r][n][3];
          } else {
            part[lr][tk] += acc[r][n][0];
            part[lr][tk + 1] += acc[r][n][1];
            part[lr + 8][tk] += acc[r][n][2];
            part[lr + 8][tk + 1] += acc[r][n][3];
          }
        }
    }
    __syncthreads();
  }
  cluster.sync();

  // rank r of the cluster finishes rows [r0, r1) of the tile over all ranks
  const int r0 = kGemvRows * rank / S, r1 = kGemvRows * (rank + 1) / S;
  const int nrows = r1 - r0;
  const int total = nrows * M;
  for (int e = threadIdx.x; e < total; e += kWarps * 32) {
    const int lr = r0 + e % nrows;
    const int tok = e / nrows;
    const int64_t grow = tile_row0 + lr;
    float sum = 0.f;
    for (int s2 = 0; s2 < S; ++s2) {
      const float* rp = cluster.map_shared_rank(&part[0][0], s2);
      sum += rp[lr * (MP + 1) + tok];
    }
    if (grow < N) Y[int64_t(tok) * N + grow] = f32_to_bf16(sum + corr[tok]);
  }
  cluster.sync();  // keep every CTA's shared memory alive until all reads are done
}

template <int NT>
cudaError_t launch_gemv_t(const uint16_t* Xpp, const float* corr, int M, const uint8_t* packed,
                          int64_t N, int64_t K, uint16_t* Y, cudaStream_t s) {
  const int64_t tiles = ceil_div(N, kGemvRows);
  const int64_t nunits = ceil_div(K, kUnit);
  int S = static_cast<int>(ceil_div(2 * kNumSMsB200, tiles));
  if (S > 8) S = 8;
  int p2 = 1;
  while (p2 * 2 <= S) p2 *= 2;
  S = p2;
  while (S > 1 && 4 * S > nunits) S /= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(S), 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(S);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT>, Xpp, corr, M, packed, N, K, Y);
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* Xpp, const float* corr, int64_t M, const uint8_t* packed,
                        int64_t d_out, int64_t d_in, uint16_t* Y, cudaStream_t s,
                        int* launches) {
  cudaError_t e;
  const int m = static_cast<int>(M);
  if (M <= 8)
    e = launch_gemv_t<1>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  else if (M <= 16)
    e = launch_gemv_t<2>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  else
    e = launch_gemv_t<4>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm_xformed(const uint16_t* Xpp, const float* corr, int64_t M,
                                const uint8_t* packed, int64_t d_out, int64_t d_in, uint16_t* Y,
                                unsigned int* err, cudaStream_t s, int* launches) {
  if (M <= 32) return launch_gemv(Xpp, corr, M, packed, d_out, d_in, Y, s, launches);
  return launch_tc_forward(Xpp, true, corr, M, packed, d_out, d_in, 8, nullptr, nullptr, Y, err, s,
                           launches);
}

}  // namespace lcvq

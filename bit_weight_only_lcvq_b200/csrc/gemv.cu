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
constexpr int kGemvIterK = 256;  // codes per row per main-loop iteration (64 B)

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

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

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

template <int NT, int R, int W>
__global__ void __launch_bounds__(W * 32) gemv_kernel(const uint16_t* __restrict__ Xpp,
                                                      const float* __restrict__ corr, int M,
                                                      const uint8_t* __restrict__ packed,
                                                      int64_t N, int64_t K,
                                                      uint16_t* __restrict__ Y) {
  static_assert(W * R * 16 == kGemvRows, "tile rows");
  constexpr int MP = NT * 8;
  __shared__ float part[kGemvRows][MP + 1];

  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.dim_blocks().y);
  const int split = static_cast<int>(cluster.block_index().y);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t tile_row0 = int64_t(blockIdx.x) * kGemvRows;
  const int64_t row0 = tile_row0 + warp * (R * 16);
  const int64_t Kb = K / 4;  // bytes of codes per row
  const int64_t niter = ceil_div(K, kGemvIterK);
  const int64_t it0 = niter * split / S;
  const int64_t it1 = niter * (split + 1) / S;

  float acc[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

  const uint8_t* rowp[R][2];
  bool rowok[R][2];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t row = row0 + r * 16 + g + 8 * h;
      rowok[r][h] = row < N;
      rowp[r][h] = packed + (rowok[r][h] ? row : 0) * Kb;
    }
  const int tok0 = static_cast<int>(blockIdx.z) * MP;  // token chunk of this CTA
  const uint16_t* xrow[NT];
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok = tok0 + n * 8 + g;
    tokok[n] = tok < M;
    xrow[n] = Xpp + int64_t(tokok[n] ? tok : 0) * K;
  }

  for (int64_t it = it0; it < it1; ++it) {
    const int64_t kbyte = it * 64 + 16 * t;
    const bool kok = kbyte < Kb;  // K % 64 == 0: a lane's 16 B are all in or all out
    uint4 cw[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        cw[r][h] = (kok && rowok[r][h]) ? ld_stream_v4(rowp[r][h] + kbyte) : make_uint4(0, 0, 0, 0);
    const int64_t kel = it * kGemvIterK + 64 * t;  // first X'' element of this lane
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 xb[NT][2];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (kok && tokok[n]) {
          const uint4* src = reinterpret_cast<const uint4*>(xrow[n] + kel + 16 * q);
          xb[n][0] = __ldg(src);
          xb[n][1] = __ldg(src + 1);
        } else {
          xb[n][0] = make_uint4(0, 0, 0, 0);
          xb[n][1] = make_uint4(0, 0, 0, 0);
        }
      }
      uint32_t a[R][2][8];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t w0 = word_of(cw[r][h], q);
          const uint32_t w6 = w0 >> 6, w12 = w0 >> 12;
          a[r][h][0] = dec_pair<0>(w0, w6, w12);
          a[r][h][1] = dec_pair<1>(w0, w6, w12);
          a[r][h][2] = dec_pair<2>(w0, w6, w12);
          a[r][h][3] = dec_pair<3>(w0, w6, w12);
          a[r][h][4] = dec_pair<4>(w0, w6, w12);
          a[r][h][5] = dec_pair<5>(w0, w6, w12);
          a[r][h][6] = dec_pair<6>(w0, w6, w12);
          a[r][h][7] = dec_pair<7>(w0, w6, w12);
        }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {  // k16 tile: pairs 2jj, 2jj+1 of word q
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint32_t b0 = word_of(xb[n][jj >> 1], (2 * jj) & 3);
          const uint32_t b1 = word_of(xb[n][jj >> 1], (2 * jj + 1) & 3);
#pragma unroll
          for (int r = 0; r < R; ++r)
            mma_bf16_16816(acc[r][n], a[r][0][2 * jj], a[r][1][2 * jj], a[r][0][2 * jj + 1],
                           a[r][1][2 * jj + 1], b0, b1);
        }
      }
    }
  }

  // partial tile -> shared memory
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int lr = warp * R * 16 + r * 16 + g;
      const int tk = n * 8 + 2 * t;
      part[lr][tk] = acc[r][n][0];
      part[lr][tk + 1] = acc[r][n][1];
      part[lr + 8][tk] = acc[r][n][2];
      part[lr + 8][tk + 1] = acc[r][n][3];
    }
  cluster.sync();

  // CTA `split` of the cluster reduces rows [r0, r1) of the tile over all ranks.
  const int r0 = kGemvRows * split / S, r1 = kGemvRows * (split + 1) / S;
  const int nrows = r1 - r0;
  const int mtok = min(MP, M - tok0);
  const int total = nrows * mtok;
  for (int e = threadIdx.x; e < total; e += W * 32) {
    const int lr = r0 + e % nrows;
    const int tok = e / nrows;
    const int64_t grow = tile_row0 + lr;
    float sum = 0.f;
    for (int s = 0; s < S; ++s) {
      const float* rp = cluster.map_shared_rank(&part[0][0], s);
      sum += rp[lr * (MP + 1) + tok];
    }
    if (grow < N) Y[int64_t(tok0 + tok) * N + grow] = f32_to_bf16(sum + corr[tok0 + tok]);
  }
  cluster.sync();  // keep every CTA's shared memory alive until all reads are done
}

template <int NT, int R, int W>
cudaError_t launch_gemv_t(const uint16_t* Xpp, const float* corr, int M, const uint8_t* packed,
                          int64_t N, int64_t K, uint16_t* Y, cudaStream_t s) {
  const int64_t tiles = ceil_div(N, kGemvRows);
  const int64_t niter = ceil_div(K, kGemvIterK);
  const int64_t chunks = ceil_div(M, NT * 8);
  int S = static_cast<int>(ceil_div(2 * kNumSMsB200, tiles * chunks));
  if (S > 8) S = 8;
  if (S > niter) S = static_cast<int>(niter);
  if (S < 1) S = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(S),
                     static_cast<unsigned>(chunks));
  cfg.blockDim = dim3(W * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(S);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, R, W>, Xpp, corr, M, packed, N, K, Y);
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* Xpp, const float* corr, int64_t M, const uint8_t* packed,
                        int64_t d_out, int64_t d_in, uint16_t* Y, cudaStream_t s,
                        int* launches) {
  cudaError_t e;
  const int m = static_cast<int>(M);
  if (M <= 8)
    e = launch_gemv_t<1, 4, 2>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  else if (M <= 16)
    e = launch_gemv_t<2, 4, 2>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  else
    e = launch_gemv_t<4, 2, 4>(Xpp, corr, m, packed, d_out, d_in, Y, s);
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

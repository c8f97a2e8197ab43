// CUDA-core paths: forward, dX and the dW epilogue for any M and either
// activation type (fp32 or bf16), with fp32 arithmetic throughout.  They carry
// the fp32 workloads (where tensor-core inputs would not meet an fp32
// tolerance) and every shape the tensor-core kernels do not take.
//
//   forward  Y[m][n]  = sum_k X[m][k] W~[n][k]            (decoupleQ eq. (1))
//   dX[m][k]          = sum_n dY[m][n] W~[n][k]            (gradient through the
//                                                           linear map, LC-QAT
//                                                           Methodology 1)
//   G[n][k]           = sum_m dY[m][n] X[m][k]   -> per d-vector epilogue:
//   dWp[n][gd+j]      = mask * sum_i A[i][j] G[n][gd+i]    (STE, Methodology 3)
//   dA[i][j] += G[n][gd+i] z[n][gd+j],  dB[i] += G[n][gd+i]  (per-tile partials)
//
// W~ tiles are decoded on chip from the packed codes (A z + B in fp32, a fixed
// FMA order) and never written to memory.
#include "common.cuh"
#include "internal.h"

namespace lcvq {

namespace {

constexpr int kT = 64;   // output tile edge
constexpr int kBK = 32;  // contraction chunk
constexpr int kThreads = 256;

template <bool kBf16>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&v)[8]) {
  if constexpr (kBf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx);
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <bool kBf16>
__device__ __forceinline__ void store_out(void* base, int64_t idx, float v) {
  if constexpr (kBf16)
    static_cast<uint16_t*>(base)[idx] = f32_to_bf16(v);
  else
    static_cast<float*>(base)[idx] = v;
}

// decode 8 consecutive weights (whole d-vectors) of one row from 16 code bits
template <int D>
__device__ __forceinline__ void decode8(uint32_t bits16, const float* sA, const float* sB,
                                        float (&w)[8]) {
#pragma unroll
  for (int v = 0; v < 8 / D; ++v) {
    float z[D];
#pragma unroll
    for (int j = 0; j < D; ++j) z[j] = static_cast<float>((bits16 >> (2 * (v * D + j))) & 3u);
#pragma unroll
    for (int i = 0; i < D; ++i) {
      float acc = sB[i];
#pragma unroll
      for (int j = 0; j < D; ++j) acc = fmaf(sA[i * D + j], z[j], acc);
      w[v * D + i] = acc;
    }
  }
}

__device__ __forceinline__ uint32_t codes16(const uint8_t* packed, int64_t Kb, int64_t row,
                                            int64_t k) {
  return *reinterpret_cast<const uint16_t*>(packed + row * Kb + (k >> 2));
}

template <int D>
__device__ __forceinline__ void load_AB(const float* A, const float* B, float* sA, float* sB) {
  for (int i = threadIdx.x; i < D * D; i += blockDim.x) sA[i] = A[i];
  for (int i = threadIdx.x; i < D; i += blockDim.x) sB[i] = B[i];
}

// ---------------------------------------------------------------- forward
template <int D, bool kBf16>
__global__ void __launch_bounds__(kThreads) simt_forward_kernel(
    const void* __restrict__ X, int64_t M, const uint8_t* __restrict__ packed, int64_t N,
    int64_t K, const float* __restrict__ A, const float* __restrict__ B, void* __restrict__ Y) {
  __shared__ float sA[D * D], sB[D];
  __shared__ float Xs[kBK][kT + 4];
  __shared__ float Ws[kBK][kT + 4];
  load_AB<D>(A, B, sA, sB);
  const int tid = threadIdx.x;
  const int64_t m0 = int64_t(blockIdx.y) * kT, n0 = int64_t(blockIdx.x) * kT;
  const int ty = tid / 16, tx = tid % 16;
  const int lrow = tid / 4, lk = (tid % 4) * 8;
  const int64_t Kb = K / 4;
  float acc[4][4] = {};
  __syncthreads();
  for (int64_t k0 = 0; k0 < K; k0 += kBK) {
    float xv[8], wv[8];
    if (m0 + lrow < M) load8<kBf16>(X, (m0 + lrow) * K + k0 + lk, xv);
    else for (int i = 0; i < 8; ++i) xv[i] = 0.f;
    if (n0 + lrow < N) decode8<D>(codes16(packed, Kb, n0 + lrow, k0 + lk), sA, sB, wv);
    else for (int i = 0; i < 8; ++i) wv[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      Xs[lk + i][lrow] = xv[i];
      Ws[lk + i][lrow] = wv[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = Xs[kk][ty * 4 + i]; b[i] = Ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) store_out<kBf16>(Y, m * N + n, acc[i][j]);
    }
}

// ---------------------------------------------------------------- dX
template <int D, bool kBf16>
__global__ void __launch_bounds__(kThreads) simt_dx_kernel(
    const void* __restrict__ dY, int64_t M, const uint8_t* __restrict__ packed, int64_t N,
    int64_t K, const float* __restrict__ A, const float* __restrict__ B, void* __restrict__ dX) {
  __shared__ float sA[D * D], sB[D];
  __shared__ float Ds[kBK][kT + 4];  // [n][m]
  __shared__ float Ws[kBK][kT + 4];  // [n][k]
  load_AB<D>(A, B, sA, sB);
  const int tid = threadIdx.x;
  const int64_t m0 = int64_t(blockIdx.y) * kT, k0 = int64_t(blockIdx.x) * kT;
  const int ty = tid / 16, tx = tid % 16;
  const int64_t Kb = K / 4;
  float acc[4][4] = {};
  __syncthreads();
  for (int64_t nb = 0; nb < N; nb += kBK) {
    {  // dY tile: 64 m x 32 n
      const int lm = tid / 4, ln = (tid % 4) * 8;
      float v[8];
      if (m0 + lm < M && nb + ln < N) load8<kBf16>(dY, (m0 + lm) * N + nb + ln, v);
      else for (int i = 0; i < 8; ++i) v[i] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) Ds[ln + i][lm] = v[i];
    }
    {  // W~ tile: 32 n x 64 k
      const int ln = tid / 8, lk = (tid % 8) * 8;
      float w[8];
      if (nb + ln < N) decode8<D>(codes16(packed, Kb, nb + ln, k0 + lk), sA, sB, w);
      else for (int i = 0; i < 8; ++i) w[i] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) Ws[ln][lk + i] = w[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int nn = 0; nn < kBK; ++nn) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = Ds[nn][ty * 4 + i]; b[i] = Ws[nn][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + ty * 4 + i, k = k0 + tx * 4 + j;
      if (m < M) store_out<kBf16>(dX, m * K + k, acc[i][j]);
    }
}

// ---------------------------------------------------------------- dW epilogue
template <int D, bool kBf16>
__global__ void __launch_bounds__(kThreads) simt_dw_kernel(
    const void* __restrict__ X, const void* __restrict__ dY, int64_t M,
    const uint8_t* __restrict__ packed, const uint8_t* __restrict__ mask, int64_t N, int64_t K,
    const float* __restrict__ A, float* __restrict__ dWp, float* __restrict__ partials) {
  constexpr int NP = D * D + D;
  __shared__ float sA[D * D];
  __shared__ float buf[2][kBK][kT + 4];  // [0]: dY tile [m][n]; [1]: X tile [m][k]; then G
  __shared__ float red[kThreads / 32][NP];
  float (*Ds)[kT + 4] = buf[0];
  float (*Xs)[kT + 4] = buf[1];
  for (int i = threadIdx.x; i < D * D; i += blockDim.x) sA[i] = A[i];
  const int tid = threadIdx.x;
  const int64_t n0 = int64_t(blockIdx.y) * kT, k0 = int64_t(blockIdx.x) * kT;
  const int ty = tid / 16, tx = tid % 16;
  const int64_t Kb = K / 4;
  float acc[4][4] = {};
  __syncthreads();
  for (int64_t mb = 0; mb < M; mb += kBK) {
    const int lm = tid / 8, lc = (tid % 8) * 8;
    float v[8];
    if (mb + lm < M && n0 + lc < N) load8<kBf16>(dY, (mb + lm) * N + n0 + lc, v);
    else for (int i = 0; i < 8; ++i) v[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) Ds[lm][lc + i] = v[i];
    if (mb + lm < M) load8<kBf16>(X, (mb + lm) * K + k0 + lc, v);
    else for (int i = 0; i < 8; ++i) v[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) Xs[lm][lc + i] = v[i];
    __syncthreads();
#pragma unroll 8
    for (int mm = 0; mm < kBK; ++mm) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = Ds[mm][ty * 4 + i]; b[i] = Xs[mm][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  // G tile -> shared memory, reusing the operand buffers (64 x 65 <= 2 x 32 x 68 floats)
  float* Gs = &buf[0][0][0];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) Gs[(ty * 4 + i) * (kT + 1) + tx * 4 + j] = acc[i][j];
  __syncthreads();

  float pa[D * D], pb[D];
#pragma unroll
  for (int i = 0; i < D * D; ++i) pa[i] = 0.f;
#pragma unroll
  for (int i = 0; i < D; ++i) pb[i] = 0.f;
  constexpr int VPR = kT / D;  // vectors per tile row
  for (int v = tid; v < kT * VPR; v += kThreads) {
    const int lr = v / VPR, gv = v % VPR;
    const int64_t n = n0 + lr;
    if (n >= N) continue;
    const int64_t kv = k0 + int64_t(gv) * D;
    float G[D];
#pragma unroll
    for (int i = 0; i < D; ++i) G[i] = Gs[lr * (kT + 1) + gv * D + i];
    float z[D];
    uint32_t mbits = 0;
#pragma unroll
    for (int j = 0; j < D; ++j) {
      const int64_t k = kv + j;
      z[j] = static_cast<float>((packed[n * Kb + (k >> 2)] >> (2 * (k & 3))) & 3u);
      if (mask != nullptr) mbits |= ((mask[n * (K / 8) + (k >> 3)] >> (k & 7)) & 1u) << j;
    }
#pragma unroll
    for (int i = 0; i < D; ++i) {
      pb[i] += G[i];
#pragma unroll
      for (int j = 0; j < D; ++j) pa[i * D + j] = fmaf(G[i], z[j], pa[i * D + j]);
    }
    if (dWp != nullptr) {
#pragma unroll
      for (int j = 0; j < D; ++j) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) s = fmaf(sA[i * D + j], G[i], s);
        dWp[n * K + kv + j] = ((mbits >> j) & 1u) ? s : 0.f;
      }
    }
  }
  // fixed-order block reduction of the D*D + D partials
  const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    float x = e < D * D ? pa[e] : pb[e - D * D];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xffffffffu, x, off);
    if (lane == 0) red[warp][e] = x;
  }
  __syncthreads();
  if (tid < NP) {
    float s = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) s += red[w][tid];
    const int64_t tile = int64_t(blockIdx.y) * gridDim.x + blockIdx.x;
    partials[tile * NP + tid] = s;
  }
}

// one CTA per output element; fp64, fixed order
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float* __restrict__ partials,
                                                              int64_t num_parts, int np, int dd,
                                                              float* __restrict__ dA,
                                                              float* __restrict__ dB) {
  __shared__ double red[256];
  const int e = blockIdx.x;
  double s = 0.0;
  for (int64_t p = threadIdx.x; p < num_parts; p += 256) s += partials[p * np + e];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {
    if (threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (e < dd) dA[e] = static_cast<float>(red[0]);
    else dB[e - dd] = static_cast<float>(red[0]);
  }
}

}  // namespace

#define LCVQ_DISPATCH_D(d, BF, KERNEL, GRID, ...)                                    \
  do {                                                                               \
    switch (d) {                                                                     \
      case 1: if (BF) KERNEL<1, true><<<GRID, kThreads, 0, s>>>(__VA_ARGS__);        \
              else KERNEL<1, false><<<GRID, kThreads, 0, s>>>(__VA_ARGS__); break;   \
      case 2: if (BF) KERNEL<2, true><<<GRID, kThreads, 0, s>>>(__VA_ARGS__);        \
              else KERNEL<2, false><<<GRID, kThreads, 0, s>>>(__VA_ARGS__); break;   \
      case 4: if (BF) KERNEL<4, true><<<GRID, kThreads, 0, s>>>(__VA_ARGS__);        \
              else KERNEL<4, false><<<GRID, kThreads, 0, s>>>(__VA_ARGS__); break;   \
      default: if (BF) KERNEL<8, true><<<GRID, kThreads, 0, s>>>(__VA_ARGS__);       \
              else KERNEL<8, false><<<GRID, kThreads, 0, s>>>(__VA_ARGS__); break;   \
    }                                                                                \
  } while (0)

cudaError_t launch_simt_forward(const void* X, bool bf16, int64_t M, const uint8_t* packed,
                                int64_t d_out, int64_t d_in, int d, const float* A,
                                const float* B, void* Y, cudaStream_t s, int* launches) {
  const dim3 grid(static_cast<unsigned>(ceil_div(d_out, kT)), static_cast<unsigned>(ceil_div(M, kT)));
  LCVQ_DISPATCH_D(d, bf16, simt_forward_kernel, grid, X, M, packed, d_out, d_in, A, B, Y);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_simt_backward_dx(const void* dY, bool bf16, int64_t M, const uint8_t* packed,
                                    int64_t d_out, int64_t d_in, int d, const float* A,
                                    const float* B, void* dX, cudaStream_t s, int* launches) {
  const dim3 grid(static_cast<unsigned>(d_in / kT), static_cast<unsigned>(ceil_div(M, kT)));
  LCVQ_DISPATCH_D(d, bf16, simt_dx_kernel, grid, dY, M, packed, d_out, d_in, A, B, dX);
  ++*launches;
  return cudaGetLastError();
}

int64_t simt_dw_num_tiles(int64_t d_out, int64_t d_in) { return ceil_div(d_out, kT) * (d_in / kT); }

cudaError_t launch_simt_backward_dw(const void* X, const void* dY, bool bf16, int64_t M,
                                    const uint8_t* packed, const uint8_t* mask_bits,
                                    int64_t d_out, int64_t d_in, int d, const float* A,
                                    float* dWp, float* partials, cudaStream_t s, int* launches) {
  const dim3 grid(static_cast<unsigned>(d_in / kT), static_cast<unsigned>(ceil_div(d_out, kT)));
  LCVQ_DISPATCH_D(d, bf16, simt_dw_kernel, grid, X, dY, M, packed, mask_bits, d_out, d_in, A,
                  dWp, partials);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_reduce_partials(const float* partials, int64_t num_parts, int d, float* dA,
                                   float* dB, cudaStream_t s, int* launches) {
  const int np = d * d + d;
  reduce_partials_kernel<<<np, 256, 0, s>>>(partials, num_parts, np, d * d, dA, dB);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace lcvq

// Prologue of the algebraic form of the forward (LC-QAT technical summary,
// Methodology 3: the forward is recast onto INT2 x FP16 matmul operators).
//
// For every activation row x and every d-vector g:
//     sum_k x_k W~[n][k] = sum_g x_g^T (A z_g + B)
//                        = sum_k X'_k z_k + sum_g x_g^T B
// with X'[g d + j] = sum_i x[g d + i] A[i][j].  Centering the codes
// (zc = z - 3/2, W~ = A zc + B', B' = B + 3/2 A 1) gives the same sum as
// sum_k X'_k zc_k + s', s' = sum_g x_g^T B'.
//
// The tensor-core main loops multiply X'' (below) with codes that are decoded
// by one LOP3 each into the bf16 value 128 + 4^p z, p = p(position) in {0,1,2}
// (the code lands in mantissa bits 2p..2p+1 of a bf16 whose exponent says 128).
// So the B operand is X'' = bf16(X') * 4^-p (exact power-of-two scaling) and
//     acc = sum_k X''_k (128 + 4^p z_k) = sum_k X'r_k z_k + 128 sum_k X''_k,
// where X'r = bf16(X').  The per-row constant
//     corr = s' - 3/2 sum_k X'r_k - 128 sum_k X''_k
// makes acc + corr = sum_k X'r_k zc_k + s': the centred form, whose only
// rounding is that of X' to bf16 (relative 2^-9 per term, against codes of
// magnitude <= 3/2).  The sums are formed in fp64.
//
// K order ("decoder order"): inside every block of 16 consecutive k, the decoder
// turns one 32-bit word of codes into 8 bf16x2 pairs, pair c holding positions
// c and c + 8 (the same bit offset in the two 16-bit halves).  X'' is stored in
// that order: element 2c of the block is position c, element 2c+1 is c + 8;
// p(c) = c mod 3.
#include "common.cuh"
#include "internal.h"
#include "xform.cuh"

namespace lcvq {

constexpr int kXfThreads = 256;

// One launch transforms the rows of up to kItems matrices' activations: CTA
// (m, i) does row m of item i (a single call is a group of one).
struct XformItem {
  const uint16_t* X;  // [M][d_in] bf16
  const float* A;     // [D*D]
  const float* B;     // [D]
  uint16_t* Xpp;      // [M][d_in] out
  float* corr;        // [M] out
  int64_t d_in;
};
template <int kItems>
struct XformGroup {
  XformItem item[kItems];
};

template <int D, int kItems>
__global__ void __launch_bounds__(kXfThreads)
    xform_kernel(const __grid_constant__ XformGroup<kItems> grp) {
  const XformItem& it = grp.item[blockIdx.y];
  // X, A and B may come from the kernel just before this one: read them with
  // ld_global_*, never through the read-only path
  const uint16_t* X = it.X;
  const float* A = it.A;
  const float* B = it.B;
  uint16_t* __restrict__ Xpp = it.Xpp;
  float* __restrict__ corr = it.corr;
  const int64_t d_in = it.d_in;
  __shared__ float sA[D * D];
  __shared__ float sB[D];
  __shared__ float sBp[D];
  __shared__ double red[3][kXfThreads / 32];
  // Programmatic dependent launch.  This kernel waits for every earlier kernel
  // before it touches anything (X may be the previous layer's output), and only
  // then lets the decode-GEMV that follows launch: that GEMV reads packed codes
  // before its own wait, which is safe because every kernel that could have
  // written them has completed by the time this wait returns, and this kernel
  // writes none.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int64_t m = blockIdx.x;
  const uint16_t* xr = X + m * d_in;
  uint16_t* orow = Xpp + m * d_in;
  // warp w takes the chunks c = w, w + 8, ... (the classes of the corr sum);
  // lane l transforms block l of the chunk.  The first chunk's activations
  // are loaded together with A and B.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nblk = d_in / 16;
  const int64_t nchunk = ceil_div(d_in, kCorrChunk);
  uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0;
  {
    const int64_t b = int64_t(warp) * (kCorrChunk / 16) + lane;
    if (warp < nchunk && b < nblk) {
      p0 = ld_global_v4(xr + 16 * b);
      p1 = ld_global_v4(xr + 16 * b + 8);
    }
  }
  if (threadIdx.x < D * D) sA[threadIdx.x] = ld_global_f32(A + threadIdx.x);
  if (threadIdx.x < D) sB[threadIdx.x] = ld_global_f32(B + threadIdx.x);
  __syncthreads();
  if (threadIdx.x < D) sBp[threadIdx.x] = shifted_offset<D>(sA + threadIdx.x * D, sB[threadIdx.x]);
  __syncthreads();

  double s_b = 0.0, s_xr = 0.0, s_xpp = 0.0;  // this class's running sums (lane 0)
  for (int64_t c = warp; c < nchunk; c += kCorrClasses) {
    const int64_t b = c * (kCorrChunk / 16) + lane;
    float sb = 0.f, sxr = 0.f, sxpp = 0.f;
    if (b < nblk) {
      uint4 u0 = p0, u1 = p1;
      if (c != warp) {
        u0 = ld_global_v4(xr + 16 * b);
        u1 = ld_global_v4(xr + 16 * b + 8);
      }
      uint32_t o[8];
      xform_block<D>(u0, u1, sA, sBp, o, sb, sxr, sxpp);
      uint4* dst = reinterpret_cast<uint4*>(orow + 16 * b);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    const double tb = chunk_tree_sum(double(sb));
    const double txr = chunk_tree_sum(double(sxr));
    const double txpp = chunk_tree_sum(double(sxpp));
    if (lane == 0) {
      s_b += tb;
      s_xr += txr;
      s_xpp += txpp;
    }
  }
  static_assert(kXfThreads / 32 == kCorrClasses, "one warp per chunk class");
  if (lane == 0) {
    red[0][warp] = s_b;
    red[1][warp] = s_xr;
    red[2][warp] = s_xpp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0, c = 0.0;
    for (int w = 0; w < kCorrClasses; ++w) {
      a += red[0][w];
      b += red[1][w];
      c += red[2][w];
    }
    corr[m] = static_cast<float>(a - 1.5 * b - 128.0 * c);
  }
}

namespace {
template <int kItems>
cudaError_t launch_xform_group(const XformGroup<kItems>& grp, int count, int64_t M, int d,
                               cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M), static_cast<unsigned>(count), 1);
  cfg.blockDim = dim3(kXfThreads, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (d) {
    case 1: return cudaLaunchKernelEx(&cfg, xform_kernel<1, kItems>, grp);
    case 2: return cudaLaunchKernelEx(&cfg, xform_kernel<2, kItems>, grp);
    case 4: return cudaLaunchKernelEx(&cfg, xform_kernel<4, kItems>, grp);
    default: return cudaLaunchKernelEx(&cfg, xform_kernel<8, kItems>, grp);
  }
}
}  // namespace

cudaError_t launch_xform(const uint16_t* X, int64_t M, int64_t d_in, int d, const float* A,
                         const float* B, uint16_t* Xpp, float* corr, cudaStream_t s,
                         int* launches) {
  XformGroup<1> grp{};
  grp.item[0] = XformItem{X, A, B, Xpp, corr, d_in};
  cudaError_t e = launch_xform_group(grp, 1, M, d, s);
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_xform_grouped(const XformJob* jobs, int count, int64_t M, int d,
                                 cudaStream_t s, int* launches) {
  for (int first = 0; first < count; first += kMaxGroupItems) {
    const int n = count - first < kMaxGroupItems ? count - first : kMaxGroupItems;
    XformGroup<kMaxGroupItems> grp{};
    for (int i = 0; i < n; ++i) {
      const XformJob& j = jobs[first + i];
      grp.item[i] = XformItem{j.X, j.A, j.B, j.Xpp, j.corr, j.d_in};
    }
    cudaError_t e = launch_xform_group(grp, n, M, d, s);
    ++*launches;
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// r[m] = sum_n dY[m][n]: the rank-1 term of the dX epilogue (the B part of
// W~ = A z + B contributes B_i r[m] to dX[m][g d + i]).
__global__ void __launch_bounds__(256) rowsum_kernel(const uint16_t* __restrict__ dY, int64_t n,
                                                     float* __restrict__ r) {
  __shared__ double red[8];
  const uint16_t* row = dY + int64_t(blockIdx.x) * n;
  double s = 0.0;
  for (int64_t j = threadIdx.x * 8; j < n; j += 256 * 8) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + j));
    s += double(bf16_lo(u.x)) + double(bf16_hi(u.x)) + double(bf16_lo(u.y)) + double(bf16_hi(u.y)) +
         double(bf16_lo(u.z)) + double(bf16_hi(u.z)) + double(bf16_lo(u.w)) + double(bf16_hi(u.w));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_down_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    r[blockIdx.x] = static_cast<float>(t);
  }
}

cudaError_t launch_rowsum(const uint16_t* dY, int64_t M, int64_t n, float* r, cudaStream_t s,
                          int* launches) {
  rowsum_kernel<<<static_cast<unsigned>(M), 256, 0, s>>>(dY, n, r);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace lcvq

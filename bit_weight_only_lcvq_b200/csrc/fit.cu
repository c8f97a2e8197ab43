// Least-squares refit of the float part (A, B) given the codes: the layer
// objective of the decoupleQ page, eq. (5), tr{(W~ - W0)^T H (W~ - W0)}, with H
// taken as its diagonal h (one weight per input channel), minimized over
// (A, B) with the integer part fixed -- the closed-form float-part step of
// its section 3.3, for LC-VQ's codewords c = A z + B (LC-QAT technical
// summary, Methodology 1).
//
// The objective splits over the output coordinate i of a vector: row i of
// [A | B] is theta_i = G_i^+ R_i with, over every vector (row n, group g) and
// its channel k = g d + i and zt = [z_0 .. z_{d-1}, 1]:
//   G_i = sum h_k zt zt^T,   R_i = sum h_k W0[n][k] zt.
//
//  * fit_accum_kernel: one pass over W0 and the codes.  Lane (v, i) of a warp
//    takes coordinate i of vector v of each group of 32/d consecutive vectors
//    (32 consecutive floats of W0: coalesced) and keeps its G_i (upper
//    triangle) and R_i in registers: fp32 sums flushed into fp64 every 16
//    elements (below).  Lanes of one i are summed by an xor-shuffle tree,
//    warps in warp order in fp64, and each CTA writes one fp64 partial.
//  * fit_solve_kernel: sums the partials in CTA order (fp64), then thread i
//    forms theta_i = G_i^+ R_i in fp64: by Cholesky when every pivot is above
//    1e-8 of the largest diagonal entry (G_i comfortably positive definite,
//    pseudo-inverse = inverse), otherwise by a cyclic Jacobi
//    eigendecomposition with eigenvalues below 1e-12 of the largest taken as
//    zero (the minimum-norm solution when G_i is singular).
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace lcvq {

namespace {

constexpr int kFitThreads = 256;
constexpr int kFitWarps = kFitThreads / 32;
constexpr double kPinvRcond = 1e-12;

template <int D>
struct FitDims {
  static constexpr int P = D + 1;                 // zt length
  static constexpr int SG = P * (P + 1) / 2;      // upper triangle of G_i
  static constexpr int S = SG + P;                // G_i then R_i
  static constexpr int kVecPerWarp = 32 / D;      // vectors per warp step
};

// Per-lane sums.  Terms are accumulated in fp32 and flushed into fp64 every
// kFitFlush elements, so the rounding of a sum is at most kFitFlush * 2^-24
// of the sum of its terms' absolute values, however long the sum.  Without
// weights every G entry is an integer count, which fp32 holds exactly.
constexpr int kFitFlush = 16;
// grid-stride steps whose loads are in flight together, and CTAs per SM:
// measured best (4096 x 14336, d = 8): unweighted 4 steps at 2 CTAs per SM
// (128 registers, no spill); weighted 8 steps at 1 CTA (its fp64 mirror of G
// does not fit 128 registers)
template <bool kWeighted>
struct FitShape {
  static constexpr int kAhead = kWeighted ? 8 : 4;
  static constexpr int kMinBlocks = kWeighted ? 1 : 2;
};

template <int D, bool kWeighted>
__global__ void __launch_bounds__(kFitThreads, FitShape<kWeighted>::kMinBlocks) fit_accum_kernel(
    const float* __restrict__ W0, const uint32_t* __restrict__ codes, int64_t n_vec,
    int64_t groups, const float* __restrict__ h, double* __restrict__ partials) {
  using F = FitDims<D>;
  constexpr int kG = F::SG;
  // an fp64 mirror of G only where its terms are not integers
  constexpr int kG64 = kWeighted ? F::SG : 1;
  __shared__ double red[kFitWarps][D][F::S];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vl = lane / D, i = lane % D;
  float g32[kG], r32[F::P];
  double g64[kG64], r64[F::P];
#pragma unroll
  for (int s = 0; s < kG; ++s) g32[s] = 0.f;
#pragma unroll
  for (int s = 0; s < kG64; ++s) g64[s] = 0.0;
#pragma unroll
  for (int s = 0; s < F::P; ++s) r32[s] = 0.f, r64[s] = 0.0;

  const int64_t steps = ceil_div(n_vec, F::kVecPerWarp);
  const int64_t st0 = int64_t(blockIdx.x) * kFitWarps + warp;
  const int64_t stride = int64_t(gridDim.x) * kFitWarps;
  // channel of this lane's element, kept up to date without a division per element
  const int64_t vstep = (stride * F::kVecPerWarp) % groups;
  int64_t g = (st0 * F::kVecPerWarp + vl) % groups;
  int pending = 0;
  // kFitAhead steps per round, their loads issued together (latency hiding)
  constexpr int kFitAhead = FitShape<kWeighted>::kAhead;
  for (int64_t st = st0; st < steps; st += stride * kFitAhead) {
    float wv[kFitAhead];
    uint32_t cw[kFitAhead];
#pragma unroll
    for (int u = 0; u < kFitAhead; ++u) {
      const int64_t vec = (st + u * stride) * F::kVecPerWarp + vl;
      if (st + u * stride < steps && vec < n_vec) {
        wv[u] = __ldcs(W0 + vec * D + i);
        // the vector's 2D code bits start at bit 2 D vec of the packed stream
        const int64_t bit = vec * (2 * D);
        cw[u] = __ldg(codes + (bit >> 5)) >> (bit & 31);
      } else {
        wv[u] = 0.f;
        cw[u] = 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < kFitAhead; ++u) {
      const int64_t vec = (st + u * stride) * F::kVecPerWarp + vl;
      if (st + u * stride < steps && vec < n_vec) {
        const float w = wv[u];
        const uint32_t word = cw[u];
        // small integers to float without the conversion unit: OR the value
        // into the mantissa of 2^23 and subtract 2^23
        float zt[F::P];
#pragma unroll
        for (int j = 0; j < D; ++j)
          zt[j] = __int_as_float(0x4B000000 | static_cast<int>((word >> (2 * j)) & 3u)) - 8388608.0f;
        zt[D] = 1.f;
        const float hw = kWeighted ? __ldg(h + g * D + i) : 1.f;
        int s = 0;
#pragma unroll
        for (int a = 0; a < F::P; ++a) {
          const float ha = kWeighted ? hw * zt[a] : zt[a];
#pragma unroll
          for (int b = a; b < F::P; ++b) {
            g32[s] = fmaf(ha, zt[b], g32[s]);
            ++s;
          }
        }
        const float hwv = hw * w;
#pragma unroll
        for (int a = 0; a < F::P; ++a) r32[a] = fmaf(hwv, zt[a], r32[a]);
        if (++pending == kFitFlush) {
          pending = 0;
          if constexpr (kWeighted) {
#pragma unroll
            for (int q = 0; q < kG; ++q) g64[q] += g32[q], g32[q] = 0.f;
          }
#pragma unroll
          for (int q = 0; q < F::P; ++q) r64[q] += r32[q], r32[q] = 0.f;
        }
      }
      g += vstep;
      if (g >= groups) g -= groups;
    }
  }
  double gsum[kG];
#pragma unroll
  for (int q = 0; q < kG; ++q) gsum[q] = kWeighted ? g64[q < kG64 ? q : 0] + g32[q] : double(g32[q]);
#pragma unroll
  for (int q = 0; q < F::P; ++q) r64[q] += r32[q];
  // lanes of one coordinate i: lanes i, i + D, ...; xor tree over those
#pragma unroll
  for (int off = D; off < 32; off <<= 1) {
#pragma unroll
    for (int q = 0; q < kG; ++q) gsum[q] += __shfl_xor_sync(0xffffffffu, gsum[q], off);
#pragma unroll
    for (int q = 0; q < F::P; ++q) r64[q] += __shfl_xor_sync(0xffffffffu, r64[q], off);
  }
  if (lane < D) {
#pragma unroll
    for (int q = 0; q < F::SG; ++q) red[warp][lane][q] = gsum[q];
#pragma unroll
    for (int q = 0; q < F::P; ++q) red[warp][lane][F::SG + q] = r64[q];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < D * F::S; e += kFitThreads) {
    const int ii = e / F::S, q = e % F::S;
    double t = 0.0;
    for (int w2 = 0; w2 < kFitWarps; ++w2) t += red[w2][ii][q];
    partials[int64_t(blockIdx.x) * D * F::S + e] = t;
  }
}

// theta = G^+ R for a symmetric positive semi-definite P x P matrix G (row-major,
// overwritten), by cyclic Jacobi rotations G = V diag(lambda) V^T.
template <int P>
__device__ void pinv_solve(double (&G)[P][P], const double (&R)[P], double (&theta)[P]) {
  double V[P][P];
  for (int a = 0; a < P; ++a)
    for (int b = 0; b < P; ++b) V[a][b] = a == b ? 1.0 : 0.0;
  for (int sweep = 0; sweep < 64; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int a = 0; a < P; ++a) {
      diag += G[a][a] * G[a][a];
      for (int b = a + 1; b < P; ++b) off += G[a][b] * G[a][b];
    }
    if (off <= 1e-32 * (diag + off) || off == 0.0) break;
    for (int p = 0; p < P; ++p)
      for (int q = p + 1; q < P; ++q) {
        const double apq = G[p][q];
        if (apq == 0.0) continue;
        // rotation angle that zeroes G[p][q]: tan(phi) = t, the smaller root of
        // t^2 + 2 tau t - 1 = 0 with tau = (G[q][q] - G[p][p]) / (2 G[p][q])
        const double tau = (G[q][q] - G[p][p]) / (2.0 * apq);
        const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
        const double c = 1.0 / sqrt(1.0 + t * t), s = t * c;
        for (int r = 0; r < P; ++r) {  // G <- G J (columns p, q)
          const double gp = G[r][p], gq = G[r][q];
          G[r][p] = c * gp - s * gq;
          G[r][q] = s * gp + c * gq;
        }
        for (int r = 0; r < P; ++r) {  // G <- J^T G (rows p, q)
          const double gp = G[p][r], gq = G[q][r];
          G[p][r] = c * gp - s * gq;
          G[q][r] = s * gp + c * gq;
        }
        for (int r = 0; r < P; ++r) {  // V <- V J
          const double vp = V[r][p], vq = V[r][q];
          V[r][p] = c * vp - s * vq;
          V[r][q] = s * vp + c * vq;
        }
      }
  }
  double lmax = 0.0;
  for (int a = 0; a < P; ++a) lmax = fmax(lmax, fabs(G[a][a]));
  for (int a = 0; a < P; ++a) theta[a] = 0.0;
  for (int e = 0; e < P; ++e) {
    const double lam = G[e][e];
    if (!(lam > kPinvRcond * lmax)) continue;  // also drops lmax == 0 and NaN
    double vr = 0.0;
    for (int a = 0; a < P; ++a) vr += V[a][e] * R[a];
    const double f = vr / lam;
    for (int a = 0; a < P; ++a) theta[a] += f * V[a][e];
  }
}

// theta = G^-1 R by Cholesky factorization when G is comfortably positive
// definite: every pivot above kCholFloor of the largest diagonal entry (then
// the pseudo-inverse equals the inverse to fp64 rounding).  Leaves G intact
// and returns false otherwise, for the eigendecomposition path.
constexpr double kCholFloor = 1e-8;
template <int P>
__device__ bool cholesky_solve(const double (&G)[P][P], const double (&R)[P], double (&theta)[P]) {
  double L[P][P];
  double dmax = 0.0;
  for (int a = 0; a < P; ++a) dmax = fmax(dmax, G[a][a]);
  if (!(dmax > 0.0)) return false;
  for (int c = 0; c < P; ++c) {
    double sum = G[c][c];
    for (int k = 0; k < c; ++k) sum -= L[c][k] * L[c][k];
    if (!(sum > kCholFloor * dmax)) return false;
    const double lcc = sqrt(sum);
    L[c][c] = lcc;
    for (int r = c + 1; r < P; ++r) {
      double v = G[r][c];
      for (int k = 0; k < c; ++k) v -= L[r][k] * L[c][k];
      L[r][c] = v / lcc;
    }
  }
  double y[P];
  for (int r = 0; r < P; ++r) {  // L y = R
    double v = R[r];
    for (int k = 0; k < r; ++k) v -= L[r][k] * y[k];
    y[r] = v / L[r][r];
  }
  for (int r = P - 1; r >= 0; --r) {  // L^T theta = y
    double v = y[r];
    for (int k = r + 1; k < P; ++k) v -= L[k][r] * theta[k];
    theta[r] = v / L[r][r];
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(256) fit_solve_kernel(const double* __restrict__ partials,
                                                        int num_parts, float* __restrict__ A,
                                                        float* __restrict__ B) {
  using F = FitDims<D>;
  __shared__ double tot[D][F::S];
  for (int e = threadIdx.x; e < D * F::S; e += blockDim.x) {
    // partials in CTA order; loads batched 8 at a time, adds in order
    const double* src = partials + e;
    const int64_t pitch = int64_t(D) * F::S;
    double t = 0.0;
    int p = 0;
    for (; p + 8 <= num_parts; p += 8) {
      double v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = src[int64_t(p + q) * pitch];
#pragma unroll
      for (int q = 0; q < 8; ++q) t += v[q];
    }
    for (; p < num_parts; ++p) t += src[int64_t(p) * pitch];
    tot[e / F::S][e % F::S] = t;
  }
  __syncthreads();
  const int i = threadIdx.x;
  if (i >= D) return;
  double G[F::P][F::P], R[F::P], th[F::P];
  int s = 0;
  for (int a = 0; a < F::P; ++a)
    for (int b = a; b < F::P; ++b) {
      G[a][b] = tot[i][s];
      G[b][a] = tot[i][s];
      ++s;
    }
  for (int a = 0; a < F::P; ++a) R[a] = tot[i][F::SG + a];
  if (!cholesky_solve<F::P>(G, R, th)) pinv_solve<F::P>(G, R, th);
  for (int j = 0; j < D; ++j) A[i * D + j] = static_cast<float>(th[j]);
  B[i] = static_cast<float>(th[D]);
}

template <int D>
int fit_grid(int64_t n_vec) {
  const int64_t steps = ceil_div(n_vec, FitDims<D>::kVecPerWarp);
  int64_t g = ceil_div(steps, kFitWarps);
  const int64_t cap = int64_t(kNumSMsB200) * 4;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

template <int D>
cudaError_t launch_fit_t(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                         const float* h, float* A, float* B, double* partials, cudaStream_t s,
                         int* launches) {
  const int64_t groups = d_in / D;
  const int64_t n_vec = d_out * groups;
  const int grid = fit_grid<D>(n_vec);
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(packed);
  const int64_t gr = groups > 0 ? groups : 1;
  if (h)
    fit_accum_kernel<D, true><<<grid, kFitThreads, 0, s>>>(W0, codes, n_vec, gr, h, partials);
  else
    fit_accum_kernel<D, false><<<grid, kFitThreads, 0, s>>>(W0, codes, n_vec, gr, h, partials);
  ++*launches;
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  fit_solve_kernel<D><<<1, 256, 0, s>>>(partials, grid, A, B);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

size_t fit_partials_bytes(int64_t d_out, int64_t d_in, int d) {
  const int64_t n_vec = d > 0 ? d_out * (d_in / d) : 0;
  switch (d) {
    case 1: return size_t(fit_grid<1>(n_vec)) * 1 * FitDims<1>::S * sizeof(double);
    case 2: return size_t(fit_grid<2>(n_vec)) * 2 * FitDims<2>::S * sizeof(double);
    case 4: return size_t(fit_grid<4>(n_vec)) * 4 * FitDims<4>::S * sizeof(double);
    default: return size_t(fit_grid<8>(n_vec)) * 8 * FitDims<8>::S * sizeof(double);
  }
}

cudaError_t launch_fit_affine(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                              int d, const float* h, float* A, float* B, double* partials,
                              cudaStream_t s, int* launches) {
  switch (d) {
    case 1: return launch_fit_t<1>(W0, packed, d_out, d_in, h, A, B, partials, s, launches);
    case 2: return launch_fit_t<2>(W0, packed, d_out, d_in, h, A, B, partials, s, launches);
    case 4: return launch_fit_t<4>(W0, packed, d_out, d_in, h, A, B, partials, s, launches);
    default: return launch_fit_t<8>(W0, packed, d_out, d_in, h, A, B, partials, s, launches);
  }
}

}  // namespace lcvq

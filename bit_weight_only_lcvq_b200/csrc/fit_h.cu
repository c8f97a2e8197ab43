// Least-squares refit of the float part (A, B) under the full input Hessian H
// (decoupleQ page, eq. (5): the layer objective tr{(W~ - W0)^T H (W~ - W0)};
// section 3.3: with the integer part fixed the float part is a quadratic,
// solved in closed form), for LC-VQ's codewords c = A z + B (LC-QAT technical
// summary, Methodology 1).
//
// In storage order the objective is sum_n r_n^T H r_n, r_n = W~[n] - W0[n].
// With theta = [A | B] and zt = [z_0 .. z_{d-1}, 1] per vector, the decoded
// element W~[n][g d + i] = sum_a theta[i][a] zt[n][g][a] is linear in theta,
// and the normal equations couple every pair of vector positions (g, h):
//     L[(i,a),(j,b)] = sum_{g,h} H[g d + i][h d + j] S~[(g,a),(h,b)]
//     R[(i,a)]       = sum_g sum_k H[g d + i][k] T~[(g,a), k]
// with the code Gram S~[(g,a),(h,b)] = sum_n zt[n][g][a] zt[n][h][b] and the
// targets times the codes T~[(g,a), k] = sum_n zt[n][g][a] W0[n][k].
//
// Three steps:
//  1. fith_prep_kernel writes Q = [1 (64 columns) | Z | W0_hi | W0_lo] in bf16,
//     [d_out][64 + 3 d_in]: codes exactly, W0 as two bf16 terms (W0_hi =
//     bf16(W0), W0_lo = bf16(W0 - W0_hi); together within 2^-18 of W0).
//  2. One tcgen05 GEMM (tc_gemm.cu, kind Gram) forms C = P^T Q over the rows,
//     P = Q's first 64 + d_in columns: C[64 + g d + a][64 + h d + b] is S~ for
//     a, b < d, row 0 and column 0 hold the code column sums (the ones),
//     C[0][0] = d_out, and C[r][64 + d_in + k] + C[r][64 + 2 d_in + k] is T~.
//     Codes and ones are exact in bf16 and their products and sums are exact
//     in the fp32 accumulator (d_out * 9 < 2^24), so S~ is exact.
//  3. fith_contract_kernel combines C with H in fp64 (exact products of fp32
//     values) into per-CTA partials of L and R, in a fixed order;
//     fith_solve_kernel sums the partials in CTA order and solves the
//     d (d+1) x d (d+1) system: Cholesky when every pivot is above 1e-8 of
//     the largest diagonal entry, otherwise a parallel cyclic Jacobi
//     eigendecomposition with eigenvalues below 1e-12 of the largest taken as
//     zero (the minimum-norm solution), as the diagonal refit does.
// Every sum runs in a fixed order: the result is bitwise reproducible.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace lcvq {

namespace {

constexpr int kOnes = 64;                 // leading ones columns of Q
constexpr double kHPinvRcond = 1e-12;
constexpr double kHCholFloor = 1e-8;
constexpr int kPrepThreads = 256;

// ---------------------------------------------------------------- 1. Q
// One thread per 8 consecutive elements of a row: reads 8 fp32 of W0 and 2
// bytes of codes, writes 16 bytes to each of the Z, W0_hi and W0_lo blocks.
__global__ void __launch_bounds__(kPrepThreads) fith_prep_kernel(const float* __restrict__ W0,
                                                                 const uint8_t* __restrict__ packed,
                                                                 int64_t N, int64_t K,
                                                                 uint16_t* __restrict__ Q) {
  const int64_t per_row = K / 8 + kOnes / 8;  // work items per row
  const int64_t total = N * per_row;
  const int64_t ldq = kOnes + 3 * K;
  for (int64_t it = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; it < total;
       it += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = it / per_row, c = it % per_row;
    uint16_t* row = Q + n * ldq;
    if (c < kOnes / 8) {  // ones: bf16 1.0 = 0x3F80
      reinterpret_cast<uint4*>(row)[c] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
      continue;
    }
    const int64_t k0 = (c - kOnes / 8) * 8;
    const float4 w0 = __ldcs(reinterpret_cast<const float4*>(W0 + n * K + k0));
    const float4 w1 = __ldcs(reinterpret_cast<const float4*>(W0 + n * K + k0) + 1);
    const uint32_t cw = *reinterpret_cast<const uint16_t*>(packed + n * (K / 4) + k0 / 4);
    const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    uint32_t zq[4], hq[4], lq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float z0 = static_cast<float>((cw >> (4 * q)) & 3u);
      const float z1 = static_cast<float>((cw >> (4 * q + 2)) & 3u);
      zq[q] = pack_bf16x2(z0, z1);
      const float h0 = bf16_to_f32(f32_to_bf16(w[2 * q])), h1 = bf16_to_f32(f32_to_bf16(w[2 * q + 1]));
      hq[q] = pack_bf16x2(h0, h1);
      lq[q] = pack_bf16x2(w[2 * q] - h0, w[2 * q + 1] - h1);  // exact differences, then rounded
    }
    *reinterpret_cast<uint4*>(row + kOnes + k0) = make_uint4(zq[0], zq[1], zq[2], zq[3]);
    *reinterpret_cast<uint4*>(row + kOnes + K + k0) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
    *reinterpret_cast<uint4*>(row + kOnes + 2 * K + k0) = make_uint4(lq[0], lq[1], lq[2], lq[3]);
  }
}

// ---------------------------------------------------------------- 3a. contraction with H
// CTA c takes the vector positions g = c, c + G, ...; for each g it streams
// column chunks of H's rows g d .. g d + d - 1 and of C's rows (g, a) through
// shared memory.  Thread (i, a) of team tm (NP = d (d+1) threads per team)
// accumulates L[(i,a), (j,b)] for all (j, b) over the h-blocks h = tm, tm +
// kTeams, ... of each chunk, and R[(i,a)] over the chunk's k = tm, tm +
// kTeams, ...; at the end the teams are added in team order into the CTA's
// partial [L (NP x NP) | R (NP)] (fp64).
constexpr int kChunkCols = 256;  // columns of H and C per shared-memory chunk
constexpr int kTeams = 3;

template <int D>
struct FitHDims {
  static constexpr int NP = D * (D + 1);
  static constexpr int kThreads = ((kTeams * NP + 31) / 32) * 32;
  static constexpr int kCols = kChunkCols;     // a multiple of every d
  static constexpr int kPart = NP * NP + NP;   // doubles per CTA partial
};

template <int D>
__global__ void __launch_bounds__(FitHDims<D>::kThreads) fith_contract_kernel(
    const float* __restrict__ H, const float* __restrict__ C, int64_t K, double* __restrict__ partials) {
  using F = FitHDims<D>;
  constexpr int NP = F::NP, P1 = D + 1, COLS = F::kCols;
  // chunk: H rows [D][COLS], S~ rows [D+1][COLS], T~ rows [D+1][COLS] as its
  // hi and lo parts, and the ones column S~[(g,a),(., d)] = C[row(g,a)][0]
  __shared__ float sH[D][COLS];
  __shared__ float sS[P1][COLS];
  __shared__ float sTh[P1][COLS];
  __shared__ float sTl[P1][COLS];
  __shared__ float sOnes[P1];
  __shared__ double sRed[kTeams][NP + 1];
  const int tid = threadIdx.x;
  const int tm = tid / NP, me = tid % NP;
  const bool active = tm < kTeams;
  const int i = me / P1, a = me % P1;
  const int64_t ldc = kOnes + 3 * K;
  const int64_t ng = K / D;
  double accL[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) accL[q] = 0.0;
  double accR = 0.0;

  for (int64_t g = blockIdx.x; g < ng; g += gridDim.x) {
    // C row of (g, a): the ones row 0 for a = d
    auto crow = [&](int aa) -> const float* {
      return C + (aa < D ? (kOnes + g * D + aa) : 0) * ldc;
    };
    __syncthreads();
    if (tid < P1) sOnes[tid] = crow(tid)[0];
    for (int64_t c0 = 0; c0 < K; c0 += COLS) {
      const int ncols = static_cast<int>(K - c0 < COLS ? K - c0 : COLS);  // multiple of D
      __syncthreads();  // the previous chunk is consumed
      for (int e = tid; e < D * COLS; e += blockDim.x) {
        const int r = e / COLS, c = e % COLS;
        sH[r][c] = c < ncols ? H[(g * D + r) * K + c0 + c] : 0.f;
      }
      for (int e = tid; e < P1 * COLS; e += blockDim.x) {
        const int r = e / COLS, c = e % COLS;
        const float* cr = crow(r);
        sS[r][c] = c < ncols ? cr[kOnes + c0 + c] : 0.f;
        sTh[r][c] = c < ncols ? cr[kOnes + K + c0 + c] : 0.f;
        sTl[r][c] = c < ncols ? cr[kOnes + 2 * K + c0 + c] : 0.f;
      }
      __syncthreads();
      if (active) {
        // L: h-blocks tm, tm + kTeams, ... of the chunk
        for (int hb = tm; hb < ncols / D; hb += kTeams) {
          double hv[D], sv[P1];
#pragma unroll
          for (int j = 0; j < D; ++j) hv[j] = static_cast<double>(sH[i][hb * D + j]);
#pragma unroll
          for (int b = 0; b < D; ++b) sv[b] = static_cast<double>(sS[a][hb * D + b]);
          sv[D] = static_cast<double>(sOnes[a]);
#pragma unroll
          for (int j = 0; j < D; ++j)
#pragma unroll
            for (int b = 0; b < P1; ++b) accL[j * P1 + b] = fma(hv[j], sv[b], accL[j * P1 + b]);
        }
        // R: columns tm, tm + kTeams, ... of the chunk
        for (int c = tm; c < ncols; c += kTeams) {
          const double hv = static_cast<double>(sH[i][c]);
          accR = fma(hv, static_cast<double>(sTh[a][c]), accR);
          accR = fma(hv, static_cast<double>(sTl[a][c]), accR);
        }
      }
    }
  }
  // teams in team order into the CTA partial: one L row (i,a) at a time
  double* out = partials + int64_t(blockIdx.x) * F::kPart;
#pragma unroll
  for (int q = 0; q < NP; ++q) {  // column (j, b) = q of every row
    __syncthreads();
    if (active) sRed[tm][me] = accL[q];
    __syncthreads();
    if (tid < NP) {
      double v = 0.0;
      for (int t = 0; t < kTeams; ++t) v += sRed[t][tid];
      out[tid * NP + q] = v;  // L[(i,a) = tid][(j,b) = q]
    }
  }
  __syncthreads();
  if (active) sRed[tm][me] = accR;
  __syncthreads();
  if (tid < NP) {
    double v = 0.0;
    for (int t = 0; t < kTeams; ++t) v += sRed[t][tid];
    out[NP * NP + tid] = v;
  }
}

// ---------------------------------------------------------------- 3b. solve
// One CTA.  Sums the partials in CTA order (thread per value), then solves
// L theta = R in shared memory.
constexpr int kSolveThreads = 256;

template <int NP>
__device__ bool chol_solve_par(double (*G)[NP], double* R, double* th, double* sdiag) {
  // in place: lower factor in G; returns false on a pivot below the floor
  const int t = threadIdx.x;
  __shared__ int ok;
  if (t == 0) {
    double dmax = 0.0;
    for (int c = 0; c < NP; ++c) dmax = fmax(dmax, G[c][c]);
    *sdiag = dmax;
    ok = dmax > 0.0;
  }
  __syncthreads();
  if (!ok) return false;
  const double dmax = *sdiag;
  for (int c = 0; c < NP; ++c) {
    if (t == 0) {
      const double piv = G[c][c];
      if (!(piv > kHCholFloor * dmax)) ok = 0;
      else G[c][c] = sqrt(piv);
    }
    __syncthreads();
    if (!ok) return false;
    const double lcc = G[c][c];
    for (int r = c + 1 + t; r < NP; r += blockDim.x) G[r][c] /= lcc;
    __syncthreads();
    // trailing update of the lower triangle: G[r][s] -= L[r][c] L[s][c], c < s <= r
    const int m = NP - c - 1;
    for (int e = t; e < m * m; e += blockDim.x) {
      const int r = c + 1 + e / m, s = c + 1 + e % m;
      if (s <= r) G[r][s] -= G[r][c] * G[s][c];
    }
    __syncthreads();
  }
  if (t == 0) {
    double y[NP];
    for (int r = 0; r < NP; ++r) {  // L y = R
      double v = R[r];
      for (int k = 0; k < r; ++k) v -= G[r][k] * y[k];
      y[r] = v / G[r][r];
    }
    for (int r = NP - 1; r >= 0; --r) {  // L^T theta = y
      double v = y[r];
      for (int k = r + 1; k < NP; ++k) v -= G[k][r] * th[k];
      th[r] = v / G[r][r];
    }
  }
  __syncthreads();
  return true;
}

// Parallel cyclic Jacobi (round-robin ordering: NP / 2 disjoint rotations per
// round, NP - 1 rounds per sweep) on the symmetric G, V accumulating the
// rotations; then theta = sum over eigenvalues above rcond of v (v^T R) / lambda.
template <int NP>
__device__ void jacobi_pinv_par(double (*G)[NP], double (*V)[NP], const double* R, double* th) {
  const int t = threadIdx.x;
  __shared__ double cs[NP / 2][2];
  __shared__ int pq[NP / 2][2];
  __shared__ int done;
  for (int e = t; e < NP * NP; e += blockDim.x) V[e / NP][e % NP] = (e / NP == e % NP) ? 1.0 : 0.0;
  __syncthreads();
  constexpr int m = NP - 1;
  for (int sweep = 0; sweep < 64; ++sweep) {
    if (t == 0) {
      double off = 0.0, diag = 0.0;
      for (int x = 0; x < NP; ++x) {
        diag += G[x][x] * G[x][x];
        for (int y = x + 1; y < NP; ++y) off += G[x][y] * G[x][y];
      }
      done = (off <= 1e-32 * (diag + off)) || off == 0.0;
    }
    __syncthreads();
    if (done) break;
    for (int round = 0; round < m; ++round) {
      if (t < NP / 2) {
        int p, q;
        if (t == 0) {
          p = m;
          q = round;
        } else {
          p = (round + t) % m;
          q = (round - t + m) % m;
        }
        if (p > q) {
          const int x = p;
          p = q;
          q = x;
        }
        pq[t][0] = p;
        pq[t][1] = q;
        const double apq = G[p][q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (G[q][q] - G[p][p]) / (2.0 * apq);
          const double tt = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + tt * tt);
          s = tt * c;
        }
        cs[t][0] = c;
        cs[t][1] = s;
      }
      __syncthreads();
      // G <- G J and V <- V J: columns p, q of every row, for each pair
      for (int e = t; e < (NP / 2) * NP; e += blockDim.x) {
        const int k = e / NP, r = e % NP;
        const int p = pq[k][0], q = pq[k][1];
        const double c = cs[k][0], s = cs[k][1];
        const double gp = G[r][p], gq = G[r][q];
        G[r][p] = c * gp - s * gq;
        G[r][q] = s * gp + c * gq;
        const double vp = V[r][p], vq = V[r][q];
        V[r][p] = c * vp - s * vq;
        V[r][q] = s * vp + c * vq;
      }
      __syncthreads();
      // G <- J^T G: rows p, q of every column
      for (int e = t; e < (NP / 2) * NP; e += blockDim.x) {
        const int k = e / NP, r = e % NP;
        const int p = pq[k][0], q = pq[k][1];
        const double c = cs[k][0], s = cs[k][1];
        const double gp = G[p][r], gq = G[q][r];
        G[p][r] = c * gp - s * gq;
        G[q][r] = s * gp + c * gq;
      }
      __syncthreads();
    }
  }
  if (t == 0) {
    double lmax = 0.0;
    for (int x = 0; x < NP; ++x) lmax = fmax(lmax, fabs(G[x][x]));
    for (int x = 0; x < NP; ++x) th[x] = 0.0;
    for (int e = 0; e < NP; ++e) {
      const double lam = G[e][e];
      if (!(lam > kHPinvRcond * lmax)) continue;  // also drops lmax == 0 and NaN
      double vr = 0.0;
      for (int x = 0; x < NP; ++x) vr += V[x][e] * R[x];
      const double f = vr / lam;
      for (int x = 0; x < NP; ++x) th[x] += f * V[x][e];
    }
  }
  __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(kSolveThreads) fith_solve_kernel(const double* __restrict__ partials,
                                                                   int num_parts, float* __restrict__ A,
                                                                   float* __restrict__ B) {
  using F = FitHDims<D>;
  constexpr int NP = F::NP;
  extern __shared__ __align__(16) unsigned char fsm[];
  double (*G)[NP] = reinterpret_cast<double (*)[NP]>(fsm);
  double (*G0)[NP] = G + NP;           // a copy for the Jacobi fallback
  double (*V)[NP] = G0 + NP;
  double* R = reinterpret_cast<double*>(V + NP);
  double* th = R + NP;
  double* sdiag = th + NP;
  const int t = threadIdx.x;
  for (int v = t; v < F::kPart; v += blockDim.x) {
    double acc = 0.0;
    for (int c = 0; c < num_parts; ++c) acc += partials[int64_t(c) * F::kPart + v];
    if (v < NP * NP) {
      // symmetrize: the partials hold the full L; average mirrored entries in a
      // fixed order so both triangles agree bit for bit
      G[v / NP][v % NP] = acc;
    } else {
      R[v - NP * NP] = acc;
    }
  }
  __syncthreads();
  for (int e = t; e < NP * NP; e += blockDim.x) {
    const int r = e / NP, c = e % NP;
    if (r < c) {
      const double s = 0.5 * (G[r][c] + G[c][r]);
      G0[r][c] = s;
      G0[c][r] = s;
    } else if (r == c) {
      G0[r][r] = G[r][r];
    }
  }
  __syncthreads();
  for (int e = t; e < NP * NP; e += blockDim.x) G[e / NP][e % NP] = G0[e / NP][e % NP];
  __syncthreads();
  if (!chol_solve_par<NP>(G, R, th, sdiag)) {
    jacobi_pinv_par<NP>(G0, V, R, th);
  }
  if (t < D * D) A[t] = static_cast<float>(th[(t / D) * (D + 1) + (t % D)]);
  if (t < D) B[t] = static_cast<float>(th[t * (D + 1) + D]);
}

template <int D>
size_t solve_smem() {
  constexpr int NP = FitHDims<D>::NP;
  return size_t(3) * NP * NP * 8 + size_t(2) * NP * 8 + 16;
}

int contract_grid(int64_t ng) {
  int64_t g = 2 * kNumSMsB200;
  if (ng < g) g = ng;
  return g < 1 ? 1 : static_cast<int>(g);
}

template <int D>
cudaError_t launch_fith_t(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                          const float* H, float* A, float* B, void* scratch, unsigned int* err,
                          cudaStream_t s, int* launches) {
  using F = FitHDims<D>;
  const int64_t ldq = kOnes + 3 * d_in;
  char* base = static_cast<char*>(scratch);
  uint16_t* Q = reinterpret_cast<uint16_t*>(base);
  const size_t q_bytes = (size_t(d_out) * ldq * 2 + 255) / 256 * 256;
  float* C = reinterpret_cast<float*>(base + q_bytes);
  const size_t c_bytes = (size_t(kOnes + d_in) * ldq * 4 + 255) / 256 * 256;
  double* partials = reinterpret_cast<double*>(base + q_bytes + c_bytes);
  {
    const int64_t items = d_out * (d_in / 8 + kOnes / 8);
    int64_t grid = ceil_div(items, kPrepThreads);
    if (grid > 8 * kNumSMsB200) grid = 8 * kNumSMsB200;
    fith_prep_kernel<<<static_cast<unsigned>(grid), kPrepThreads, 0, s>>>(W0, packed, d_out, d_in, Q);
    ++*launches;
    if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  }
  if (cudaError_t e = launch_tc_gram(Q, d_out, kOnes + d_in, ldq, C, err, s, launches);
      e != cudaSuccess)
    return e;
  const int grid = contract_grid(d_in / D);
  fith_contract_kernel<D><<<grid, F::kThreads, 0, s>>>(H, C, d_in, partials);
  ++*launches;
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  auto sk = fith_solve_kernel<D>;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(sk), solve_smem<D>());
      e != cudaSuccess)
    return e;
  sk<<<1, kSolveThreads, solve_smem<D>(), s>>>(partials, grid, A, B);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

size_t fith_scratch_bytes(int64_t d_out, int64_t d_in, int d) {
  const int64_t ldq = kOnes + 3 * d_in;
  const size_t q_bytes = (size_t(d_out) * ldq * 2 + 255) / 256 * 256;
  const size_t c_bytes = (size_t(kOnes + d_in) * ldq * 4 + 255) / 256 * 256;
  const int np = d * (d + 1);
  const size_t p_bytes = size_t(contract_grid(d_in / (d > 0 ? d : 1))) * size_t(np * np + np) * 8;
  return q_bytes + c_bytes + p_bytes;
}

cudaError_t launch_fit_affine_h(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                                int d, const float* H, float* A, float* B, void* scratch,
                                unsigned int* err, cudaStream_t s, int* launches) {
  if (d_out == 0 || d_in == 0) {  // empty sums: the minimum-norm solution is zero
    if (cudaError_t e = cudaMemsetAsync(A, 0, size_t(d) * d * 4, s); e != cudaSuccess) return e;
    return cudaMemsetAsync(B, 0, size_t(d) * 4, s);
  }
  switch (d) {
    case 1: return launch_fith_t<1>(W0, packed, d_out, d_in, H, A, B, scratch, err, s, launches);
    case 2: return launch_fith_t<2>(W0, packed, d_out, d_in, H, A, B, scratch, err, s, launches);
    case 4: return launch_fith_t<4>(W0, packed, d_out, d_in, H, A, B, scratch, err, s, launches);
    default: return launch_fith_t<8>(W0, packed, d_out, d_in, H, A, B, scratch, err, s, launches);
  }
}

}  // namespace lcvq

// lcvq_oracle.cpp -- plain C++17 fp64 reference of the LC-VQ hot path.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// CPU-baseline legs of bench.py load it (through oracle/cpp.py).  The CUDA
// library never links or loads it, and it includes nothing from the library:
// the two share no code, header, table or constant.
//
// It writes out the same definitions as the numpy oracle (oracle/lcvq_oracle.py),
// from the same passages:
//   * LC-QAT page (gist.science technical summary of "LC-QAT: Data-Efficient
//     2-Bit QAT for LLMs via Linear-Constrained Vector Quantization"),
//     Methodology 1: codewords c = A z + B, z in {0,1,2,3}^d, A (d x d) and B
//     (d) shared by one weight matrix; finding the code is rounding and
//     clamping; gradients flow through the linear map.
//     Methodology 3: proxy weights are rounded and clamped to W_z, decoded as
//     A W_z + B and used in the layer's matmul; the backward passes the
//     rounding straight through (the STE of the gradient-estimator ablation).
//   * decoupleQ page, eq. (1): the layer is Y = X W~ (W~ stored here as
//     [d_out][d_in], so Y[m][n] = sum_k X[m][k] W~[n][k]).
//   * decoupleQ page, eq. (5) and section 3.3: the (A, B) refits for fixed
//     codes (diagonal and full Hessian); eq. (8)-(11) with LC-QAT's
//     Methodology 2: the H-aware sequential code assignment.
//   * LC-QAT page, the gradient estimator DGE: a smooth curve through the
//     rounding (the curve itself is a reading; see lco_dge_phi).
//
// Readings where the pages are silent (the same as the numpy oracle's):
// round half to even; clamp to [0, 3]; NaN -> 0, +inf -> 3, -inf -> 0; the STE
// mask is 0 <= W_p <= 3 on the proxy weight; vectors are d consecutive
// elements along d_in; A acts on column vectors, c_i = sum_j A[i][j] z_j;
// packed format V1 (4 codes per byte, LSB first; mask 8 bits per byte, LSB
// first).
//
// Arithmetic: fp64 throughout (inputs are fp64; the callers widen fp32/bf16
// values exactly).  Every output element is computed by one thread in a fixed
// order, so results do not depend on the thread count; threads only split the
// output rows.  Each dot product over d_in is kept as 8 interleaved partial
// sums (index mod 8) added at the end, a fixed order that lets the compiler
// use vector registers; an axpy-style sum (dX, G) runs over its index in
// increasing order.  Every floating result comes with the normaliser D = the
// sum of the absolute values of its terms, propagated through each output's
// own terms (the parity metric is |got - ref| / D).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr double kCodeMax = 3.0;

// rows [0, n) split into contiguous ranges, one per thread
template <class F>
void parallel_rows(int64_t n, int threads, F fn) {
  if (threads < 1) threads = 1;
  if (int64_t(threads) > n) threads = n > 0 ? int(n) : 1;
  if (threads == 1) {
    fn(int64_t(0), n);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t per = (n + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    const int64_t a = t * per, b = std::min(n, a + per);
    if (a >= b) break;
    pool.emplace_back([=] { fn(a, b); });
  }
  for (auto& th : pool) th.join();
}

// the code of one proxy weight: rint (ties to even) then clamp to [0, 3]
uint8_t code_of(double w) {
  if (std::isnan(w)) return 0;
  double r = std::nearbyint(w);  // default rounding mode: to nearest, ties to even
  if (r < 0.0) r = 0.0;
  if (r > kCodeMax) r = kCodeMax;
  return static_cast<uint8_t>(r);
}

// decode one row: w[g d + i] = sum_j A[i][j] z[g d + j] + B[i]
template <class Z>
void decode_row(const Z* z, int64_t K, int d, const double* A, const double* B, double* w,
                double* wabs) {
  for (int64_t g = 0; g < K / d; ++g) {
    for (int i = 0; i < d; ++i) {
      double c = 0.0;
      for (int j = 0; j < d; ++j) c += A[i * d + j] * double(z[g * d + j]);
      c += B[i];
      w[g * d + i] = c;
      if (wabs) wabs[g * d + i] = std::fabs(c);
    }
  }
}

// sum_k a[k] b[k] as 8 interleaved partial sums (k mod 8), added pairwise
double dot8(const double* a, const double* b, int64_t K) {
  double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int64_t k = 0;
  for (; k + 8 <= K; k += 8)
    for (int l = 0; l < 8; ++l) s[l] += a[k + l] * b[k + l];
  for (int l = 0; k < K; ++k, ++l) s[l] += a[k] * b[k];
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

void axpy(double* y, double a, const double* x, int64_t K) {
  for (int64_t k = 0; k < K; ++k) y[k] += a * x[k];
}

// the codes of row n: z + n K, or unpacked from format V1 into buf
template <class Z>
const Z* row_codes(const Z* z, const uint8_t* packed, int64_t n, int64_t K, Z* buf) {
  if (packed == nullptr) return z + n * K;
  const uint8_t* p = packed + n * (K / 4);
  for (int64_t b = 0; b < K / 4; ++b)
    for (int q = 0; q < 4; ++q) buf[4 * b + q] = Z((p[b] >> (2 * q)) & 3u);
  return buf;
}

// Y[m][n] = sum_k X[m][k] W~[n][k]; D[m][n] = sum_k |X[m][k]| |W~[n][k]|.
// The codes come as z [N][K] or, when packed is non-null, in format V1.
template <class Z>
void forward_t(const double* X, int64_t M, const Z* z, const uint8_t* packed, int64_t N,
               int64_t K, int d, const double* A, const double* B, double* Y, double* D,
               int threads) {
  std::vector<double> Xa(size_t(M) * size_t(K));
  for (int64_t i = 0; i < M * K; ++i) Xa[i] = std::fabs(X[i]);
  constexpr int64_t kRows = 8;  // weight rows decoded at once
  parallel_rows(N, threads, [&](int64_t n0, int64_t n1) {
    std::vector<double> w(size_t(kRows) * K), wa(size_t(kRows) * K);
    std::vector<Z> zbuf(packed ? K : 0);
    for (int64_t nb = n0; nb < n1; nb += kRows) {
      const int64_t nr = std::min(kRows, n1 - nb);
      for (int64_t r = 0; r < nr; ++r)
        decode_row(row_codes(z, packed, nb + r, K, zbuf.data()), K, d, A, B, &w[r * K],
                   &wa[r * K]);
      for (int64_t m = 0; m < M; ++m)
        for (int64_t r = 0; r < nr; ++r) {
          Y[m * N + nb + r] = dot8(X + m * K, &w[r * K], K);
          D[m * N + nb + r] = dot8(&Xa[m * K], &wa[r * K], K);
        }
    }
  });
}

// The straight-through backward (Methodology 1 and 3):
//   dX[m][k]  = sum_n dY[m][n] W~[n][k]
//   G[n][k]   = sum_m dY[m][n] X[m][k]                    (dL/dW~, per row)
//   dA[i][j]  = sum_{n,g} G[n][g d + i] z[n][g d + j]
//   dB[i]     = sum_{n,g} G[n][g d + i]
//   dWp[n][g d + j] = mask[n][g d + j] sum_i A[i][j] G[n][g d + i]
// with the normalisers D_dX = |dY| |W~|, D_G = |dY|^T |X| and the others from
// D_G as their own terms' absolute values.  dA and dB are summed over the
// rows n in increasing order from per-row partials.
template <class Z>
void backward_t(const double* X, const double* dY, int64_t M, const Z* z, const uint8_t* mask,
                int64_t N, int64_t K, int d, const double* A, const double* B, double* dX,
                double* D_dX, double* dA, double* D_dA, double* dB, double* D_dB, double* dWp,
                double* D_dWp, int threads) {
  // W~ and |W~| once, shared read-only
  std::vector<double> W(size_t(N) * K), Wa(size_t(N) * K);
  parallel_rows(N, threads, [&](int64_t a, int64_t b) {
    for (int64_t n = a; n < b; ++n) decode_row(z + n * K, K, d, A, B, &W[n * K], &Wa[n * K]);
  });
  // dX, rows m split over threads; each element sums n = 0 .. N-1 in order
  parallel_rows(M, threads, [&](int64_t m0, int64_t m1) {
    for (int64_t m = m0; m < m1; ++m) {
      double* out = dX + m * K;
      double* outD = D_dX + m * K;
      std::fill(out, out + K, 0.0);
      std::fill(outD, outD + K, 0.0);
      for (int64_t n = 0; n < N; ++n) {
        const double a = dY[m * N + n];
        axpy(out, a, &W[n * K], K);
        axpy(outD, std::fabs(a), &Wa[n * K], K);
      }
    }
  });
  W.clear();
  W.shrink_to_fit();
  Wa.clear();
  Wa.shrink_to_fit();
  // |X| once
  std::vector<double> Xa(size_t(M) * K);
  for (int64_t i = 0; i < M * K; ++i) Xa[i] = std::fabs(X[i]);
  const int dd = d * d;
  std::vector<double> pA(size_t(N) * dd), pDA(size_t(N) * dd), pB(size_t(N) * d),
      pDB(size_t(N) * d);
  parallel_rows(N, threads, [&](int64_t n0, int64_t n1) {
    std::vector<double> G(K), DG(K);
    for (int64_t n = n0; n < n1; ++n) {
      std::fill(G.begin(), G.end(), 0.0);
      std::fill(DG.begin(), DG.end(), 0.0);
      for (int64_t m = 0; m < M; ++m) {  // G[n][:] = sum_m dY[m][n] X[m][:], m in order
        const double a = dY[m * N + n];
        axpy(G.data(), a, X + m * K, K);
        axpy(DG.data(), std::fabs(a), &Xa[m * K], K);
      }
      double* a_ = &pA[n * dd];
      double* da_ = &pDA[n * dd];
      double* b_ = &pB[n * d];
      double* db_ = &pDB[n * d];
      std::fill(a_, a_ + dd, 0.0);
      std::fill(da_, da_ + dd, 0.0);
      std::fill(b_, b_ + d, 0.0);
      std::fill(db_, db_ + d, 0.0);
      const Z* zr = z + n * K;
      for (int64_t g = 0; g < K / d; ++g) {
        const double* Gg = &G[g * d];
        const double* DGg = &DG[g * d];
        for (int i = 0; i < d; ++i) {
          for (int j = 0; j < d; ++j) {
            a_[i * d + j] += Gg[i] * double(zr[g * d + j]);
            da_[i * d + j] += DGg[i] * double(zr[g * d + j]);
          }
          b_[i] += Gg[i];
          db_[i] += DGg[i];
        }
        if (dWp) {
          for (int j = 0; j < d; ++j) {
            const int64_t k = g * d + j;
            const bool on = mask[n * K + k] != 0;
            double v = 0.0, vd = 0.0;
            for (int i = 0; i < d; ++i) {
              v += A[i * d + j] * Gg[i];
              vd += std::fabs(A[i * d + j]) * DGg[i];
            }
            dWp[n * K + k] = on ? v : 0.0;
            D_dWp[n * K + k] = on ? vd : 0.0;
          }
        }
      }
    }
  });
  for (int t = 0; t < dd; ++t) dA[t] = D_dA[t] = 0.0;
  for (int t = 0; t < d; ++t) dB[t] = D_dB[t] = 0.0;
  for (int64_t n = 0; n < N; ++n) {  // rows in increasing order
    for (int t = 0; t < dd; ++t) {
      dA[t] += pA[n * dd + t];
      D_dA[t] += pDA[n * dd + t];
    }
    for (int t = 0; t < d; ++t) {
      dB[t] += pB[n * d + t];
      D_dB[t] += pDB[n * d + t];
    }
  }
}

// Eigen-decomposition of the symmetric n x n matrix S (row-major; destroyed):
// on return the diagonal of S holds the eigenvalues and the columns of V
// (row-major) the eigenvectors.  Cyclic Jacobi: every off-diagonal pair (p, q)
// in turn is zeroed by the plane rotation of the symmetric Schur step (Golub
// and Van Loan, "Matrix Computations", the cyclic Jacobi method), sweeps until
// the off-diagonal part is below 1e-30 of the whole (squared norms).
void jacobi_eigen(std::vector<double>& S, int n, std::vector<double>& V) {
  V.assign(size_t(n) * size_t(n), 0.0);
  for (int i = 0; i < n; ++i) V[size_t(i) * n + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, all = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = 0; q < n; ++q) {
        const double v = S[size_t(p) * n + q] * S[size_t(p) * n + q];
        all += v;
        if (p != q) off += v;
      }
    if (off <= 1e-30 * all) break;
    for (int p = 0; p < n - 1; ++p)
      for (int q = p + 1; q < n; ++q) {
        const double apq = S[size_t(p) * n + q];
        if (apq == 0.0) continue;
        const double app = S[size_t(p) * n + p], aqq = S[size_t(q) * n + q];
        const double tau = (aqq - app) / (2.0 * apq);
        const double t = (tau >= 0.0 ? 1.0 : -1.0) / (std::fabs(tau) + std::sqrt(1.0 + tau * tau));
        const double c = 1.0 / std::sqrt(1.0 + t * t), sn = t * c;
        for (int k = 0; k < n; ++k) {  // S J
          const double skp = S[size_t(k) * n + p], skq = S[size_t(k) * n + q];
          S[size_t(k) * n + p] = c * skp - sn * skq;
          S[size_t(k) * n + q] = sn * skp + c * skq;
        }
        for (int k = 0; k < n; ++k) {  // J^T (S J)
          const double spk = S[size_t(p) * n + k], sqk = S[size_t(q) * n + k];
          S[size_t(p) * n + k] = c * spk - sn * sqk;
          S[size_t(q) * n + k] = sn * spk + c * sqk;
        }
        for (int k = 0; k < n; ++k) {  // V J
          const double vkp = V[size_t(k) * n + p], vkq = V[size_t(k) * n + q];
          V[size_t(k) * n + p] = c * vkp - sn * vkq;
          V[size_t(k) * n + q] = sn * vkp + c * vkq;
        }
      }
  }
}

// x = G^+ r for the symmetric n x n G: the eigenvalues at or below rcond of the
// largest in magnitude count as zero (the minimum-norm least-squares solution)
constexpr double kPinvRcond = 1e-12;
void pinv_solve(std::vector<double> G, int n, const double* r, double* x) {
  std::vector<double> V;
  jacobi_eigen(G, n, V);
  double lmax = 0.0;
  for (int e = 0; e < n; ++e) lmax = std::max(lmax, std::fabs(G[size_t(e) * n + e]));
  for (int i = 0; i < n; ++i) x[i] = 0.0;
  for (int e = 0; e < n; ++e) {
    const double lam = G[size_t(e) * n + e];
    if (!(std::fabs(lam) > kPinvRcond * lmax)) continue;
    double vr = 0.0;
    for (int i = 0; i < n; ++i) vr += V[size_t(i) * n + e] * r[i];
    for (int i = 0; i < n; ++i) x[i] += V[size_t(i) * n + e] * (vr / lam);
  }
}

}  // namespace

extern "C" {

// Assign (Methodology 1 and 3: rounding and clamping): z = clamp(rint(Wp), 0, 3)
// as u8 [N][K], mask = (0 <= Wp <= 3) as u8 [N][K].
void lco_assign(const double* Wp, int64_t n, uint8_t* z, uint8_t* mask) {
  for (int64_t i = 0; i < n; ++i) {
    const double w = Wp[i];
    z[i] = code_of(w);
    mask[i] = (w >= 0.0 && w <= kCodeMax) ? 1 : 0;  // false for NaN
  }
}

// Format V1: element k of a row in byte k / 4, bits 2 (k % 4) .. + 1.
void lco_pack_codes(const uint8_t* z, int64_t N, int64_t K, uint8_t* packed) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < K / 4; ++b) {
      uint8_t v = 0;
      for (int q = 0; q < 4; ++q) v |= uint8_t((z[n * K + 4 * b + q] & 3u) << (2 * q));
      packed[n * (K / 4) + b] = v;
    }
}

void lco_unpack_codes(const uint8_t* packed, int64_t N, int64_t K, uint8_t* z) {
  for (int64_t b = 0; b < N * (K / 4); ++b)  // byte b holds elements 4b .. 4b + 3
    for (int q = 0; q < 4; ++q) z[4 * b + q] = (packed[b] >> (2 * q)) & 3u;
}

// Mask bits: element k of a row in byte k / 8, bit k % 8.
void lco_pack_mask(const uint8_t* mask, int64_t N, int64_t K, uint8_t* bits) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < K / 8; ++b) {
      uint8_t v = 0;
      for (int q = 0; q < 8; ++q) v |= uint8_t((mask[n * K + 8 * b + q] & 1u) << q);
      bits[n * (K / 8) + b] = v;
    }
}

void lco_unpack_mask(const uint8_t* bits, int64_t N, int64_t K, uint8_t* mask) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) mask[n * K + k] = (bits[n * (K / 8) + k / 8] >> (k % 8)) & 1u;
}

// Decode (Methodology 1: c = A z + B): W [N][K] and, if non-null, |W|.
// z holds u8 codes (z8) or fp64 values (zf: the STE surrogate's clamped
// proxy weights).
void lco_decode_z8(const uint8_t* z, int64_t N, int64_t K, int d, const double* A,
                   const double* B, double* W, int threads) {
  parallel_rows(N, threads, [&](int64_t a, int64_t b) {
    for (int64_t n = a; n < b; ++n) decode_row(z + n * K, K, d, A, B, W + n * K, nullptr);
  });
}
void lco_decode_zf(const double* z, int64_t N, int64_t K, int d, const double* A,
                   const double* B, double* W, int threads) {
  parallel_rows(N, threads, [&](int64_t a, int64_t b) {
    for (int64_t n = a; n < b; ++n) decode_row(z + n * K, K, d, A, B, W + n * K, nullptr);
  });
}

// Forward (decoupleQ eq. (1); Methodology 3): Y, D [M][N].
void lco_forward_z8(const double* X, int64_t M, const uint8_t* z, int64_t N, int64_t K, int d,
                    const double* A, const double* B, double* Y, double* D, int threads) {
  forward_t(X, M, z, static_cast<const uint8_t*>(nullptr), N, K, d, A, B, Y, D, threads);
}
void lco_forward_zf(const double* X, int64_t M, const double* z, int64_t N, int64_t K, int d,
                    const double* A, const double* B, double* Y, double* D, int threads) {
  forward_t(X, M, z, static_cast<const uint8_t*>(nullptr), N, K, d, A, B, Y, D, threads);
}
// the same with the codes in format V1 (unpacked row by row)
void lco_forward_packed(const double* X, int64_t M, const uint8_t* packed, int64_t N, int64_t K,
                        int d, const double* A, const double* B, double* Y, double* D,
                        int threads) {
  forward_t(X, M, static_cast<const uint8_t*>(nullptr), packed, N, K, d, A, B, Y, D, threads);
}

// STE backward (Methodology 1 and 3).  mask is u8 [N][K]; dWp/D_dWp may be null.
void lco_backward_z8(const double* X, const double* dY, int64_t M, const uint8_t* z,
                     const uint8_t* mask, int64_t N, int64_t K, int d, const double* A,
                     const double* B, double* dX, double* D_dX, double* dA, double* D_dA,
                     double* dB, double* D_dB, double* dWp, double* D_dWp, int threads) {
  backward_t(X, dY, M, z, mask, N, K, d, A, B, dX, D_dX, dA, D_dA, dB, D_dB, dWp, D_dWp, threads);
}
void lco_backward_zf(const double* X, const double* dY, int64_t M, const double* z,
                     const uint8_t* mask, int64_t N, int64_t K, int d, const double* A,
                     const double* B, double* dX, double* D_dX, double* dA, double* D_dA,
                     double* dB, double* D_dB, double* dWp, double* D_dWp, int threads) {
  backward_t(X, dY, M, z, mask, N, K, d, A, B, dX, D_dX, dA, D_dA, dB, D_dB, dWp, D_dWp, threads);
}

// H-aware sequential assignment (decoupleQ page, section 3.3, eq. (8)-(11):
// fix one element by rounding and clipping, then re-solve the rest of the
// quadratic objective without the integer constraint and the box -- the error
// feedback of LDLQ, which the LC-QAT technical summary, Methodology 2, names
// for the initial codes).  For every row of the code-space targets P [N][K],
// in increasing j:
//     t_j = p_j + sum_{i<j} U[i][j] (p_i - z_i),   z_j = clamp(rint(t_j), 0, 3),
// the sum over i in increasing order.  Only the strictly upper triangle of
// U [K][K] is read.  Z is u8 [N][K].
void lco_ldlq_assign(const double* P, int64_t N, int64_t K, const double* U, uint8_t* Z,
                     int threads) {
  parallel_rows(N, threads, [=](int64_t a, int64_t b) {
    std::vector<double> e(static_cast<size_t>(K), 0.0);
    for (int64_t n = a; n < b; ++n) {
      const double* p = P + n * K;
      uint8_t* z = Z + n * K;
      for (int64_t j = 0; j < K; ++j) {
        double c = 0.0;
        for (int64_t i = 0; i < j; ++i) c += U[i * K + j] * e[size_t(i)];
        z[j] = code_of(p[j] + c);
        e[size_t(j)] = p[j] - double(z[j]);
      }
    }
  });
}

// DGE (the LC-QAT technical summary's gradient estimator: a smooth,
// differentiable curve through the rounding).  The pages give no curve; the
// reading taken is the tanh staircase on [0, 3], clamped outside:
//     phi_k(w) = floor(w) + 1/2 + tanh(k (frac(w) - 1/2)) / (2 tanh(k / 2)),
// with w = 3 on the last step.  phi_k'(w) = (k / (2 tanh(k / 2))) / cosh^2(k (frac(w) - 1/2))
// on [0, 3] and 0 outside (and for NaN): the factor DGE puts where the STE
// puts the clamp mask.
void lco_dge_phi(const double* w, int64_t n, double k, double* out) {
  for (int64_t t = 0; t < n; ++t) {
    const double x = std::min(std::max(w[t], 0.0), kCodeMax);
    const double fl = std::min(std::floor(x), kCodeMax - 1.0);
    out[t] = fl + 0.5 + std::tanh(k * (x - fl - 0.5)) / (2.0 * std::tanh(k / 2.0));
  }
}
void lco_dge_derivative(const double* w, int64_t n, double k, double* out) {
  for (int64_t t = 0; t < n; ++t) {
    const double x = w[t];
    if (!(x >= 0.0 && x <= kCodeMax)) {
      out[t] = 0.0;
      continue;
    }
    const double fl = std::min(std::floor(x), kCodeMax - 1.0);
    const double c = std::cosh(k * (x - fl - 0.5));
    out[t] = (k / (2.0 * std::tanh(k / 2.0))) / (c * c);
  }
}

// Least-squares refit of (A, B) given the codes (decoupleQ page, eq. (5) with
// H replaced by its diagonal h, and section 3.3: with the integer part fixed
// the float part is a quadratic, solved in closed form).  The objective
// sum_n sum_k h_k (W0[n][k] - W~[n][k])^2 splits over the output coordinate i;
// with zt = [z_0 .. z_{d-1}, 1] per vector (row n, position g):
//     G_i = sum_{n,g} h_{g d + i} zt zt^T,   R_i = sum_{n,g} h_{g d + i} W0[n][g d + i] zt,
// and row i of [A | B] is G_i^+ R_i.  h may be null (h = 1).
void lco_fit_affine(const double* W0, const uint8_t* z, int64_t N, int64_t K, int d,
                    const double* h, double* A, double* B) {
  const int m = d + 1;
  for (int i = 0; i < d; ++i) {
    std::vector<double> G(static_cast<size_t>(m * m), 0.0), R(static_cast<size_t>(m), 0.0);
    std::vector<double> th(static_cast<size_t>(m), 0.0);
    std::vector<double> zt(static_cast<size_t>(m), 0.0);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t g = 0; g < K / d; ++g) {
        const int64_t k = g * d + i;
        const double hk = h ? h[k] : 1.0;
        for (int a = 0; a < d; ++a) zt[size_t(a)] = double(z[n * K + g * d + a]);
        zt[size_t(d)] = 1.0;
        for (int a = 0; a < m; ++a) {
          for (int b = 0; b < m; ++b) G[size_t(a) * m + b] += hk * zt[size_t(a)] * zt[size_t(b)];
          R[size_t(a)] += hk * W0[n * K + k] * zt[size_t(a)];
        }
      }
    pinv_solve(G, m, R.data(), th.data());
    for (int a = 0; a < d; ++a) A[i * d + a] = th[size_t(a)];
    B[i] = th[size_t(d)];
  }
}

// The same refit under the full K x K input Hessian H (decoupleQ page, eq. (5):
// the objective sum_n (W~[n] - W0[n])^T H (W~[n] - W0[n]); section 3.3's closed
// form).  theta = [A | B] enters every decoded element linearly,
// W~[n][g d + i] = sum_a theta[i][a] zt[n][g][a], so one joint system of
// d (d + 1) unknowns, index (i, a) -> i (d + 1) + a:
//     L[(i,a)][(j,b)] = sum_{g,h} H[g d + i][h d + j] S[(g,a)][(h,b)],
//     R[(i,a)]        = sum_g sum_k H[g d + i][k] T[k][(g,a)],
// with the code Gram S[(g,a)][(h,b)] = sum_n zt[n][g][a] zt[n][h][b] and
// T[k][(g,a)] = sum_n W0[n][k] zt[n][g][a] (the sums over n taken first);
// theta = L^+ R.
void lco_fit_affine_h(const double* W0, const uint8_t* z, int64_t N, int64_t K, int d,
                      const double* H, double* A, double* B) {
  const int m = d + 1, np = d * m;
  const int64_t ng = K / d, w = ng * m;  // width of S and T: (g, a) pairs
  std::vector<double> zt(static_cast<size_t>(w), 0.0);
  std::vector<double> S(size_t(w) * size_t(w), 0.0), T(size_t(K) * size_t(w), 0.0);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < ng; ++g) {
      for (int a = 0; a < d; ++a) zt[size_t(g * m + a)] = double(z[n * K + g * d + a]);
      zt[size_t(g * m + d)] = 1.0;
    }
    for (int64_t u = 0; u < w; ++u)
      for (int64_t v = 0; v < w; ++v) S[size_t(u * w + v)] += zt[size_t(u)] * zt[size_t(v)];
    for (int64_t k = 0; k < K; ++k)
      for (int64_t u = 0; u < w; ++u) T[size_t(k * w + u)] += W0[n * K + k] * zt[size_t(u)];
  }
  std::vector<double> L(static_cast<size_t>(np * np), 0.0), R(static_cast<size_t>(np), 0.0);
  std::vector<double> th(static_cast<size_t>(np), 0.0);
  for (int i = 0; i < d; ++i)
    for (int a = 0; a < m; ++a)
      for (int j = 0; j < d; ++j)
        for (int b = 0; b < m; ++b) {
          double acc = 0.0;
          for (int64_t g = 0; g < ng; ++g)
            for (int64_t hh = 0; hh < ng; ++hh)
              acc += H[(g * d + i) * K + hh * d + j] * S[size_t((g * m + a) * w + hh * m + b)];
          L[size_t(i * m + a) * np + j * m + b] = acc;
        }
  for (int i = 0; i < d; ++i)
    for (int a = 0; a < m; ++a) {
      double acc = 0.0;
      for (int64_t g = 0; g < ng; ++g)
        for (int64_t k = 0; k < K; ++k) acc += H[(g * d + i) * K + k] * T[size_t(k * w + g * m + a)];
      R[size_t(i * m + a)] = acc;
    }
  pinv_solve(L, np, R.data(), th.data());
  for (int i = 0; i < d; ++i) {
    for (int a = 0; a < d; ++a) A[i * d + a] = th[size_t(i * m + a)];
    B[i] = th[size_t(i * m + d)];
  }
}

}  // extern "C"

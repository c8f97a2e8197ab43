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
//     fith_reduce_kernel sums the partials in CTA order; fith_solve_kernel
//     solves the
//     d (d+1) x d (d+1) system: Cholesky when every pivot is above 1e-8 of
//     the largest diagonal entry, otherwise a parallel cyclic Jacobi
//     eigendecomposition with eigenvalues below 1e-12 of the largest taken as
//     zero (the minimum-norm solution), as the diagonal refit does.
// Every sum runs in a fixed order: the result is bitwise reproducible.
#include <math.h>
#include <stddef.h>

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
// shared memory, converted to fp64 once per element.  For every h-block of a
// chunk with h >= g, L gains the Kronecker product of the H block
// H[g d + i][h d + j] and the code Gram block S~[(g,a),(h,b)] (half of it for
// h = g): H and S~ are symmetric, so the (h, g) block adds the transpose of
// the (g, h) block and the solve forms L as L_half + L_half^T.  A thread owns a
// register tile of
// kJT values of j (for one i) times the d + 1 values of b (for one a), so it
// loads kJT + d + 1 values per kJT (d + 1) fused multiply-adds.  The kTeams
// teams of a CTA take alternate h-blocks; R[(i,a)] is split over the CTA's
// threads by k mod parts.  At the end the teams (and the parts of R) are
// added in a fixed order into the CTA's partial [L (NP x NP) | R (NP)] (fp64).
constexpr int kChunkCols = 192;  // columns of H and C per shared-memory chunk
constexpr int kRowPad = 1;       // doubles of padding per shared row: rows 2 banks apart
constexpr int kTeams = 2;

// the system: d (d + 1) unknowns; a CTA's partial is [L (NP x NP) | R (NP)]
template <int D>
struct FitHDims {
  static constexpr int NP = D * (D + 1);
  static constexpr int kPart = NP * NP + NP;  // doubles per CTA partial
};
// the CUDA-core contraction's thread layout (d != 8)
template <int D>
struct FitHContract {
  static constexpr int NP = FitHDims<D>::NP;
  static constexpr int P1 = D + 1;
  static constexpr int kJT = D < 4 ? D : 4;           // j values per thread tile
  static constexpr int kTeam = D * (D / kJT) * P1;    // threads per team
  static constexpr int kThreads = ((kTeams * kTeam + 31) / 32) * 32;
  static constexpr int kRParts = kThreads / NP;       // threads per R value
  static constexpr int kCols = kChunkCols;            // a multiple of every d
  static constexpr int kPart = FitHDims<D>::kPart;
};

template <int D>
__global__ void __launch_bounds__(FitHContract<D>::kThreads) fith_contract_kernel(
    const float* __restrict__ H, const float* __restrict__ C, int64_t K, double* __restrict__ partials) {
  using F = FitHContract<D>;
  constexpr int NP = F::NP, P1 = F::P1, COLS = F::kCols, JT = F::kJT;
  __shared__ double sH[D][COLS + kRowPad];
  __shared__ double sS[P1][COLS + kRowPad];
  __shared__ double sT[P1][COLS + kRowPad];  // T~ = hi + lo, in fp64
  __shared__ double sOnes[P1];
  __shared__ double sRed[kTeams > F::kRParts ? kTeams : F::kRParts][NP + 1];
  const int tid = threadIdx.x;
  // L tile: team tm, i, j block jb (j = jb JT .. jb JT + JT - 1), a
  const int tm = tid / F::kTeam, mt = tid % F::kTeam;
  const bool lact = tm < kTeams;
  const int a = mt % P1, ij = mt / P1;
  const int i = ij / (D / JT), j0 = (ij % (D / JT)) * JT;
  // R: value ro = (i, a), part rp takes the chunk columns rp, rp + kRParts, ...
  const int ro = tid % NP, rp = tid / NP;
  const bool ract = rp < F::kRParts;
  const int ri = ro / P1, ra = ro % P1;
  const int64_t ldc = kOnes + 3 * K;
  const int64_t ng = K / D;
  double acc[JT][P1];
#pragma unroll
  for (int x = 0; x < JT; ++x)
#pragma unroll
    for (int b = 0; b < P1; ++b) acc[x][b] = 0.0;
  double accR = 0.0;

  for (int64_t g = blockIdx.x; g < ng; g += gridDim.x) {
    // C row of (g, a): the ones row 0 for a = d
    auto crow = [&](int aa) -> const float* {
      return C + (aa < D ? (kOnes + g * D + aa) : 0) * ldc;
    };
    __syncthreads();
    if (tid < P1) sOnes[tid] = static_cast<double>(crow(tid)[0]);
    for (int64_t c0 = 0; c0 < K; c0 += COLS) {
      const int ncols = static_cast<int>(K - c0 < COLS ? K - c0 : COLS);  // multiple of 64
      __syncthreads();  // the previous chunk is consumed
      // 16-byte loads (K, the row pitches and the chunk starts are multiples of 4)
      constexpr int V = COLS / 4;
      const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int e = tid; e < (D + 2 * P1) * V; e += blockDim.x) {
        const int r = e / V, c = (e % V) * 4;
        double* dst;
        float4 v = zero4;
        if (r < D) {
          if (c < ncols) v = __ldg(reinterpret_cast<const float4*>(H + (g * D + r) * K + c0 + c));
          dst = &sH[r][c];
        } else if (r < D + P1) {
          if (c < ncols) v = __ldcg(reinterpret_cast<const float4*>(crow(r - D) + kOnes + c0 + c));
          dst = &sS[r - D][c];
        } else {
          if (c < ncols) {
            const float* cr = crow(r - D - P1) + kOnes + K + c0 + c;
            const float4 hi = __ldcg(reinterpret_cast<const float4*>(cr));
            const float4 lo = __ldcg(reinterpret_cast<const float4*>(cr + K));
            dst = &sT[r - D - P1][c];
            dst[0] = double(hi.x) + double(lo.x);
            dst[1] = double(hi.y) + double(lo.y);
            dst[2] = double(hi.z) + double(lo.z);
            dst[3] = double(hi.w) + double(lo.w);
            continue;
          }
          dst = &sT[r - D - P1][c];
        }
        dst[0] = v.x;
        dst[1] = v.y;
        dst[2] = v.z;
        dst[3] = v.w;
      }
      __syncthreads();
      if (lact) {
        // L: h-blocks tm, tm + kTeams, ... of the chunk with h >= g (the (h, g)
        // block adds the transpose of the (g, h) block; the diagonal block
        // counts half, so L = L_half + L_half^T)
        const int hfirst = static_cast<int>(g - c0 / D);  // chunk's h-block index of h = g
        for (int hb = tm; hb < ncols / D; hb += kTeams) {
          if (hb < hfirst) continue;
          const double wgt = hb == hfirst ? 0.5 : 1.0;
          double hv[JT], sv[P1];
#pragma unroll
          for (int x = 0; x < JT; ++x) hv[x] = wgt * sH[i][hb * D + j0 + x];
#pragma unroll
          for (int b = 0; b < D; ++b) sv[b] = sS[a][hb * D + b];
          sv[D] = sOnes[a];
#pragma unroll
          for (int x = 0; x < JT; ++x)
#pragma unroll
            for (int b = 0; b < P1; ++b) acc[x][b] = fma(hv[x], sv[b], acc[x][b]);
        }
      }
      if (ract)
        for (int c = rp; c < ncols; c += F::kRParts) accR = fma(sH[ri][c], sT[ra][c], accR);
    }
  }
  // teams in team order into the CTA partial, one L column (j, b) at a time
  double* out = partials + int64_t(blockIdx.x) * F::kPart;
#pragma unroll
  for (int x = 0; x < JT; ++x)
#pragma unroll
    for (int b = 0; b < P1; ++b) {
      // this thread's value is L[(i,a)][(j0 + x, b)]; threads with the same
      // (i, a) but another j block hold other columns, so one pass per j block
      for (int jb = 0; jb < D / JT; ++jb) {
        __syncthreads();
        if (lact && (ij % (D / JT)) == jb) sRed[tm][i * P1 + a] = acc[x][b];
        __syncthreads();
        if (tid < NP) {
          double v = 0.0;
          for (int t2 = 0; t2 < kTeams; ++t2) v += sRed[t2][tid];
          out[tid * NP + (jb * JT + x) * P1 + b] = v;  // L[(i,a) = tid][(j,b)]
        }
      }
    }
  __syncthreads();
  if (ract) sRed[rp][ro] = accR;
  __syncthreads();
  if (tid < NP) {
    double v = 0.0;
    for (int t2 = 0; t2 < F::kRParts; ++t2) v += sRed[t2][tid];
    out[NP * NP + tid] = v;
  }
}

// ---------------------------------------------------------------- 3a'. d = 8: tiles and fp64 MMA
// The same partial [L_half | R] as fith_contract_kernel, for d = 8.  The L sum
// is a product once reindexed: with U_p = H's block (g, h) (8 x 8, rows i,
// columns j) and V_p = S~'s block ((g, a), (h, b)) (9 x 9), over the position
// pairs p = (g, h >= g),
//     L_half[(i,a),(j,b)] = sum_p w_p U_p[i][j] V_p[a][b],   w = 1/2 if g = h, else 1,
// a 64 x 81 x #pairs product, run on the fp64 tensor-core MMA (m8n8k4).  CTA
// c takes the 64 x 64 tiles (gb, hb >= gb) of positions 8 gb .. 8 gb + 7 by
// 8 hb .. 8 hb + 7 in turn: it stages the tile of H, of the code Gram and of
// T~ (both T~ tiles (gb rows, hb columns) and (hb rows, gb columns)) in fp64
// shared memory; warp i accumulates the rows (i, j) of L over the tile's 64
// pairs (the pairs are the MMA's k), 11 column tiles of 8 over the 81 (a, b).
// R comes from the same tile, also on the fp64 MMA: warp pl takes position
// pl of the tile's row block gb against the columns of hb and, by H's
// symmetry, position pl of hb against the columns of gb (R's rows i are the
// MMA's 8 rows, its 9 values of a two column tiles, the columns of H its k),
// so every (row block, column block) of H and T~ is read once; the warps'
// parts of R are added in warp order at the end.
constexpr int kC8Tile = 64;               // tile side in elements (8 positions)
// doubles per shared row, 4 mod 16: fragments that take 8 rows and 4
// columns (or 8 columns and 4 rows) fill the 16 double slots of the banks twice
constexpr int kC8Pitch = kC8Tile + 4;
constexpr int kC8Threads = 256;           // 8 warps: warp i owns the L rows (i, j)
struct C8Smem {
  double U[kC8Tile][kC8Pitch];   // H[64 gb + r][64 hb + c]
  double S[kC8Tile][kC8Pitch];   // C[64 + 64 gb + r][64 + 64 hb + c]: code Gram S~ (a, b < 8)
  double T1[kC8Tile][kC8Pitch];  // T~ rows 64 gb + r, columns 64 hb + c (hi + lo)
  double T2[kC8Tile][kC8Pitch];  // T~ rows 64 hb + r, columns 64 gb + c
  double Ro[kC8Tile];            // C[0][64 + 64 hb + c]: S~'s ones row over hb
  double Co[kC8Tile];            // C[64 + 64 gb + r][0]: S~'s ones column over gb
  double To1[kC8Tile];           // T~ of the ones row over hb columns
  double To2[kC8Tile];           // ... over gb columns
  double N;                      // C[0][0]: the number of rows
  double zero;                   // 0: the padding columns of L's and R's MMAs
  double Rred[8][72];            // the warps' parts of R
};

__device__ __forceinline__ void dmma_m8n8k4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(kC8Threads, 1) fith_contract8_kernel(
    const float* __restrict__ H, const float* __restrict__ C, int64_t K, double* __restrict__ partials) {
  constexpr int D = 8, P1 = 9, NP = 72, kNT = 11;  // 11 column tiles of 8 over the 81 (a, b)
  extern __shared__ __align__(16) unsigned char c8smem[];
  C8Smem& sm = *reinterpret_cast<C8Smem*>(c8smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t ldc = kOnes + 3 * K;
  const int nb = static_cast<int>(K / kC8Tile);
  const int ntiles = nb * (nb + 1) / 2;
  // L: this lane's MMA coordinates.  A: row j = lane / 4, pair lane % 4 of a
  // k step; B and D: columns n = 8 nt + lane / 4 and (D) 8 nt + 2 (lane % 4) + e
  const int i = warp, jrow = lane >> 2, kq = lane & 3;
  // where column n = 8 nt + lane / 4 of V_p sits, as a double offset in the
  // shared struct plus strides per gl and hl (branch-free loads):
  //   a, b < 8: S[8 gl + a][8 hl + b];  b = 8: Co[8 gl + a];  a = 8: Ro[8 hl + b];
  //   a = b = 8: N;  n >= 81: zero
  const double* smd = reinterpret_cast<const double*>(c8smem);
  constexpr int oS = offsetof(C8Smem, S) / 8, oCo = offsetof(C8Smem, Co) / 8;
  constexpr int oRo = offsetof(C8Smem, Ro) / 8, oN = offsetof(C8Smem, N) / 8;
  constexpr int oZ = offsetof(C8Smem, zero) / 8;
  int bo[kNT], bsg[kNT], bsh[kNT];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    const int n = nt * 8 + jrow, a = n / P1, b = n % P1;
    if (n >= P1 * P1) bo[nt] = oZ, bsg[nt] = 0, bsh[nt] = 0;
    else if (a < D && b < D) bo[nt] = oS + a * kC8Pitch + b, bsg[nt] = D * kC8Pitch, bsh[nt] = D;
    else if (a < D) bo[nt] = oCo + a, bsg[nt] = D, bsh[nt] = 0;
    else if (b < D) bo[nt] = oRo + b, bsg[nt] = 0, bsh[nt] = D;
    else bo[nt] = oN, bsg[nt] = 0, bsh[nt] = 0;
  }
  double acc[kNT][2];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) acc[nt][0] = acc[nt][1] = 0.0;
  // R: warp pl's MMA: A = H rows (8 pl + i) over 4 columns, B = T~ rows
  // (8 pl + a) over the same columns (a = 8: the ones row; a > 8: zero)
  double accR[2][2] = {{0.0, 0.0}, {0.0, 0.0}};

  for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
    int gb = 0, rem = t;  // tile t of the upper triangle, row by row
    while (rem >= nb - gb) {
      rem -= nb - gb;
      ++gb;
    }
    const int hb = gb + rem;
    const bool diag = gb == hb;
    __syncthreads();  // the previous tile is consumed
    const int64_t g0 = int64_t(gb) * kC8Tile, h0 = int64_t(hb) * kC8Tile;
    // one element per thread and array: a warp reads 128 contiguous bytes of a
    // row and writes 32 consecutive doubles (no bank conflicts)
#pragma unroll 4
    for (int e = tid; e < kC8Tile * kC8Tile; e += kC8Threads) {
      const int r = e / kC8Tile, c = e % kC8Tile;
      const float* crow = C + (kOnes + g0 + r) * ldc;
      const float u = __ldg(H + (g0 + r) * K + h0 + c);
      const float sv = __ldcg(crow + kOnes + h0 + c);
      const float t1h = __ldcg(crow + kOnes + K + h0 + c);
      const float t1l = __ldcg(crow + kOnes + 2 * K + h0 + c);
      sm.U[r][c] = u;
      sm.S[r][c] = sv;
      sm.T1[r][c] = double(t1h) + double(t1l);
      if (!diag) {
        const float* crow2 = C + (kOnes + h0 + r) * ldc;
        sm.T2[r][c] = double(__ldcg(crow2 + kOnes + K + g0 + c)) +
                      double(__ldcg(crow2 + kOnes + 2 * K + g0 + c));
      }
    }
    if (tid < kC8Tile) {
      sm.Ro[tid] = C[kOnes + h0 + tid];
      sm.Co[tid] = C[(kOnes + g0 + tid) * ldc];
      sm.To1[tid] = double(C[kOnes + K + h0 + tid]) + double(C[kOnes + 2 * K + h0 + tid]);
      sm.To2[tid] = double(C[kOnes + K + g0 + tid]) + double(C[kOnes + 2 * K + g0 + tid]);
    }
    if (tid == 0) {
      sm.N = C[0];
      sm.zero = 0.0;
    }
    __syncthreads();

    // L: the tile's 64 pairs p = 8 gl + hl, four per k step
#pragma unroll 2
    for (int ks = 0; ks < 16; ++ks) {
      const int p = ks * 4 + kq, gl = p >> 3, hl = p & 7;
      const double w = diag ? (hl > gl ? 1.0 : (hl == gl ? 0.5 : 0.0)) : 1.0;
      const double av = w * sm.U[gl * D + i][hl * D + jrow];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
        dmma_m8n8k4(acc[nt], av, smd[bo[nt] + gl * bsg[nt] + hl * bsh[nt]]);
    }
    // R, position pl = warp: rows of gb against the columns of hb; off the
    // diagonal also the rows of hb against the columns of gb
    // (H[64 hb + 8 pl + i][64 gb + c] = U[c][8 pl + i])
    {
      const int pl = warp, ar = jrow;  // B column: a = ar (tile 0), 8 + ar (tile 1)
#pragma unroll 4
      for (int c0 = 0; c0 < kC8Tile; c0 += 4) {
        const int c = c0 + kq;
        const double av = sm.U[pl * D + jrow][c];
        dmma_m8n8k4(accR[0], av, sm.T1[pl * D + ar][c]);
        dmma_m8n8k4(accR[1], av, ar == 0 ? sm.To1[c] : 0.0);
      }
      if (!diag) {
#pragma unroll 4
        for (int c0 = 0; c0 < kC8Tile; c0 += 4) {
          const int c = c0 + kq;
          const double av = sm.U[c][pl * D + jrow];
          dmma_m8n8k4(accR[0], av, sm.T2[pl * D + ar][c]);
          dmma_m8n8k4(accR[1], av, ar == 0 ? sm.To2[c] : 0.0);
        }
      }
    }
  }
  // the CTA's partial: every L value belongs to one lane of one warp
  double* out = partials + int64_t(blockIdx.x) * (NP * NP + NP);
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = nt * 8 + 2 * kq + e;
      if (n < P1 * P1) out[(i * P1 + n / P1) * NP + jrow * P1 + n % P1] = acc[nt][e];
    }
  // R: lane holds rows i = lane / 4 and columns a = 2 (lane % 4) + e (tile 0)
  // and 8 + 2 (lane % 4) + e (tile 1: only a = 8 exists)
  __syncthreads();
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    sm.Rred[warp][jrow * P1 + 2 * kq + e] = accR[0][e];
    if (kq == 0 && e == 0) sm.Rred[warp][jrow * P1 + D] = accR[1][0];
  }
  __syncthreads();
  if (tid < NP) {
    double v = 0.0;
    for (int w = 0; w < 8; ++w) v += sm.Rred[w][tid];
    out[NP * NP + tid] = v;
  }
}

// ---------------------------------------------------------------- 3b. reduce, solve
// The partials are summed in CTA order, one thread per value, 8 loads of a
// thread in flight at a time (a fixed order: bitwise reproducible).
template <int D>
__global__ void __launch_bounds__(256) fith_reduce_kernel(const double* __restrict__ partials,
                                                          int num_parts, double* __restrict__ red) {
  using F = FitHDims<D>;
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= F::kPart) return;
  double acc = 0.0;
  int c = 0;
  for (; c + 8 <= num_parts; c += 8) {
    double x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldcg(partials + int64_t(c + u) * F::kPart + v);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += x[u];
  }
  for (; c < num_parts; ++c) acc += __ldcg(partials + int64_t(c) * F::kPart + v);
  red[v] = acc;
}

// One CTA: L theta = R in shared memory, from the reduced [L | R].
constexpr int kSolveThreads = 256;

// Cholesky G = L L^T in place (lower triangle) by the whole CTA, one column
// at a time; then the two triangular solves by warp 0, column by column (lanes
// take rows).  Returns false, for every thread, on a pivot below kHCholFloor
// of the largest diagonal entry (G is then partly overwritten).  th (shared)
// receives theta.
template <int NP>
__device__ bool chol_solve_cta(double (*G)[NP], const double* R, double* th) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  constexpr int kW = kSolveThreads / 32;
  __shared__ double dmax;
  __shared__ double rdiag[NP];  // 1 / L[c][c]
  if (t == 0) {
    double m = 0.0;
    for (int c = 0; c < NP; ++c) m = fmax(m, G[c][c]);
    dmax = m;
  }
  __syncthreads();
  const double dm = dmax;
  if (!(dm > 0.0)) return false;
  for (int c = 0; c < NP; ++c) {
    // every thread forms the pivot itself: one decision, no barrier for it
    const double piv = G[c][c];
    if (!(piv > kHCholFloor * dm)) return false;  // the same for every thread
    const double lcc = sqrt(piv), rl = 1.0 / lcc;
    if (t == 0) {
      rdiag[c] = rl;
    }
    __syncthreads();  // every thread has read G[c][c]
    if (t == 0) G[c][c] = lcc;
    for (int r = c + 1 + t; r < NP; r += blockDim.x) G[r][c] *= rl;
    __syncthreads();
    // trailing update of the lower triangle: G[r][s] -= L[r][c] L[s][c], c < s <= r;
    // warp w takes the rows c + 1 + w, c + 1 + w + 8, ...; lanes the columns
    for (int r = c + 1 + warp; r < NP; r += kW) {
      const double lrc = G[r][c];
      for (int s2 = c + 1 + lane; s2 <= r; s2 += 32) G[r][s2] -= lrc * G[s2][c];
    }
    __syncthreads();
  }
  if (t < 32) {
    for (int r = lane; r < NP; r += 32) th[r] = R[r];
    __syncwarp();
    for (int c = 0; c < NP; ++c) {  // L y = R, y in th
      if (lane == 0) th[c] *= rdiag[c];
      __syncwarp();
      const double yc = th[c];
      for (int r = c + 1 + lane; r < NP; r += 32) th[r] -= G[r][c] * yc;
      __syncwarp();
    }
    for (int c = NP - 1; c >= 0; --c) {  // L^T theta = y, in place
      if (lane == 0) th[c] *= rdiag[c];
      __syncwarp();
      const double tc = th[c];
      for (int r = lane; r < c; r += 32) th[r] -= G[c][r] * tc;
      __syncwarp();
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
__global__ void __launch_bounds__(kSolveThreads) fith_solve_kernel(const double* __restrict__ red,
                                                                   float* __restrict__ A,
                                                                   float* __restrict__ B) {
  using F = FitHDims<D>;
  constexpr int NP = F::NP;
  extern __shared__ __align__(16) unsigned char fsm[];
  double (*G)[NP] = reinterpret_cast<double (*)[NP]>(fsm);
  double (*G0)[NP] = G + NP;           // a copy for the Jacobi fallback
  double (*V)[NP] = G0 + NP;
  double* R = reinterpret_cast<double*>(V + NP);
  double* th = R + NP;
  const int t = threadIdx.x;
  for (int v = t; v < F::kPart; v += blockDim.x) {
    const double acc = red[v];
    if (v < NP * NP) {
      G[v / NP][v % NP] = acc;  // L_half
    } else {
      R[v - NP * NP] = acc;
    }
  }
  __syncthreads();
  // L = L_half + L_half^T (the contraction accumulated the pairs h >= g only)
  for (int e = t; e < NP * NP; e += blockDim.x) {
    const int r = e / NP, c = e % NP;
    if (r < c) {
      const double s = G[r][c] + G[c][r];
      G0[r][c] = s;
      G0[c][r] = s;
    } else if (r == c) {
      G0[r][r] = 2.0 * G[r][r];
    }
  }
  __syncthreads();
  for (int e = t; e < NP * NP; e += blockDim.x) G[e / NP][e % NP] = G0[e / NP][e % NP];
  __syncthreads();
  if (!chol_solve_cta<NP>(G, R, th)) jacobi_pinv_par<NP>(G0, V, R, th);
  if (t < D * D) A[t] = static_cast<float>(th[(t / D) * (D + 1) + (t % D)]);
  if (t < D) B[t] = static_cast<float>(th[t * (D + 1) + D]);
}

template <int D>
size_t solve_smem() {
  constexpr int NP = FitHDims<D>::NP;
  return size_t(3) * NP * NP * 8 + size_t(2) * NP * 8 + 16;
}

// CTAs of the contraction: d = 8 takes the (K/64)(K/64 + 1)/2 tiles on one CTA
// per SM, other d the K/d vector positions on two
int contract_grid(int64_t d_in, int d) {
  int64_t g, work;
  if (d == 8) {
    const int64_t nb = d_in / kC8Tile;
    g = kNumSMsB200;
    work = nb * (nb + 1) / 2;
  } else {
    g = 2 * kNumSMsB200;
    work = d_in / (d > 0 ? d : 1);
  }
  if (work < g) g = work;
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
  const int grid = contract_grid(d_in, D);
  double* red = partials + size_t(grid) * F::kPart;  // the reduced [L | R]
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
  if constexpr (D == 8) {
    if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(fith_contract8_kernel),
                                             sizeof(C8Smem));
        e != cudaSuccess)
      return e;
    fith_contract8_kernel<<<grid, kC8Threads, sizeof(C8Smem), s>>>(H, C, d_in, partials);
  } else {
    fith_contract_kernel<D><<<grid, FitHContract<D>::kThreads, 0, s>>>(H, C, d_in, partials);
  }
  ++*launches;
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  fith_reduce_kernel<D><<<static_cast<unsigned>(ceil_div(F::kPart, 256)), 256, 0, s>>>(partials, grid,
                                                                                     red);
  ++*launches;
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  auto sk = fith_solve_kernel<D>;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(sk), solve_smem<D>());
      e != cudaSuccess)
    return e;
  sk<<<1, kSolveThreads, solve_smem<D>(), s>>>(red, A, B);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

size_t fith_scratch_bytes(int64_t d_out, int64_t d_in, int d) {
  const int64_t ldq = kOnes + 3 * d_in;
  const size_t q_bytes = (size_t(d_out) * ldq * 2 + 255) / 256 * 256;
  const size_t c_bytes = (size_t(kOnes + d_in) * ldq * 4 + 255) / 256 * 256;
  const int np = d * (d + 1);
  const size_t p_bytes = (size_t(contract_grid(d_in, d)) + 1) * size_t(np * np + np) * 8;
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

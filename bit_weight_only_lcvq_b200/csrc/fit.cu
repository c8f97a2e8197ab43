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
//  * fit_accum_kernel: one pass over W0 and the codes, forming per vector
//    position the integer Gram of its codes and the products of its targets
//    with its codes; h is applied afterwards, per CTA, in fp64 (below).  Each
//    CTA writes one fp64 partial of every G_i and R_i.
//  * fit_solve_kernel: CTA i sums coordinate i's partials in a fixed order
//    (fp64), then forms theta_i = G_i^+ R_i in fp64: by Cholesky when every pivot is above
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

constexpr double kPinvRcond = 1e-12;

template <int D>
struct FitDims {
  static constexpr int P = D + 1;                 // zt length
  static constexpr int SG = P * (P + 1) / 2;      // upper triangle of G_i
  static constexpr int S = SG + P;                // G_i then R_i
};

// The pass over W0 and the codes.  With h applied per channel, the normal
// equations are sums over the vector positions g of a row (channel k = g d + i):
//     G_i = sum_g h_{gd+i} S_g,   S_g = sum_n zt zt^T   (zt of vector (n, g)),
//     R_i = sum_g h_{gd+i} T_{g,i},   T_{g,i} = sum_n W0[n][gd+i] zt,
// so the pass only forms S_g (an integer Gram: exact in fp32 over the rows
// of one thread) and T_g; h enters afterwards, in fp64.
//
// fit_accum_kernel: lane l of a CTA owns vector position g = 32 c + l of column
// tile c and its 4 warps split the CTA's rows.  Per row a lane loads the d
// floats of its vector (a warp reads 32 d consecutive floats) and its code,
// forms zt = [z_0 .. z_{d-1}, 1] once, and adds d (d+1) products to T and the
// (d+1)(d+2)/2 upper-triangle products to S: about 2.3 (d+1) instructions per
// weight instead of a Gram per weight.  T is fp32 flushed into fp64 (shared
// memory) every kFitFlush rows, so each fp32 partial sums at most kFitFlush
// terms.  The CTA then sums its warps in warp order, applies h per coordinate
// in fp64 over its 32 positions in order, and writes one partial [d][G_i, R_i].
constexpr int kFitFlush = 16;
constexpr int kFitLanes = 32;            // vector positions per CTA
constexpr int kFitRowWarps = 4;          // warps per CTA, each a share of the rows
constexpr int kFitThreads2 = kFitLanes * kFitRowWarps;
constexpr int kFitAhead2 = 4;            // rows whose loads are in flight together
constexpr int kFitTargetCtas = 2 * kNumSMsB200;

template <int D>
struct FitSmem {
  using F = FitDims<D>;
  static constexpr int kT = D * F::P;                        // T entries per position
  static constexpr int kStage = (kT > F::SG ? kT : F::SG);   // fp64 per thread
  static constexpr size_t kStageBytes = size_t(kStage) * kFitThreads2 * 8;
  static constexpr size_t kPosBytes = size_t(kFitLanes) * (F::SG + kT) * 8;
  static constexpr size_t kBytes = kStageBytes + kPosBytes;
};

template <int D>
__global__ void __launch_bounds__(kFitThreads2, 2) fit_accum_kernel(
    const float* __restrict__ W0, const uint32_t* __restrict__ codes, int64_t N, int64_t groups,
    int64_t row_splits, const float* __restrict__ h, double* __restrict__ partials) {
  using F = FitDims<D>;
  using L = FitSmem<D>;
  constexpr int P = F::P, kT = L::kT;
  extern __shared__ __align__(16) unsigned char fit_smem[];
  double* stage = reinterpret_cast<double*>(fit_smem);                 // [kStage][threads]
  double* pos = reinterpret_cast<double*>(fit_smem + L::kStageBytes);   // [32][SG + kT]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t ct = int64_t(blockIdx.x) / row_splits, rs = int64_t(blockIdx.x) % row_splits;
  const int64_t g = ct * kFitLanes + lane;
  const bool live = g < groups;
  const int64_t rows_per = ceil_div(N, row_splits);
  const int64_t r_begin = rs * rows_per, r_end = r_begin + rows_per < N ? r_begin + rows_per : N;
  const int64_t K = groups * D;
  const int64_t words_per_row = K / 16;  // d_in % 16 == 0
  const int64_t gbit = g * (2 * D);      // the vector's bits within its row
  const uint32_t cshift = static_cast<uint32_t>(gbit & 31);

  for (int q = 0; q < L::kStage; ++q) stage[q * kFitThreads2 + tid] = 0.0;
  float t32[kT], s32[F::SG];
#pragma unroll
  for (int q = 0; q < kT; ++q) t32[q] = 0.f;
#pragma unroll
  for (int q = 0; q < F::SG; ++q) s32[q] = 0.f;

  auto flush = [&]() {
#pragma unroll
    for (int q = 0; q < kT; ++q) {
      stage[q * kFitThreads2 + tid] += double(t32[q]);
      t32[q] = 0.f;
    }
  };
  int pending = 0;
  for (int64_t n0 = r_begin + warp; n0 < r_end; n0 += int64_t(kFitRowWarps) * kFitAhead2) {
    float wv[kFitAhead2][D];
    uint32_t cw[kFitAhead2];
#pragma unroll
    for (int u = 0; u < kFitAhead2; ++u) {
      const int64_t n = n0 + int64_t(u) * kFitRowWarps;
      const bool ok = live && n < r_end;
      const float* src = W0 + n * K + g * D;
      if constexpr (D % 4 == 0) {
#pragma unroll
        for (int q = 0; q < D / 4; ++q) {
          const float4 v = ok ? __ldcs(reinterpret_cast<const float4*>(src) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
          wv[u][4 * q] = v.x, wv[u][4 * q + 1] = v.y, wv[u][4 * q + 2] = v.z, wv[u][4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < D; ++q) wv[u][q] = ok ? __ldcs(src + q) : 0.f;
      }
      cw[u] = ok ? __ldg(codes + n * words_per_row + (gbit >> 5)) >> cshift : 0u;
    }
#pragma unroll
    for (int u = 0; u < kFitAhead2; ++u) {
      const int64_t n = n0 + int64_t(u) * kFitRowWarps;
      if (!(live && n < r_end)) continue;
      // small integers to float without the conversion unit: OR the value
      // into the mantissa of 2^23 and subtract 2^23
      float zt[P];
#pragma unroll
      for (int j = 0; j < D; ++j)
        zt[j] = __int_as_float(0x4B000000 | static_cast<int>((cw[u] >> (2 * j)) & 3u)) - 8388608.0f;
      zt[D] = 1.f;
#pragma unroll
      for (int i = 0; i < D; ++i) {
#pragma unroll
        for (int j = 0; j < D; ++j) t32[i * P + j] = fmaf(wv[u][i], zt[j], t32[i * P + j]);
        t32[i * P + D] += wv[u][i];
      }
      int q = 0;
#pragma unroll
      for (int a = 0; a < P; ++a)
#pragma unroll
        for (int b = a; b < P; ++b) {
          s32[q] = fmaf(zt[a], zt[b], s32[q]);
          ++q;
        }
      if (++pending == kFitFlush) {
        pending = 0;
        flush();
      }
    }
  }
  flush();
  __syncthreads();
  // per position: T summed over the warps in warp order ...
  for (int e = tid; e < kFitLanes * kT; e += kFitThreads2) {
    const int l = e / kT, q = e % kT;
    double t = 0.0;
    for (int w = 0; w < kFitRowWarps; ++w) t += stage[q * kFitThreads2 + w * 32 + l];
    pos[l * (F::SG + kT) + F::SG + q] = t;
  }
  __syncthreads();
  // ... then S (exact integers) through the same staging area
#pragma unroll
  for (int q = 0; q < F::SG; ++q) stage[q * kFitThreads2 + tid] = double(s32[q]);
  __syncthreads();
  for (int e = tid; e < kFitLanes * F::SG; e += kFitThreads2) {
    const int l = e / F::SG, q = e % F::SG;
    double t = 0.0;
    for (int w = 0; w < kFitRowWarps; ++w) t += stage[q * kFitThreads2 + w * 32 + l];
    pos[l * (F::SG + kT) + q] = t;
  }
  __syncthreads();
  // h per coordinate, positions in order: one partial [d][G_i (SG), R_i (P)]
  for (int e = tid; e < D * F::S; e += kFitThreads2) {
    const int i = e / F::S, q = e % F::S;
    double t = 0.0;
    for (int l = 0; l < kFitLanes; ++l) {
      const int64_t gg = ct * kFitLanes + l;
      if (gg >= groups) break;
      const double hw = h ? double(__ldg(h + gg * D + i)) : 1.0;
      const double v = q < F::SG ? pos[l * (F::SG + kT) + q] : pos[l * (F::SG + kT) + F::SG + i * P + (q - F::SG)];
      t += hw * v;
    }
    partials[int64_t(blockIdx.x) * D * F::S + e] = t;
  }
}

// d = 8 on the tensor cores (mma.sync m16n8k8, tf32 in, fp32 out).  Warp w of
// a CTA owns the 4 vector positions 32 c + 4 w .. + 3 of column tile c over
// the CTA's rows, 8 rows per step.  Per position and step:
//   T: A = the targets [16 x 8 rows]: rows 0..7 the tf32 "hi" parts of the 8
//      channels, rows 8..15 the "lo" parts (w - hi rounded to tf32, so hi + lo
//      is w to 2^-22); B = the codes [8 rows x 8] (exact); D rows i and i + 8
//      add up to T[i][j] = sum w_i z_j.
//   S: A = the codes [8 x 8 rows] with a ninth row of ones, B = the codes:
//      D = the integer Gram (exact), row 8 the code sums.
// The products are exact.  S is a sum of small integers and stays in the
// MMA's fp32 accumulator (exact below 2^24).  T's MMA sums 8 products from
// zero; its hi and lo rows are added and kept in fp32 for kFitFlush terms,
// then added into fp64: a T entry's rounding is at most about 20 2^-24 of its
// terms' absolute sum (the split's 2^-22, the MMA's partial sums, the two fp32
// additions).  T[i][8] = sum w_i and S[8][8] (the row count) are added on the
// CUDA cores.
constexpr int kFit8Warps = 8;
constexpr int kFit8PosPerWarp = 4;

// x rounded to tf32 (10 explicit mantissa bits), to nearest with ties away from
// zero, on the integer pipe: add half of the 13 dropped bits to the magnitude
// and clear them (a carry moves into the exponent, as it should)
__device__ __forceinline__ uint32_t to_tf32(float x) {
  return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
}
// d = A B (from zero) or d += A B
__device__ __forceinline__ void mma_tf32_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}
__device__ __forceinline__ void mma_tf32_1688_acc(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Each warp streams its 8-row steps through a ring of kFit8Stages shared-memory
// stages by cp.async (rows padded to 160 bytes: the lanes' reads hit distinct
// banks), so that kFit8Stages - 1 steps of W0 are in flight per warp.
constexpr int kFit8Stages = 6;
constexpr int kFit8Pitch = 160;                              // bytes per staged row of W0
constexpr int kFit8StageBytes = 8 * kFit8Pitch + 8 * 16;     // W0 rows + the rows' code words
constexpr int kFit8RingBytes = kFit8Warps * kFit8Stages * kFit8StageBytes;

__device__ __forceinline__ void fit_cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void fit_cp_async(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

__global__ void __launch_bounds__(kFit8Warps * 32, 2) fit8_mma_kernel(
    const float* __restrict__ W0, const uint32_t* __restrict__ codes, int64_t N, int64_t groups,
    int64_t row_splits, const float* __restrict__ h, double* __restrict__ partials) {
  using F = FitDims<8>;
  constexpr int P = F::P, kT = 8 * P;
  __shared__ double pos[kFitLanes][F::SG + kT];
  extern __shared__ __align__(16) unsigned char fit8_ring[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t ct = int64_t(blockIdx.x) / row_splits, rs = int64_t(blockIdx.x) % row_splits;
  const int64_t rows_per = ceil_div(N, row_splits);
  const int64_t r_begin = rs * rows_per, r_end = r_begin + rows_per < N ? r_begin + rows_per : N;
  const int64_t K = groups * 8;
  const int64_t words_per_row = K / 16;
  const int64_t g0 = ct * kFitLanes + warp * kFit8PosPerWarp;  // first position of this warp
  const uint32_t one_row = gq == 0 ? __float_as_uint(1.0f) : 0u;  // A_S row 8
  unsigned char* ring = fit8_ring + warp * (kFit8Stages * kFit8StageBytes);
  const uint32_t ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(ring));

  // step t covers rows r_begin + 8 t ..; lane l copies 16-byte chunks l and l + 32
  // of its 8 x 128 bytes of W0 (row c / 8, chunk c % 8), lanes 0..15 code word
  // l % 2 of row l / 2.  Sources advance by 8 rows per step; only the last,
  // partial step checks rows.
  const int nsteps = static_cast<int>(ceil_div(r_end - r_begin, 8));
  const int nfull = static_cast<int>((r_end - r_begin) / 8);
  const int crow0 = lane >> 3, ccol = lane & 7;  // chunk lane: row crow0 (and crow0 + 4), column ccol
  const bool wcol_ok = g0 + (ccol >> 1) < groups;
  const float* wsrc = W0 + (r_begin + crow0) * K + g0 * 8 + ccol * 4;
  const int64_t wstep = 8 * K, wrow4 = 4 * K;
  const uint32_t wdst = static_cast<uint32_t>(crow0 * kFit8Pitch + ccol * 16);
  const int cv = lane & 1, crow = (lane >> 1) & 7;
  const bool ccol_ok = lane < 16 && g0 + 2 * cv < groups;
  const uint32_t* csrc = codes + (r_begin + crow) * words_per_row + (g0 >> 1) + cv;
  const int64_t cstep = 8 * words_per_row;
  const uint32_t cdst = static_cast<uint32_t>(8 * kFit8Pitch + crow * 16 + cv * 4);
  // sources of the next step to issue, advanced by one step per issue
  const float* ws = wsrc;
  const uint32_t* cs = csrc;
  auto issue = [&](int t, int stage) {
    const uint32_t st = ring_s + static_cast<uint32_t>(stage) * kFit8StageBytes;
    if (t < nfull) {
      fit_cp_async(st + wdst, wcol_ok ? static_cast<const void*>(ws) : W0, wcol_ok);
      fit_cp_async(st + wdst + 4 * kFit8Pitch, wcol_ok ? static_cast<const void*>(ws + wrow4) : W0, wcol_ok);
      if (lane < 16) fit_cp_async4(st + cdst, ccol_ok ? static_cast<const void*>(cs) : codes, ccol_ok);
    } else {
      const int64_t n0 = r_begin + 8 * int64_t(t);
      const bool ra = n0 + crow0 < r_end, rb = n0 + crow0 + 4 < r_end, rc = n0 + crow < r_end;
      fit_cp_async(st + wdst, wcol_ok && ra ? static_cast<const void*>(ws) : W0, wcol_ok && ra);
      fit_cp_async(st + wdst + 4 * kFit8Pitch, wcol_ok && rb ? static_cast<const void*>(ws + wrow4) : W0,
                   wcol_ok && rb);
      if (lane < 16)
        fit_cp_async4(st + cdst, ccol_ok && rc ? static_cast<const void*>(cs) : codes, ccol_ok && rc);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    ws += wstep;
    cs += cstep;
  };

  double t64[kFit8PosPerWarp][2], sw64[kFit8PosPerWarp];
  float t32[kFit8PosPerWarp][2], s32[kFit8PosPerWarp][4], sw32[kFit8PosPerWarp];
#pragma unroll
  for (int q = 0; q < kFit8PosPerWarp; ++q) {
    t64[q][0] = t64[q][1] = 0.0, t32[q][0] = t32[q][1] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) s32[q][e] = 0.f;
    sw64[q] = 0.0, sw32[q] = 0.f;
  }
  for (int t = 0; t < kFit8Stages - 1; ++t) {
    if (t < nsteps) issue(t, t);
    else asm volatile("cp.async.commit_group;\n" ::: "memory");
  }
  int flush_steps = 0;
  int s_use = 0, s_issue = kFit8Stages - 1;
  // lane's reads in a stage: rows tq and tq + 4, channel gq of each position
  const uint32_t ra_off = static_cast<uint32_t>(tq * kFit8Pitch + gq * 4);
  const uint32_t ca_off = static_cast<uint32_t>(8 * kFit8Pitch + tq * 16);
  for (int t = 0; t < nsteps; ++t) {
    // keep kFit8Stages - 1 steps in flight: issue step t + S - 1, then wait for step t
    if (t + kFit8Stages - 1 < nsteps) issue(t + kFit8Stages - 1, s_issue);
    else asm volatile("cp.async.commit_group;\n" ::: "memory");
    s_issue = s_issue + 1 == kFit8Stages ? 0 : s_issue + 1;
    asm volatile("cp.async.wait_group %0;\n" ::"n"(kFit8Stages - 1) : "memory");
    __syncwarp();
    const unsigned char* st = ring + s_use * kFit8StageBytes;
    s_use = s_use + 1 == kFit8Stages ? 0 : s_use + 1;
    const uint2 cwa = *reinterpret_cast<const uint2*>(st + ca_off);
    const uint2 cwb = *reinterpret_cast<const uint2*>(st + ca_off + 4 * 16);
#pragma unroll
    for (int q = 0; q < kFit8PosPerWarp; ++q) {
      const float wa = *reinterpret_cast<const float*>(st + ra_off + q * 32);
      const float wb = *reinterpret_cast<const float*>(st + ra_off + 4 * kFit8Pitch + q * 32);
      const uint32_t sh = 16u * (q & 1) + 2u * gq;  // code gq of position q within its word
      const uint32_t wa_c = (q >> 1) ? cwa.y : cwa.x, wb_c = (q >> 1) ? cwb.y : cwb.x;
      const uint32_t za = __float_as_uint(__int_as_float(0x4B000000 | ((wa_c >> sh) & 3u)) - 8388608.0f);
      const uint32_t zb = __float_as_uint(__int_as_float(0x4B000000 | ((wb_c >> sh) & 3u)) - 8388608.0f);
      const uint32_t ha = to_tf32(wa), hb = to_tf32(wb);
      const uint32_t la = to_tf32(wa - __uint_as_float(ha)), lb = to_tf32(wb - __uint_as_float(hb));
      float d[4];
      mma_tf32_1688(d, ha, la, hb, lb, za, zb);
      t32[q][0] += d[0] + d[2];  // rows gq (hi) and gq + 8 (lo)
      t32[q][1] += d[1] + d[3];
      mma_tf32_1688_acc(s32[q], za, one_row, zb, one_row, za, zb);
      sw32[q] += wa + wb;
    }
    __syncwarp();  // the stage is read before a later issue overwrites it
    if (++flush_steps == kFitFlush / 8) {  // t32: kFitFlush terms; sw32: 2 per step
      flush_steps = 0;
#pragma unroll
      for (int q = 0; q < kFit8PosPerWarp; ++q) {
        t64[q][0] += double(t32[q][0]), t64[q][1] += double(t32[q][1]);
        t32[q][0] = t32[q][1] = 0.f;
        sw64[q] += double(sw32[q]), sw32[q] = 0.f;
      }
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
#pragma unroll
  for (int q = 0; q < kFit8PosPerWarp; ++q) {
    t64[q][0] += double(t32[q][0]), t64[q][1] += double(t32[q][1]);
    sw64[q] += double(sw32[q]);
    // lanes of one channel gq: tq = 0..3 (xor over lane bits 0, 1)
    sw64[q] += __shfl_xor_sync(0xffffffffu, sw64[q], 1);
    sw64[q] += __shfl_xor_sync(0xffffffffu, sw64[q], 2);
  }
  // scatter into pos[l][S upper triangle | T[i][j]] for l = 4 warp + q
  auto sidx = [](int a, int b) {  // upper-triangle index of (a <= b) in a P x P matrix
    return a * P - a * (a - 1) / 2 + (b - a);
  };
#pragma unroll
  for (int q = 0; q < kFit8PosPerWarp; ++q) {
    double* pp = &pos[warp * kFit8PosPerWarp + q][0];
    const int j0 = 2 * tq;
    // T: D rows gq (hi) and gq + 8 (lo), columns 2tq, 2tq + 1
    pp[F::SG + gq * P + j0] = t64[q][0];
    pp[F::SG + gq * P + j0 + 1] = t64[q][1];
    if (tq == 0) pp[F::SG + gq * P + 8] = sw64[q];
    // S: rows a = gq, columns b = 2tq, 2tq + 1 (upper triangle: a <= b)
    if (gq <= j0) pp[sidx(gq, j0)] = double(s32[q][0]);
    if (gq <= j0 + 1) pp[sidx(gq, j0 + 1)] = double(s32[q][1]);
    if (gq == 0) {  // row 8 (the ones): S[8][b] = sum z_b, stored as S[b][8]
      pp[sidx(j0, 8)] = double(s32[q][2]);
      pp[sidx(j0 + 1, 8)] = double(s32[q][3]);
    }
    if (lane == 0) pp[sidx(8, 8)] = double(r_end > r_begin ? r_end - r_begin : 0);
  }
  __syncthreads();
  // h per coordinate, positions in order: one partial [8][G_i (SG), R_i (P)]
  for (int e = tid; e < 8 * F::S; e += kFit8Warps * 32) {
    const int i = e / F::S, q = e % F::S;
    double t = 0.0;
    for (int l = 0; l < kFitLanes; ++l) {
      const int64_t gg = ct * kFitLanes + l;
      if (gg >= groups) break;
      const double hw = h ? double(__ldg(h + gg * 8 + i)) : 1.0;
      const double v = q < F::SG ? pos[l][q] : pos[l][F::SG + i * P + (q - F::SG)];
      t += hw * v;
    }
    partials[int64_t(blockIdx.x) * 8 * F::S + e] = t;
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

// One CTA per coordinate i: sums its (d+1)(d+2)/2 + (d+1) values over the
// partials -- thread (q, c) adds partials c, c + 4, c + 8, ... of value q in
// order, 14 loads in flight, and the 4 chunk sums are added in chunk order
// (a fixed order: bitwise reproducible) -- then solves theta_i.
constexpr int kSolveChunks = 4;
constexpr int kSolveBatch = 14;

template <int D>
__global__ void __launch_bounds__(256) fit_solve_kernel(const double* __restrict__ partials,
                                                        int num_parts, float* __restrict__ A,
                                                        float* __restrict__ B) {
  using F = FitDims<D>;
  static_assert(F::S * kSolveChunks <= 256, "one thread per value and chunk");
  __shared__ double part[kSolveChunks][F::S];
  const int i = blockIdx.x;
  const int t = threadIdx.x;
  if (t < F::S * kSolveChunks) {
    const int q = t % F::S, c = t / F::S;
    const int64_t pitch = int64_t(D) * F::S * kSolveChunks;  // partials c, c + 4, ...
    const double* src = partials + int64_t(c) * D * F::S + i * F::S + q;
    double acc = 0.0;
    int p = c;
    for (; p + kSolveChunks * (kSolveBatch - 1) < num_parts; p += kSolveChunks * kSolveBatch) {
      double v[kSolveBatch];
#pragma unroll
      for (int u = 0; u < kSolveBatch; ++u) v[u] = src[int64_t(u) * pitch];
#pragma unroll
      for (int u = 0; u < kSolveBatch; ++u) acc += v[u];
      src += int64_t(kSolveBatch) * pitch;
    }
    for (; p < num_parts; p += kSolveChunks) {
      acc += *src;
      src += pitch;
    }
    part[c][q] = acc;
  }
  __syncthreads();
  if (t != 0) return;
  double tot[F::S];
  for (int q = 0; q < F::S; ++q) {
    double v = 0.0;
    for (int c = 0; c < kSolveChunks; ++c) v += part[c][q];
    tot[q] = v;
  }
  double G[F::P][F::P], R[F::P], th[F::P];
  int s = 0;
  for (int a = 0; a < F::P; ++a)
    for (int b = a; b < F::P; ++b) {
      G[a][b] = tot[s];
      G[b][a] = tot[s];
      ++s;
    }
  for (int a = 0; a < F::P; ++a) R[a] = tot[F::SG + a];
  if (!cholesky_solve<F::P>(G, R, th)) pinv_solve<F::P>(G, R, th);
  for (int j = 0; j < D; ++j) A[i * D + j] = static_cast<float>(th[j]);
  B[i] = static_cast<float>(th[D]);
}

// column tiles of 32 positions times row splits, about two CTAs per SM
struct FitGrid {
  int64_t tiles, splits;
  int64_t ctas() const { return tiles * splits; }
};
inline FitGrid fit_grid(int64_t d_out, int64_t groups) {
  FitGrid f{ceil_div(groups > 0 ? groups : 1, kFitLanes), 1};
  if (f.tiles < kFitTargetCtas) f.splits = kFitTargetCtas / f.tiles;
  const int64_t max_splits = ceil_div(d_out > 0 ? d_out : 1, 16);
  if (f.splits > max_splits) f.splits = max_splits;
  // the code Gram stays exact in fp32 while a CTA's rows times 9 is below 2^24
  const int64_t min_splits = ceil_div(d_out > 0 ? d_out : 1, int64_t(1) << 20);
  if (f.splits < min_splits) f.splits = min_splits;
  if (f.splits < 1) f.splits = 1;
  return f;
}

template <int D>
cudaError_t launch_fit_t(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                         const float* h, float* A, float* B, double* partials, cudaStream_t s,
                         int* launches) {
  const int64_t groups = d_in / D;
  const FitGrid fg = fit_grid(d_out, groups);
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(packed);
  if constexpr (D == 8) {
    auto kern8 = fit8_mma_kernel;
    if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern8), kFit8RingBytes);
        e != cudaSuccess)
      return e;
    kern8<<<static_cast<unsigned>(fg.ctas()), kFit8Warps * 32, kFit8RingBytes, s>>>(
        W0, codes, d_out, groups, fg.splits, h, partials);
  } else {
    auto kern = fit_accum_kernel<D>;
    if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), FitSmem<D>::kBytes);
        e != cudaSuccess)
      return e;
    kern<<<static_cast<unsigned>(fg.ctas()), kFitThreads2, FitSmem<D>::kBytes, s>>>(
        W0, codes, d_out, groups, fg.splits, h, partials);
  }
  ++*launches;
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  fit_solve_kernel<D><<<D, 256, 0, s>>>(partials, static_cast<int>(fg.ctas()), A, B);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

size_t fit_partials_bytes(int64_t d_out, int64_t d_in, int d) {
  if (d <= 0) return 0;
  const size_t ctas = size_t(fit_grid(d_out, d_in / d).ctas());
  switch (d) {
    case 1: return ctas * 1 * FitDims<1>::S * sizeof(double);
    case 2: return ctas * 2 * FitDims<2>::S * sizeof(double);
    case 4: return ctas * 4 * FitDims<4>::S * sizeof(double);
    default: return ctas * 8 * FitDims<8>::S * sizeof(double);
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

// Tensor-core GEMMs of the LC-VQ layer on tcgen05 (sm_100a): the prefill
// forward in both formulations, and the two contractions of the straight-
// through backward.  One persistent, warp-specialized kernel template:
//
//   warp 0          TMA producer: A tiles, and B tiles or packed-code tiles
//   warp 1          TMEM allocator + single-thread MMA issuer
//   DEC warps       code decoders: packed 2-bit codes in shared memory ->
//                   bf16 B tiles in the SW128 layout the MMA reads
//   4 warps         epilogue: TMEM -> registers -> fused epilogue -> global
//
// D tiles are 128 x 256 fp32 in TMEM, double buffered (512 columns), so the
// epilogue of one tile overlaps the main loop of the next.  Shared memory holds
// STAGES (A, B, codes) stages; mbarriers hand them between the roles.  Every
// wait is bounded: a wait that gives up records LCVQ_ERR_DEVICE_TIMEOUT in the
// workspace error word and the kernel winds down without trapping.
//
// Kinds (D[i][j] = sum_c A[i][c] B[j][c]):
//   FwdAlg  Y[m][n]  = sum_k X''[m][k] v[n][k] + corr[m]      A = X'' (K-major)
//           v = 128 + 4^p z: one LOP3 per bf16 pair (see xform.cu)
//   FwdDec  Y[m][n]  = sum_k X[m][k] bf16(A z + B)[n][k]      A = X (K-major)
//           decoders evaluate A z + B in fp32 (LC-QAT Methodology 1, c = A z + B)
//   Dx      P[m][k]  = sum_n dY[m][n] v[n][k]                 A = dY (K-major),
//           B = codes as an MN-major operand; the epilogue maps P back to
//           dX[m][g d + i] = sum_j A[i][j] Pz[m][g d + j] + B[i] r[m]
//           with Pz = (P - 128 r) 4^-p, r[m] = sum_n dY[m][n]  (gradient through
//           the linear map, Methodology 1)
//   Dw      G[n][k]  = sum_m dY[m][n] X[m][k]                 A = dY^T, B = X^T
//           (both MN-major); the epilogue never stores G: it writes
//           dWp = mask * A^T G per d-vector (STE, Methodology 3) and accumulates
//           sum G_i z_j, sum G_i into per-CTA partials of dA, dB.
//   Gram    C[r][c]  = sum_n P[n][r] Q[n][c]                  A = P^T, B = Q^T
//           (both MN-major, bf16 from TMA); the epilogue stores C in fp32.  The
//           refit under a full Hessian forms the code Gram and the targets
//           times the codes this way (fit_h.cu).
#include <cudaTypedefs.h>

#include <mutex>

#include "codec.cuh"
#include "common.cuh"
#include "decode_mma.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lcvq {

using namespace sm100;

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int C_BYTES = 4096;         // packed codes of one stage
// CTA pairs: k blocks per forwarded "odd half decoded" arrive (measured on the
// 2048 x 4096 -> 11008 decode form: 1, 2, 3 -> 724, 815, 857 TFLOP/s)
constexpr int kPairPeerGroup = 3;
constexpr int kTmemCols = 512;

enum Kind { kFwdAlg = 0, kFwdDec = 1, kDx = 2, kDw = 3, kGram = 4 };

struct Params {
  int64_t M, N, K;    // D is M x N, contraction K (see each kind)
  int64_t d_in, d_out;
  const uint8_t* codes;
  const uint8_t* mask;
  const float* corr;
  const float* rsum;
  const float* Amat;
  const float* Bvec;
  void* out;
  float* partials;
  unsigned int* err;
};

template <int KIND, int DW>
struct Cfg {
  static constexpr int kThreads = 32 * (2 + DW + 4);
  static constexpr bool kHasCodes = KIND != kDw && KIND != kGram;
  static constexpr bool kAmn = KIND == kDw || KIND == kGram;
  static constexpr bool kBmn = KIND == kDx || KIND == kDw || KIND == kGram;
  static constexpr uint32_t kStageTx = A_BYTES + (kHasCodes ? C_BYTES : B_BYTES);
};

// 1024 B of alignment slack, the stages, then barriers, TMEM address, abort
// flag, A/B (<= 72 floats) and the dA/dB reduction scratch (4 x 72 floats)
constexpr size_t kTailBytes = 4096;
constexpr size_t kSmemBytes = 1024 + size_t(STAGES) * (A_BYTES + B_BYTES + C_BYTES) + kTailBytes;

// Tile order: bands of kBand D-row tiles, column-major inside a band, so the
// CTAs that run at the same time share a few row blocks and a few column
// blocks of the operands (both stay in L2 while the contraction sweeps).
__device__ __forceinline__ void tile_coords(int64_t tile, int64_t m_tiles, int64_t n_tiles,
                                            int band, int& mt, int& nt) {
  const int64_t per_band = int64_t(band) * n_tiles;
  const int64_t b = tile / per_band, r = tile % per_band;
  const int64_t rows = (b + 1) * band <= m_tiles ? band : m_tiles - b * band;
  mt = static_cast<int>(b * band + r % rows);
  nt = static_cast<int>(r / rows);
}

__device__ __forceinline__ void fail(const Params& p, volatile int* abort_flag, unsigned site) {
  record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, site);
  *abort_flag = 1;
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// One 32-column chunk of a D row (registers r[] from TMEM): the fused
// epilogue of each kind.  gm is the D row, gn0 the first D column.
template <int KIND, int D>
__device__ __forceinline__ void epilogue_chunk(const Params& p, const float* sAm,
                                               const uint32_t (&r)[32], int64_t gm, int64_t gn0,
                                               float addc, float rs, float (&pa)[D * D],
                                               float (&pb)[D]) {
  if constexpr (KIND == kFwdAlg || KIND == kFwdDec) {
    uint16_t* Y = static_cast<uint16_t*>(p.out) + gm * p.N + gn0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (gn0 + 8 * q >= p.N) break;
      uint4 v;
      v.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]) + addc, __uint_as_float(r[8 * q + 1]) + addc);
      v.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]) + addc, __uint_as_float(r[8 * q + 3]) + addc);
      v.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]) + addc, __uint_as_float(r[8 * q + 5]) + addc);
      v.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]) + addc, __uint_as_float(r[8 * q + 7]) + addc);
      *reinterpret_cast<uint4*>(Y + 8 * q) = v;
    }
  } else if constexpr (KIND == kDx) {
    uint16_t* dX = static_cast<uint16_t*>(p.out) + gm * p.N + gn0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {  // two 16-blocks of output k
      float pz[16];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const float inv = (cc % 3 == 0) ? 1.0f : ((cc % 3 == 1) ? 0.25f : 0.0625f);
        pz[cc] = (__uint_as_float(r[16 * b + 2 * cc]) - 128.0f * rs) * inv;
        pz[cc + 8] = (__uint_as_float(r[16 * b + 2 * cc + 1]) - 128.0f * rs) * inv;
      }
      float o[16];
#pragma unroll
      for (int v = 0; v < 16 / D; ++v)
#pragma unroll
        for (int i = 0; i < D; ++i) {
          float a = sAm[D * D + i] * rs;
#pragma unroll
          for (int j = 0; j < D; ++j) a = fmaf(sAm[i * D + j], pz[v * D + j], a);
          o[v * D + i] = a;
        }
      uint4 v0, v1;
      v0.x = pack_bf16x2(o[0], o[1]); v0.y = pack_bf16x2(o[2], o[3]);
      v0.z = pack_bf16x2(o[4], o[5]); v0.w = pack_bf16x2(o[6], o[7]);
      v1.x = pack_bf16x2(o[8], o[9]); v1.y = pack_bf16x2(o[10], o[11]);
      v1.z = pack_bf16x2(o[12], o[13]); v1.w = pack_bf16x2(o[14], o[15]);
      reinterpret_cast<uint4*>(dX + 16 * b)[0] = v0;
      reinterpret_cast<uint4*>(dX + 16 * b)[1] = v1;
    }
  } else if constexpr (KIND == kGram) {
    float* C = static_cast<float*>(p.out) + gm * p.N + gn0;
    if (gn0 + 32 <= p.N) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(C)[q] =
            make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                        __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (gn0 + q < p.N) C[q] = __uint_as_float(r[q]);
    }
  } else {  // kDw: D row = n (d_out), D column = k (d_in)
    const int64_t n = gm, k0 = gn0;
    const uint2 zc = *reinterpret_cast<const uint2*>(p.codes + n * (p.d_in / 4) + k0 / 4);
    const uint32_t mb = p.mask != nullptr
                            ? *reinterpret_cast<const uint32_t*>(p.mask + n * (p.d_in / 8) + k0 / 8)
                            : 0xFFFFFFFFu;
    float* dWp = static_cast<float*>(p.out);
    float o[32];
#pragma unroll
    for (int v = 0; v < 32 / D; ++v) {
      float G[D], z[D];
#pragma unroll
      for (int i = 0; i < D; ++i) G[i] = __uint_as_float(r[v * D + i]);
#pragma unroll
      for (int j = 0; j < D; ++j) {
        const int e = v * D + j;
        const uint32_t word = e < 16 ? zc.x : zc.y;
        z[j] = static_cast<float>((word >> (2 * (e & 15))) & 3u);
      }
#pragma unroll
      for (int i = 0; i < D; ++i) {
        pb[i] += G[i];
#pragma unroll
        for (int j = 0; j < D; ++j) pa[i * D + j] = fmaf(G[i], z[j], pa[i * D + j]);
      }
#pragma unroll
      for (int j = 0; j < D; ++j) {
        float sacc = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) sacc = fmaf(sAm[i * D + j], G[i], sacc);
        o[v * D + j] = ((mb >> (v * D + j)) & 1u) ? sacc : 0.f;
      }
    }
    if (dWp != nullptr) {
      float4* dst = reinterpret_cast<float4*>(dWp + n * p.d_in + k0);
#pragma unroll
      for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    }
  }
}

// Per-CTA partials of dA and dB: warp tree, then the 4 epilogue warps in a
// fixed order; one row of p.partials per CTA.
template <int D>
__device__ __forceinline__ void dw_block_partials(const Params& p, float (&pa)[D * D],
                                                  float (&pb)[D], float* sRed, int quarter,
                                                  int lane) {
  // per-CTA partials of dA, dB: warp tree, then the 4 warps in order
  constexpr int NP = D * D + D;
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    float x = e < D * D ? pa[e] : pb[e - D * D];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xffffffffu, x, off);
    if (lane == 0) sRed[quarter * NP + e] = x;
  }
  asm volatile("bar.sync 1, 128;\n" ::: "memory");  // the 4 epilogue warps only
  if (quarter == 0 && lane < 1) {
    for (int e = 0; e < NP; ++e)
      p.partials[int64_t(blockIdx.x) * NP + e] =
          ((sRed[e] + sRed[NP + e]) + sRed[2 * NP + e]) + sRed[3 * NP + e];
  }
}

template <int KIND, int D, int DW>
__global__ void __launch_bounds__(Cfg<KIND, DW>::kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const Params p) {
  using C = Cfg<KIND, DW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sC = sB + STAGES * B_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + STAGES * C_BYTES);
  uint64_t* full = bars;
  uint64_t* decd = bars + STAGES;
  uint64_t* empty = bars + 2 * STAGES;
  uint64_t* tfull = bars + 3 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* sAm = reinterpret_cast<float*>(tmem_holder + 4);  // D*D + D floats
  float* sRed = sAm + 80;                                 // 4 x (D*D + D) floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kBand = 16;
  const int64_t m_tiles = ceil_div(p.M, BM), n_tiles = ceil_div(p.N, BN);
  const int64_t tiles = m_tiles * n_tiles;
  const int64_t kblocks = ceil_div(p.K, BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&decd[s], DW > 0 ? DW : 1);     // one arrive per decoder warp
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);                 // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (KIND != kFwdAlg && KIND != kGram) {  // these never touch A, B
    if (threadIdx.x < D * D) sAm[threadIdx.x] = p.Amat[threadIdx.x];
    if (KIND != kDw && threadIdx.x >= 64 && threadIdx.x < 64 + D)
      sAm[D * D + threadIdx.x - 64] = p.Bvec[threadIdx.x - 64];
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const long long lim = wait_limit(p.err);
  // the abort flag as one decision per warp (lane 0's read), for the roles whose
  // lanes go on to warp-wide instructions together
  auto warp_abort = [&]() { return __shfl_sync(0xffffffffu, *abort_flag, 0) != 0; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t tile = blockIdx.x; tile < tiles && !*abort_flag; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, m_tiles, n_tiles, kBand, mt, nt);
        for (int64_t kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, lim)) { fail(p, abort_flag, 1); break; }
          if (*abort_flag) break;
          ++issued;
          mbar_arrive_expect_tx(&full[s], C::kStageTx);
          const int kx = static_cast<int>(kb);
          if constexpr (KIND == kFwdAlg || KIND == kFwdDec) {
            tma_load_2d(&tmA, &full[s], sA + s * A_BYTES, kx * BK, mt * BM);
            tma_load_2d(&tmB, &full[s], sC + s * C_BYTES, kx * (BK / 4), nt * BN);
          } else if constexpr (KIND == kDx) {
            tma_load_2d(&tmA, &full[s], sA + s * A_BYTES, kx * BK, mt * BM);
            tma_load_2d(&tmB, &full[s], sC + s * C_BYTES, nt * (BN / 4), kx * BK);
          } else {
            tma_load_2d(&tmA, &full[s], sA + s * A_BYTES, mt * BM, kx * BK);
            tma_load_2d(&tmA, &full[s], sA + s * A_BYTES + 8192, mt * BM + 64, kx * BK);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tma_load_2d(&tmB, &full[s], sB + s * B_BYTES + q * 8192, nt * BN + q * 64, kx * BK);
          }
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) {  // no copy may land in shared memory after the CTA exits
        // (the default limit: copies in flight finish in microseconds)
        for (int64_t n = issued - 1; n >= 0 && n >= issued - STAGES; --n)
          mbar_wait(&full[n % STAGES], static_cast<uint32_t>((n / STAGES) & 1), kDefaultWaitLimit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, C::kAmn, C::kBmn);
      int s = 0;
      uint32_t ph = 0;
      int64_t local = 0;
      bool issued = false;
      for (int64_t tile = blockIdx.x; tile < tiles && !*abort_flag; tile += gridDim.x, ++local) {
        const int buf = static_cast<int>(local & 1);
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1) ^ 1, lim)) { fail(p, abort_flag, 2); break; }
        tc_fence_after();
        const uint32_t dt = tmem + buf * BN;
        bool ok = true;
        for (int64_t kb = 0; kb < kblocks; ++kb) {
          uint64_t* ready = (DW > 0) ? &decd[s] : &full[s];
          if (!mbar_wait(ready, ph, lim)) { fail(p, abort_flag, 3); ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = C::kAmn ? sdesc_sw128(a0 + k * 2048, 8192, 1024)
                                        : sdesc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = C::kBmn ? sdesc_sw128(b0 + k * 2048, 8192, 1024)
                                        : sdesc_sw128(b0 + k * 32, 16, 1024);
            mma_ss(dt, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit(&empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
      }
      if (issued) {  // no MMA may still run when TMEM is released
        mma_commit(drain);
        // the default limit: running MMAs finish in microseconds, and TMEM may
        // be released only after them
        if (!mbar_wait(drain, 0, kDefaultWaitLimit)) fail(p, abort_flag, 4);
      }
    }
  } else if (warp < 2 + DW) {
    // ------------------------------------------------------------ decoders
    const int dt = threadIdx.x - 64;  // 0 .. 32*DW-1
    int s = 0;
    uint32_t ph = 0;
    for (int64_t tile = blockIdx.x; tile < tiles && !warp_abort(); tile += gridDim.x) {
      for (int64_t kb = 0; kb < kblocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, lim))) {  // one outcome per warp
          fail(p, abort_flag, 5);
          break;
        }
        const uint8_t* cs = sC + s * C_BYTES;
        const uint32_t bs = smem_u32(sB + s * B_BYTES);
        if constexpr (KIND == kFwdAlg) {
#pragma unroll
          for (int rr = 0; rr < BN / (32 * DW); ++rr) {
            const int r = dt + rr * 32 * DW;
            const uint4 cw = *reinterpret_cast<const uint4*>(cs + r * 16);
            const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
            const uint32_t row = bs + r * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 c0, c1;
              dec_word(w[q], c0, c1);
              st_shared_v4(row + (((2 * q) ^ (r & 7)) << 4), c0);
              st_shared_v4(row + (((2 * q + 1) ^ (r & 7)) << 4), c1);
            }
          }
        } else if constexpr (KIND == kFwdDec) {
#pragma unroll
          for (int rr = 0; rr < BN / (32 * DW); ++rr) {
            const int r = dt + rr * 32 * DW;
            const uint4 cw = *reinterpret_cast<const uint4*>(cs + r * 16);
            const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
            const uint32_t row = bs + r * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 16 natural-order weights per word
              float o[16];
#pragma unroll
              for (int v = 0; v < 16 / D; ++v) {
                float z[D];
#pragma unroll
                for (int j = 0; j < D; ++j) z[j] = static_cast<float>((w[q] >> (2 * (v * D + j))) & 3u);
#pragma unroll
                for (int i = 0; i < D; ++i) {
                  float a = sAm[D * D + i];
#pragma unroll
                  for (int j = 0; j < D; ++j) a = fmaf(sAm[i * D + j], z[j], a);
                  o[v * D + i] = a;
                }
              }
              const uint4 c0 = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                          pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
              const uint4 c1 = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                                          pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
              st_shared_v4(row + (((2 * q) ^ (r & 7)) << 4), c0);
              st_shared_v4(row + (((2 * q + 1) ^ (r & 7)) << 4), c1);
            }
          }
        } else if constexpr (KIND == kDx) {
          // codes tile [64 contraction rows n][64 B = 256 output k]; B tile is
          // MN-major: 4 blocks of 64 k (8 KB), each [64 n lines][128 B]
#pragma unroll
          for (int it = 0; it < (64 * 4) / (32 * DW); ++it) {
            const int u = dt + it * 32 * DW;  // (row n_l, block q): a warp = 32 rows of one block
            const int nl = u & 63, q = u >> 6;
            const uint4 cw = *reinterpret_cast<const uint4*>(cs + nl * 64 + q * 16);
            const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
            const uint32_t line = bs + q * 8192 + nl * 128;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              uint4 c0, c1;
              dec_word(w[qq], c0, c1);
              st_shared_v4(line + (((2 * qq) ^ (nl & 7)) << 4), c0);
              st_shared_v4(line + (((2 * qq + 1) ^ (nl & 7)) << 4), c1);
            }
          }
        }
        fence_async_smem();  // this lane's B tile stores -> visible to the MMA
        __syncwarp();
        if (lane == 0) mbar_arrive(&decd[s]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    float pa[D * D], pb[D];
    if constexpr (KIND == kDw) {
#pragma unroll
      for (int i = 0; i < D * D; ++i) pa[i] = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) pb[i] = 0.f;
    }
    int64_t local = 0;
    for (int64_t tile = blockIdx.x; tile < tiles && !warp_abort(); tile += gridDim.x, ++local) {
      int mt, nt;
      tile_coords(tile, m_tiles, n_tiles, kBand, mt, nt);
      const int buf = static_cast<int>(local & 1);
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], use & 1, lim))) {  // one outcome per warp
        fail(p, abort_flag, 6);
        break;
      }
      tc_fence_after();
      const int64_t gm = int64_t(mt) * BM + row;  // D row
      const uint32_t tbase = tmem + buf * BN + (static_cast<uint32_t>(quarter * 32) << 16);
      float addc = 0.f;
      if constexpr (KIND == kFwdAlg) addc = gm < p.M ? p.corr[gm] : 0.f;
      float rs = 0.f;
      if constexpr (KIND == kDx) rs = gm < p.M ? p.rsum[gm] : 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_ld_wait();
        const int64_t gn0 = int64_t(nt) * BN + c * 32;  // first D column of the chunk
        if (gm >= p.M || gn0 >= p.N) continue;
        epilogue_chunk<KIND, D>(p, sAm, r, gm, gn0, addc, rs, pa, pb);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
    if constexpr (KIND == kDw) dw_block_partials<D>(p, pa, pb, sRed, quarter, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- CTA pairs
// The same GEMMs on CTA pairs (cta_group::2): a pair computes a 256 x 256 tile;
// each CTA holds 128 rows of A and 128 rows (N) of B, the even CTA issues the
// 256 x 256 x 16 MMAs for both and each CTA's TMEM receives its 128 rows of D.
// Per SM this halves the B tile the tensor core reads and the codes each CTA
// decodes.  Barriers: fullA/decd/tempty/drain live in the even CTA (the
// odd CTA's TMA loads and arrivals are counted there); fullC, empty and tfull
// are per CTA (the MMA commits arrive on both CTAs' copies).
template <int KIND, int DW>
struct Cfg2 {
  static constexpr int kThreads = 32 * (2 + DW + 4);
  // groups of decoder warps take alternate k blocks: 8-warp groups for the
  // decode form (a group decodes a stage's 128 rows with 8 warps), 4-warp
  // groups otherwise
  static constexpr int kDecGroups = DW < 8 ? 1 : (KIND == kFwdDec ? DW / 8 : DW / 4);
  static constexpr int kDecGroupWarps = DW / kDecGroups > 0 ? DW / kDecGroups : 1;
  static constexpr bool kHasCodes = KIND != kDw;
  static constexpr bool kAmn = KIND == kDw;
  static constexpr bool kBmn = KIND == kDx || KIND == kDw;
  static constexpr int kStages = 6;
  static constexpr int kA = 16384;                      // 128 rows x 64 bf16
  static constexpr int kB = 16384;                      // this CTA's 128 rows of B
  static constexpr int kC = kHasCodes ? 2048 : 0;       // codes of those 128 rows
  static constexpr int kStage = kA + kB + kC;
  static constexpr uint32_t kOperandTx = kHasCodes ? kA : kA + kB;  // per CTA, to fullA
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStage + 4096;
};

template <int KIND, int D, int DW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg2<KIND, DW>::kThreads, 1)
    tc2_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
  using C = Cfg2<KIND, DW>;
  constexpr int S = C::kStages;
  // k blocks per odd-to-even "decoded" arrive: group q (k blocks q G .. q G + G - 1
  // of the pair's stream) uses decd_peer[q % S] in phase (q / S) & 1
  constexpr int kPeerGroup = kPairPeerGroup;
  static_assert(kPeerGroup >= 1 && kPeerGroup < S, "a group must not span the whole ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(S) * C::kStage);
  uint64_t* fullA = bars;            // [S]  even CTA: A (+B) of both CTAs landed
  uint64_t* fullC = bars + S;        // [S]  per CTA: its codes landed
  uint64_t* decd = bars + 2 * S;     // [S]  per CTA: its own B half decoded
  uint64_t* empty = bars + 3 * S;    // [S]  per CTA: the MMA is done with stage s
  uint64_t* decd_peer = bars + 4 * S; // [S] even CTA: the odd CTA's B halves of a group decoded
  uint64_t* tfull = bars + 5 * S;    // [2]  per CTA: accumulator buffer ready
  uint64_t* tempty = tfull + 2;      // [2]  even CTA: both epilogues drained the buffer
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* sAm = reinterpret_cast<float*>(tmem_holder + 4);
  float* sRed = sAm + 80;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  constexpr int kBand = 8;
  const int64_t m_tiles = ceil_div(p.M, 2 * BM), n_tiles = ceil_div(p.N, BN);
  const int64_t tiles = m_tiles * n_tiles;
  const int64_t kblocks = ceil_div(p.K, BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullA[s], 1);
      mbar_init(&fullC[s], 1);
      // this CTA's decoder warps of the group that owns stage s's k block
      mbar_init(&decd[s], DW > 0 ? C::kDecGroupWarps : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&decd_peer[s], 1);            // one forwarded arrive per group from the odd CTA
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (KIND != kFwdAlg) {
    if (threadIdx.x < D * D) sAm[threadIdx.x] = p.Amat[threadIdx.x];
    if (KIND != kDw && threadIdx.x >= 64 && threadIdx.x < 64 + D)
      sAm[D * D + threadIdx.x - 64] = p.Bvec[threadIdx.x - 64];
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const long long lim = wait_limit(p.err);
  auto warp_abort = [&]() { return __shfl_sync(0xffffffffu, *abort_flag, 0) != 0; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t tile = pair; tile < tiles && !*abort_flag; tile += npairs) {
        int mt, nt;
        tile_coords(tile, m_tiles, n_tiles, kBand, mt, nt);
        const int row0 = mt * 2 * BM + static_cast<int>(rank) * BM;  // this CTA's A rows
        const int col0 = nt * BN + static_cast<int>(rank) * (BN / 2);  // this CTA's B rows
        for (int64_t kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, lim)) { fail(p, abort_flag, 11); break; }
          if (*abort_flag) break;
          ++issued;
          uint8_t* st = smem + size_t(s) * C::kStage;
          const uint32_t fa0 = mapa_shared(smem_u32(&fullA[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&fullA[s], 2 * C::kOperandTx);
          const int kx = static_cast<int>(kb);
          if constexpr (KIND == kFwdAlg || KIND == kFwdDec) {
            mbar_arrive_expect_tx(&fullC[s], C::kC);
            tma_load_2d(&tmB, &fullC[s], st + C::kA + C::kB, kx * (BK / 4), col0);
            tma_load_2d_pair(&tmA, fa0, st, kx * BK, row0);
          } else if constexpr (KIND == kDx) {
            mbar_arrive_expect_tx(&fullC[s], C::kC);
            tma_load_2d(&tmB, &fullC[s], st + C::kA + C::kB, col0 / 4, kx * BK);
            tma_load_2d_pair(&tmA, fa0, st, kx * BK, row0);
          } else {
            tma_load_2d_pair(&tmA, fa0, st, row0, kx * BK);
            tma_load_2d_pair(&tmA, fa0, st + 8192, row0 + 64, kx * BK);
            tma_load_2d_pair(&tmB, fa0, st + C::kA, col0, kx * BK);
            tma_load_2d_pair(&tmB, fa0, st + C::kA + 8192, col0 + 64, kx * BK);
          }
          if (++s == S) { s = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) {
        // wait for this CTA's own copies in flight (codes, on its own barrier);
        // the even CTA also waits for the operand stages, which count both
        // CTAs' bytes.  The default limit: copies in flight finish quickly.
        for (int64_t n = issued - 1; n >= 0 && n >= issued - S; --n) {
          const uint32_t par = static_cast<uint32_t>((n / S) & 1);
          if (C::kHasCodes) mbar_wait(&fullC[n % S], par, kDefaultWaitLimit);
          if (rank == 0) mbar_wait(&fullA[n % S], par, kDefaultWaitLimit);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, C::kAmn, C::kBmn);
      int s = 0;
      uint32_t ph = 0;
      int64_t local = 0, it = 0;
      bool issued = false;
      for (int64_t tile = pair; tile < tiles && !*abort_flag; tile += npairs, ++local) {
        const int buf = static_cast<int>(local & 1);
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        // the odd CTA's epilogue arrives from the other SM: acquire at cluster scope
        if (!mbar_wait_cluster(&tempty[buf], (use & 1) ^ 1, lim)) { fail(p, abort_flag, 12); break; }
        tc_fence_after();
        const uint32_t dt = tmem + buf * BN;
        bool ok = true;
        for (int64_t kb = 0; kb < kblocks; ++kb, ++it) {
          if (!mbar_wait(&fullA[s], ph, lim)) { fail(p, abort_flag, 13); ok = false; break; }
          if constexpr (C::kHasCodes) {
            if (!mbar_wait(&decd[s], ph, lim)) { fail(p, abort_flag, 14); ok = false; break; }
            // the odd CTA's half of B: one cluster-scope wait per group of k blocks
            const int64_t q = it / kPeerGroup;
            if (it % kPeerGroup == 0 &&
                !mbar_wait_cluster(&decd_peer[q % S], static_cast<uint32_t>((q / S) & 1),
                                   lim)) {
              fail(p, abort_flag, 18);
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + size_t(s) * C::kStage);
          const uint32_t b0 = a0 + C::kA;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = C::kAmn ? sdesc_sw128(a0 + k * 2048, 8192, 1024)
                                        : sdesc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = C::kBmn ? sdesc_sw128(b0 + k * 2048, 8192, 1024)
                                        : sdesc_sw128(b0 + k * 32, 16, 1024);
            mma_ss_pair(dt, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit_pair(&empty[s]);
          if (++s == S) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[buf]);
      }
      if (issued) {
        mma_commit_pair(drain);
        // the default limit: TMEM may be released only after the running MMAs
        if (!mbar_wait(drain, 0, kDefaultWaitLimit)) fail(p, abort_flag, 15);
      }
    } else if (rank == 1 && lane == 0 && C::kHasCodes) {
      // odd CTA: forward "B half decoded" to the even CTA, one cluster-scope
      // arrive per group of kPeerGroup k blocks (and after the last one), so
      // the decoder warps only ever arrive locally and the cluster-scope
      // handover, whose cost sets the pace when it runs every k block, runs
      // once per group
      int s = 0;
      uint32_t ph = 0;
      int64_t it = 0;
      for (int64_t tile = pair; tile < tiles && !*abort_flag; tile += npairs) {
        const bool last_tile = tile + npairs >= tiles;
        for (int64_t kb = 0; kb < kblocks; ++kb, ++it) {
          if (!mbar_wait(&decd[s], ph, lim)) { fail(p, abort_flag, 19); break; }
          if (it % kPeerGroup == kPeerGroup - 1 || (last_tile && kb + 1 == kblocks))
            mbar_arrive_cluster(mapa_shared(smem_u32(&decd_peer[(it / kPeerGroup) % S]), 0));
          if (++s == S) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp < 2 + DW) {
    // ------------------------------------------------------------ decoders (both CTAs)
    // kGroups groups of decoder warps take alternate k blocks, so each group has
    // kGroups MMA k-block times to decode and publish one stage.
    constexpr int kGroups = C::kDecGroups;
    constexpr int kGroupWarps = C::kDecGroupWarps;
    const int grp = (warp - 2) / kGroupWarps;
    const int dt = (threadIdx.x - 64) % (32 * kGroupWarps);
    // d = 8 decode form on the tensor cores: this lane's operands of A z + B
    [[maybe_unused]] uint32_t db0 = 0, db1 = 0;
    [[maybe_unused]] float dc0 = 0.f, dc1 = 0.f;
    if constexpr (KIND == kFwdDec && D == 8)
      dec8::operands(sAm, sAm + D * D, lane >> 2, lane & 3, db0, db1, dc0, dc1);
    int s = 0;
    uint32_t ph = 0;
    int64_t it = 0;
    for (int64_t tile = pair; tile < tiles && !warp_abort(); tile += npairs) {
      for (int64_t kb = 0; kb < kblocks; ++kb, ++it) {
        if (it % kGroups != grp) {
          if (++s == S) { s = 0; ph ^= 1; }
          continue;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&fullC[s], ph, lim))) {  // one outcome per warp
          fail(p, abort_flag, 16);
          break;
        }
        uint8_t* st = smem + size_t(s) * C::kStage;
        const uint8_t* cs = st + C::kA + C::kB;
        const uint32_t bs = smem_u32(st + C::kA);
        if constexpr (KIND == kFwdAlg) {  // 128 rows, one per thread
          const int r = dt;
          const uint4 cw = *reinterpret_cast<const uint4*>(cs + r * 16);
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
          const uint32_t row = bs + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 c0, c1;
            dec_word(w[q], c0, c1);
            st_shared_v4(row + (((2 * q) ^ (r & 7)) << 4), c0);
            st_shared_v4(row + (((2 * q + 1) ^ (r & 7)) << 4), c1);
          }
        } else if constexpr (KIND == kFwdDec && D == 8) {
          // warp w of the decoders takes rows 16 w .. 16 w + 15: MMA v decodes
          // vector v of rows 16 w + g and 16 w + 8 + g (decode_mma.cuh) and
          // stores 4 bytes per lane into the rows' SW128 chunk v (conflict-free:
          // the 8 rows of one store have distinct chunk positions)
          const int g = lane >> 2, t = lane & 3;
          const int r1 = 16 * (dt >> 5) + g, r2 = r1 + 8;
          const uint4 ca = *reinterpret_cast<const uint4*>(cs + r1 * 16);
          const uint4 cb = *reinterpret_cast<const uint4*>(cs + r2 * 16);
          const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w}, wb[4] = {cb.x, cb.y, cb.z, cb.w};
          const uint32_t row1 = bs + r1 * 128, row2 = bs + r2 * 128;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint32_t sh = 16u * (v & 1) + 2u * t;
            float d4[4];
            dec8::mma(d4, dec8::code_pair_bf16(wa[v >> 1], sh), dec8::code_pair_bf16(wb[v >> 1], sh),
                      db0, db1, dc0, dc1);
            st_shared_u32(row1 + ((v ^ (r1 & 7)) << 4) + 4 * t, dec8::bf16x2_rn(d4[0], d4[1]));
            st_shared_u32(row2 + ((v ^ (r2 & 7)) << 4) + 4 * t, dec8::bf16x2_rn(d4[2], d4[3]));
          }
        } else if constexpr (KIND == kFwdDec) {  // 128 rows, two threads per row
          const int r = dt >> 1, h = dt & 1;
          const uint2 cw = *reinterpret_cast<const uint2*>(cs + r * 16 + h * 8);
          const uint32_t w[2] = {cw.x, cw.y};
          const uint32_t row = bs + r * 128;
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const int q = 2 * h + qq;
            float o[16];
#pragma unroll
            for (int v = 0; v < 16 / D; ++v) {
              float z[D];
#pragma unroll
              for (int j = 0; j < D; ++j) z[j] = static_cast<float>((w[qq] >> (2 * (v * D + j))) & 3u);
#pragma unroll
              for (int i = 0; i < D; ++i) {
                float a = sAm[D * D + i];
#pragma unroll
                for (int j = 0; j < D; ++j) a = fmaf(sAm[i * D + j], z[j], a);
                o[v * D + i] = a;
              }
            }
            const uint4 c0 = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                        pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
            const uint4 c1 = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                                        pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
            st_shared_v4(row + (((2 * q) ^ (r & 7)) << 4), c0);
            st_shared_v4(row + (((2 * q + 1) ^ (r & 7)) << 4), c1);
          }
        } else if constexpr (KIND == kDx) {  // [64 contraction rows][2 MN blocks of 64]
          const int nl = dt & 63, q = dt >> 6;
          const uint4 cw = *reinterpret_cast<const uint4*>(cs + nl * 32 + q * 16);
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
          const uint32_t line = bs + q * 8192 + nl * 128;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            uint4 c0, c1;
            dec_word(w[qq], c0, c1);
            st_shared_v4(line + (((2 * qq) ^ (nl & 7)) << 4), c0);
            st_shared_v4(line + (((2 * qq + 1) ^ (nl & 7)) << 4), c1);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&decd[s]);
        if (++s == S) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    float pa[D * D], pb[D];
    if constexpr (KIND == kDw) {
#pragma unroll
      for (int i = 0; i < D * D; ++i) pa[i] = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) pb[i] = 0.f;
    }
    int64_t local = 0;
    for (int64_t tile = pair; tile < tiles && !warp_abort(); tile += npairs, ++local) {
      int mt, nt;
      tile_coords(tile, m_tiles, n_tiles, kBand, mt, nt);
      const int buf = static_cast<int>(local & 1);
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], use & 1, lim))) {  // one outcome per warp
        fail(p, abort_flag, 17);
        break;
      }
      tc_fence_after();
      const int64_t gm = int64_t(mt) * 2 * BM + int64_t(rank) * BM + row;
      const uint32_t tbase = tmem + buf * BN + (static_cast<uint32_t>(quarter * 32) << 16);
      float addc = 0.f;
      if constexpr (KIND == kFwdAlg) addc = gm < p.M ? p.corr[gm] : 0.f;
      float rs = 0.f;
      if constexpr (KIND == kDx) rs = gm < p.M ? p.rsum[gm] : 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_ld_wait();
        const int64_t gn0 = int64_t(nt) * BN + c * 32;
        if (gm >= p.M || gn0 >= p.N) continue;
        epilogue_chunk<KIND, D>(p, sAm, r, gm, gn0, addc, rs, pa, pb);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
    }
    if constexpr (KIND == kDw) dw_block_partials<D>(p, pa, pb, sRed, quarter, lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its peer may still use its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2D tensor map: inner (contiguous) extent `inner`, `outer` rows of `row_bytes`.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              bool swizzle128) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int sms = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = kNumSMsB200;
  });
  return sms;
}

template <int KIND, int D, int DW>
cudaError_t launch_kind(const CUtensorMap& a, const CUtensorMap& b, const Params& p,
                        cudaStream_t s, int* grid_out) {
  using C = Cfg<KIND, DW>;
  auto kern = tc_gemm_kernel<KIND, D, DW>;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), kSmemBytes);
      e != cudaSuccess)
    return e;
  const int64_t tiles = ceil_div(p.M, BM) * ceil_div(p.N, BN);
  int grid = num_sms();
  if (tiles < grid) grid = static_cast<int>(tiles);
  if (grid < 1) grid = 1;
  if (grid_out) *grid_out = grid;
  kern<<<grid, C::kThreads, kSmemBytes, s>>>(a, b, p);
  return cudaGetLastError();
}

template <int KIND, int DW>
cudaError_t launch_kind_d(int d, const CUtensorMap& a, const CUtensorMap& b, const Params& p,
                          cudaStream_t s, int* grid_out) {
  switch (d) {
    case 1: return launch_kind<KIND, 1, DW>(a, b, p, s, grid_out);
    case 2: return launch_kind<KIND, 2, DW>(a, b, p, s, grid_out);
    case 4: return launch_kind<KIND, 4, DW>(a, b, p, s, grid_out);
    default: return launch_kind<KIND, 8, DW>(a, b, p, s, grid_out);
  }
}

template <int KIND, int D, int DW>
cudaError_t launch_kind2(const CUtensorMap& a, const CUtensorMap& b, const Params& p,
                         cudaStream_t s, int* grid_out) {
  using C = Cfg2<KIND, DW>;
  auto kern = tc2_gemm_kernel<KIND, D, DW>;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), C::kSmem);
      e != cudaSuccess)
    return e;
  const int64_t tiles = ceil_div(p.M, 2 * BM) * ceil_div(p.N, BN);
  int pairs = num_sms() / 2;
  if (tiles < pairs) pairs = static_cast<int>(tiles);
  if (pairs < 1) pairs = 1;
  if (grid_out) *grid_out = 2 * pairs;
  kern<<<2 * pairs, C::kThreads, C::kSmem, s>>>(a, b, p);
  return cudaGetLastError();
}

template <int KIND, int DW>
cudaError_t launch_kind2_d(int d, const CUtensorMap& a, const CUtensorMap& b, const Params& p,
                           cudaStream_t s, int* grid_out) {
  switch (d) {
    case 1: return launch_kind2<KIND, 1, DW>(a, b, p, s, grid_out);
    case 2: return launch_kind2<KIND, 2, DW>(a, b, p, s, grid_out);
    case 4: return launch_kind2<KIND, 4, DW>(a, b, p, s, grid_out);
    default: return launch_kind2<KIND, 8, DW>(a, b, p, s, grid_out);
  }
}

}  // namespace

int tc_max_grid() { return num_sms(); }

bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                        uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                        bool swizzle128) {
  return make_map(map, dt, base, inner, outer, row_bytes, box_inner, box_outer, swizzle128);
}

cudaError_t launch_tc_forward(const uint16_t* Xa, bool algebraic, const float* corr, int64_t M,
                              const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                              const float* A, const float* B, uint16_t* Y, unsigned int* err,
                              cudaStream_t s, int* launches) {
  // The algebraic form runs on single CTAs (its B tile is a full 256-row
  // block of codes); the decode form runs on CTA pairs (each CTA holds and
  // decodes 128 of those rows), where splitting the decode pays off.
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Xa, d_in, M, d_in * 2, BK, BM, true) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, d_in / 4, d_out, d_in / 4, BK / 4,
                algebraic ? BN : BN / 2, false))
    return cudaErrorInvalidValue;
  Params p{};
  p.M = M; p.N = d_out; p.K = d_in; p.d_in = d_in; p.d_out = d_out;
  p.codes = packed; p.corr = corr; p.Amat = A; p.Bvec = B; p.out = Y; p.err = err;
  cudaError_t e = algebraic ? launch_kind<kFwdAlg, 8, 4>(ta, tb, p, s, nullptr)
                            : launch_kind2_d<kFwdDec, 8>(d, ta, tb, p, s, nullptr);
  ++*launches;
  return e;
}

cudaError_t launch_tc_backward_dx(const uint16_t* dY, const float* rsum, int64_t M,
                                  const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                                  const float* A, const float* B, uint16_t* dX, unsigned int* err,
                                  cudaStream_t s, int* launches) {
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, d_out, M, d_out * 2, BK, BM, true) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, d_in / 4, d_out, d_in / 4, BN / 4, BK,
                false))
    return cudaErrorInvalidValue;
  Params p{};
  p.M = M; p.N = d_in; p.K = d_out; p.d_in = d_in; p.d_out = d_out;
  p.codes = packed; p.rsum = rsum; p.Amat = A; p.Bvec = B; p.out = dX; p.err = err;
  cudaError_t e = launch_kind_d<kDx, 4>(d, ta, tb, p, s, nullptr);
  ++*launches;
  return e;
}

cudaError_t launch_tc_gram(const uint16_t* Q, int64_t rows, int64_t cols_p, int64_t cols_q,
                           float* C, unsigned int* err, cudaStream_t s, int* launches) {
  // P is the first cols_p columns of Q (same rows and row pitch)
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, cols_p, rows, cols_q * 2, 64, BK, true) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, cols_q, rows, cols_q * 2, 64, BK, true))
    return cudaErrorInvalidValue;
  Params p{};
  p.M = cols_p; p.N = cols_q; p.K = rows; p.out = C; p.err = err;
  cudaError_t e = launch_kind<kGram, 8, 0>(ta, tb, p, s, nullptr);
  ++*launches;
  return e;
}

cudaError_t launch_tc_backward_dw(const uint16_t* X, const uint16_t* dY, int64_t M,
                                  const uint8_t* packed, const uint8_t* mask, int64_t d_out,
                                  int64_t d_in, int d, const float* A, float* dWp,
                                  float* partials, int* num_parts, unsigned int* err,
                                  cudaStream_t s, int* launches) {
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, d_out, M, d_out * 2, 64, BK, true) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, d_in, M, d_in * 2, 64, BK, true))
    return cudaErrorInvalidValue;
  Params p{};
  p.M = d_out; p.N = d_in; p.K = M; p.d_in = d_in; p.d_out = d_out;
  p.codes = packed; p.mask = mask; p.Amat = A; p.Bvec = A; p.out = dWp; p.partials = partials;
  p.err = err;
  cudaError_t e = launch_kind2_d<kDw, 0>(d, ta, tb, p, s, num_parts);
  ++*launches;
  return e;
}

}  // namespace lcvq

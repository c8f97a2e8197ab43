// H-aware sequential code assignment: the PTQ initialisation of the codes
// (LC-QAT technical summary, Methodology 2: the initial integer weights come
// from LDLQ, column-wise quantization with sequential compensation of the
// reconstruction error; decoupleQ page, section 3.3, eq. (8)-(11): round and
// clip one element, then re-solve the rest of the quadratic objective without
// the integer constraint and the box).
//
// For one weight row with code-space target p and code-space Hessian
// Q = (I + U) diag(D) (I + U)^T (U strictly upper triangular), element j is
//     z_j = clamp(rint(t_j), 0, 3),   t_j = p_j + sum_{i<j} U[i][j] (p_i - z_i).
// Rows are independent; within a row every t_j waits for all z_{i<j}.
//
// ldlq_kernel: one CTA per 32 rows (one CTA per SM), K in blocks of 64
// columns, three kinds of warps working one block apart:
//   * warps 0..7 form, for block b (columns j0 .. j0 + 63, j0 = 64 b), the
//     compensation from the earlier blocks, T_b = E_{<b} U[<j0, block]: a
//     32 x 64 x j0 product, split over the warps by k rows of every 64-row
//     chunk, fp32 FFMA with a lane tile of 8 rows x 8 columns (16 values
//     loaded per 64 FMAs, which balances the shared-memory and FMA pipes);
//     the 8 partial tiles are summed in warp order into T_b in shared memory;
//   * warp 8 rounds block b in order, one lane per row: t_j = p_j + c_j, z_j
//     by a clamp and the magic-number rounding (ties to even, on the FMA
//     pipe), e_j = p_j - z_j, and the later columns of the block take
//     U[j0 + j][j0 + k] e_j (the diagonal tile, read as warp-wide broadcasts).
//     It goes in sub-blocks of 8 columns: a sub-block first takes the errors
//     of the earlier sub-blocks as a small product, then runs in order, so
//     only 8 compensations are live.  Its errors go to shared memory, where
//     warps 0..7 take the newest chunk of T_{b+1} from, and to the workspace,
//     where the older chunks come from; it prefetches the next block's
//     targets with cp.async;
//   * warp 9 streams, through TMA, the 64 x 64 tiles U[64c .., j0 ..] with the
//     CTA's error chunks E[64c .., 32 rows] (a ring of stages) and the
//     diagonal tiles (two buffers).
// While warp 8 rounds block b, warps 0..7 already work on T_{b+1}: only its
// last chunk waits for block b's errors.  The work is N K (K - 1) / 2 fused
// multiply-adds, on the CUDA cores in fp32 (a code can differ from the fp64
// rule only within fp32 rounding of a rounding boundary).  Every wait is
// bounded; a warp that gives up records LCVQ_ERR_DEVICE_TIMEOUT, raises the
// CTA's abort flag, and the CTA winds down through the same barriers.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lcvq {

namespace {

constexpr int kLqRows = 32;                         // weight rows per CTA
constexpr int kLqBlk = 64;                          // columns per block = k rows per chunk
constexpr int kLqGemm = 8;                          // product warps
constexpr int kLqSeqWarp = kLqGemm;                 // the in-order warp
constexpr int kLqProdWarp = kLqGemm + 1;            // the TMA producer
constexpr int kLqThreads = (kLqGemm + 2) * 32;
constexpr int kLqStages = 3;
constexpr int kLqTPitch = kLqBlk + 4;               // padded rows: conflict-free row reads
constexpr uint32_t kLqUBytes = kLqBlk * kLqBlk * 4;          // 64 x 64 fp32 tile of U
constexpr uint32_t kLqEBytes = kLqBlk * kLqRows * 4;         // 64 k x 32 rows of errors
constexpr uint32_t kLqStageBytes = kLqUBytes + kLqEBytes;
constexpr uint32_t kLqDiagOff = kLqStages * kLqStageBytes;  // 2 diagonal tiles
constexpr uint32_t kLqRedOff = kLqDiagOff + 2 * kLqUBytes;  // [8 warps][32][64] partials
constexpr uint32_t kLqRedBytes = kLqGemm * kLqRows * kLqBlk * 4;
constexpr uint32_t kLqTOff = kLqRedOff + kLqRedBytes;       // T_b [32][68]
constexpr uint32_t kLqTBytes = kLqRows * kLqTPitch * 4;
constexpr uint32_t kLqEstOff = kLqTOff + kLqTBytes;         // newest errors [64][32]
constexpr uint32_t kLqPOff = kLqEstOff + kLqEBytes;         // targets, 2 x [32][68]
constexpr uint32_t kLqBarOff = kLqPOff + 2 * kLqTBytes;
constexpr int kLqNumBars = 2 * kLqStages + 4 + 4;           // full, empty, dfull x2, dempty x2,
                                                            // tready, eready, ebar x2
constexpr size_t kLqSmem = 128 + kLqBarOff + kLqNumBars * 8 + 16;
constexpr long long kLqWaitLimit = 1LL << 32;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x in [0, 3] to an integer
static_assert(kLqStageBytes % 128 == 0 && kLqDiagOff % 128 == 0, "TMA destinations stay aligned");
static_assert(kLqTBytes % 16 == 0 && kLqEstOff % 16 == 0 && kLqPOff % 16 == 0, "16-byte rows");
static_assert(kLqGemm * 32 * 8 == kLqRows * kLqBlk, "each product thread sums 8 outputs");
static_assert(kLqSmem <= 232448, "fits in one SM's shared memory");

struct LdlqParams {
  CUtensorMap u;        // U [K][K] fp32, box 64 x 64, no swizzle
  const float* P;       // [N][K] targets
  float* E;             // workspace [ceil(N/32)][K][32]: p - z per CTA, column-major in rows
  uint8_t* packed;      // [N][K/4]
  int64_t N, K;
  unsigned int* err;
};

__device__ __forceinline__ void gemm_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(kLqGemm * 32) : "memory");
}
// generic-proxy global writes -> visible to later bulk (async-proxy) reads
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

__global__ void __launch_bounds__(kLqThreads, 1) ldlq_kernel(const __grid_constant__ LdlqParams p) {
  extern __shared__ __align__(128) unsigned char lq_raw[];
  unsigned char* sm = lq_raw + ((128 - (sm100::smem_u32(lq_raw) & 127)) & 127);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kLqBarOff);
  uint64_t* empty = full + kLqStages;
  uint64_t* dfull = empty + kLqStages;
  uint64_t* dempty = dfull + 2;
  uint64_t* tready = dempty + 2;  // T_b in shared memory (phase b - 1)
  uint64_t* eready = tready + 1;  // block b's errors in shared memory (phase b)
  // block b's errors in the workspace: ebar[b & 1], phase b / 2 (one barrier per
  // parity of b, so that the producer, which waits for block b - 2, never finds
  // the barrier two phases ahead of the one it waits for)
  uint64_t* ebar = eready + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ebar + 2);
  float* diag = reinterpret_cast<float*>(sm + kLqDiagOff);
  float* red = reinterpret_cast<float*>(sm + kLqRedOff);
  float* tbuf = reinterpret_cast<float*>(sm + kLqTOff);
  float* est = reinterpret_cast<float*>(sm + kLqEstOff);
  float* pbuf = reinterpret_cast<float*>(sm + kLqPOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t K = p.K;
  const int nb = static_cast<int>(K / kLqBlk);
  const int64_t row0 = int64_t(blockIdx.x) * kLqRows;
  float* Ecta = p.E + int64_t(blockIdx.x) * K * kLqRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLqStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], kLqGemm);
    }
    for (int s = 0; s < 2; ++s) {
      sm100::mbar_init(&dfull[s], 1);
      sm100::mbar_init(&dempty[s], 1);
    }
    sm100::mbar_init(tready, kLqGemm * 32);
    sm100::mbar_init(eready, 32);
    sm100::mbar_init(&ebar[0], 32);
    sm100::mbar_init(&ebar[1], 32);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();

  // bounded wait; after a timeout anywhere in the CTA every later wait is skipped
  auto wait = [&](uint64_t* bar, uint32_t parity, unsigned site) {
    if (*abort_flag) return false;
    if (!sm100::mbar_wait(bar, parity, kLqWaitLimit)) {
      if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, site);
      *abort_flag = 1;
      return false;
    }
    return true;
  };

  if (warp == kLqProdWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) sm100::tma_prefetch_map(&p.u);
    int seq = 0, nd = 0;  // ring stages and diagonal tiles issued
    for (int b = 0; b < nb && !*abort_flag; ++b) {
      const int db = b & 1;
      if (!wait(&dempty[db], ((b >> 1) & 1) ^ 1, 70)) break;
      if (lane == 0) {
        sm100::mbar_arrive_expect_tx(&dfull[db], kLqUBytes);
        sm100::tma_load_2d(&p.u, &dfull[db], diag + db * (kLqBlk * kLqBlk), b * kLqBlk, b * kLqBlk);
      }
      __syncwarp();
      ++nd;
      for (int c = 0; c < b; ++c) {
        const int s = seq % kLqStages;
        if (!wait(&empty[s], ((seq / kLqStages) & 1) ^ 1, 71)) break;
        // chunk b - 1 of the errors is read from shared memory by the product
        // warps; the older ones come from the workspace, once stored
        const bool with_e = c + 1 < b;
        if (with_e && c == b - 2 && !wait(&ebar[b & 1], ((b - 2) >> 1) & 1, 72)) break;
        if (lane == 0) {
          unsigned char* st = sm + s * kLqStageBytes;
          sm100::mbar_arrive_expect_tx(&full[s], kLqUBytes + (with_e ? kLqEBytes : 0u));
          sm100::tma_load_2d(&p.u, &full[s], st, b * kLqBlk, c * kLqBlk);
          if (with_e)
            sm100::bulk_load(sm100::smem_u32(st + kLqUBytes), Ecta + int64_t(c) * kLqBlk * kLqRows,
                             kLqEBytes, &full[s]);
        }
        __syncwarp();
        ++seq;
      }
    }
    // no copy may outlive the CTA: wait until the last tiles issued have landed
    for (int q = seq > kLqStages ? seq - kLqStages : 0; q < seq; ++q)
      if (!sm100::mbar_wait(&full[q % kLqStages], (q / kLqStages) & 1, kLqWaitLimit)) {
        if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 73);
        break;
      }
    for (int q = nd > 2 ? nd - 2 : 0; q < nd; ++q)
      if (!sm100::mbar_wait(&dfull[q & 1], (q >> 1) & 1, kLqWaitLimit)) {
        if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 74);
        break;
      }
    return;
  }

  if (warp == kLqSeqWarp) {
    // ------------------------------------------------------------ in order, lane = row
    const int64_t grow = row0 + lane;
    const bool live = grow < p.N;
    const float* prow = p.P + (live ? grow : 0) * K;
    auto prefetch = [&](int b) {
      const uint32_t dst = sm100::smem_u32(pbuf + (b & 1) * (kLqRows * kLqTPitch) + lane * kLqTPitch);
#pragma unroll
      for (int m = 0; m < kLqBlk / 4; ++m) cp_async16(dst + 16 * m, prow + int64_t(b) * kLqBlk + 4 * m, live);
      cp_async_commit();
    };
    prefetch(0);
    for (int b = 0; b < nb; ++b) {
      const int64_t j0 = int64_t(b) * kLqBlk;
      cp_async_wait_all();
      __syncwarp();
      // the block's targets stay in shared memory (read 4 at a time below)
      const float4* pr = reinterpret_cast<const float4*>(pbuf + (b & 1) * (kLqRows * kLqTPitch) + lane * kLqTPitch);
      if (b + 1 < nb) prefetch(b + 1);  // into the other buffer
      if (b > 0) wait(tready, (b - 1) & 1, 75);
      const int db = b & 1;
      wait(&dfull[db], (b >> 1) & 1, 76);
      const float* dg = diag + db * (kLqBlk * kLqBlk);
      uint32_t code[4] = {0u, 0u, 0u, 0u};
      float* erow = Ecta + j0 * kLqRows + lane;
      // eight sub-blocks of 8 columns: sub-block q first takes the errors of
      // sub-blocks 0 .. q-1 as a small product (independent FMAs), then runs
      // its 8 columns in order; only 8 compensations are live at a time
      const float4* dg4 = reinterpret_cast<const float4*>(dg);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float cs[8];
        if (b > 0) {
          const float4 t0 = *reinterpret_cast<const float4*>(tbuf + lane * kLqTPitch + 8 * q);
          const float4 t1 = *reinterpret_cast<const float4*>(tbuf + lane * kLqTPitch + 8 * q + 4);
          cs[0] = t0.x, cs[1] = t0.y, cs[2] = t0.z, cs[3] = t0.w;
          cs[4] = t1.x, cs[5] = t1.y, cs[6] = t1.z, cs[7] = t1.w;
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) cs[k] = 0.f;
        }
#pragma unroll 4
        for (int j = 0; j < 8 * q; ++j) {
          const float e = est[j * kLqRows + lane];
          const float4 u0 = dg4[j * (kLqBlk / 4) + 2 * q];
          const float4 u1 = dg4[j * (kLqBlk / 4) + 2 * q + 1];
          cs[0] = fmaf(u0.x, e, cs[0]), cs[1] = fmaf(u0.y, e, cs[1]);
          cs[2] = fmaf(u0.z, e, cs[2]), cs[3] = fmaf(u0.w, e, cs[3]);
          cs[4] = fmaf(u1.x, e, cs[4]), cs[5] = fmaf(u1.y, e, cs[5]);
          cs[6] = fmaf(u1.z, e, cs[6]), cs[7] = fmaf(u1.w, e, cs[7]);
        }
        const float4 p0 = pr[2 * q], p1 = pr[2 * q + 1];
        const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = 8 * q + jj;
          const float xc = fminf(fmaxf(pv[jj] + cs[jj], 0.f), 3.f);  // NaN -> 0
          const float zb = __fadd_rn(xc, kRoundMagic);               // integer in the low bits
          const float e = pv[jj] - __fadd_rn(zb, -kRoundMagic);
          code[j >> 4] |= (__float_as_uint(zb) & 3u) << (2 * (j & 15));
          est[j * kLqRows + lane] = e;
          erow[j * kLqRows] = e;
          if (jj < 7) {  // only U[i][j] with i < j is read: the columns after j
            const float4 u0 = dg4[j * (kLqBlk / 4) + 2 * q];
            const float4 u1 = dg4[j * (kLqBlk / 4) + 2 * q + 1];
            const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int k = jj + 1; k < 8; ++k) cs[k] = fmaf(uv[k], e, cs[k]);
          }
        }
      }
      if (live)
        *reinterpret_cast<uint4*>(p.packed + grow * (K / 4) + j0 / 4) =
            make_uint4(code[0], code[1], code[2], code[3]);
      __syncwarp();
      sm100::mbar_arrive(eready);
      fence_async_global();
      sm100::mbar_arrive(&ebar[b & 1]);
      if (lane == 0) sm100::mbar_arrive(&dempty[db]);
    }
    cp_async_wait_all();
    return;
  }

  // ------------------------------------------------------------ product warps
  // lane tile 8 x 8: rows 8 rg .. 8 rg + 7, columns 4 cg .. 4 cg + 3 and
  // 32 + 4 cg .. 32 + 4 cg + 3, so that every quarter-warp reads 128 contiguous
  // bytes of U and one broadcast 16 bytes of E per shared-memory load
  const int rg = lane >> 3, cg = lane & 7;
  int seq = 0;  // ring stages consumed
  for (int b = 1; b < nb; ++b) {
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[i][q] = 0.f;
    for (int c = 0; c < b; ++c, ++seq) {
      const int s = seq % kLqStages;
      wait(&full[s], (seq / kLqStages) & 1, 77);
      const float* us = reinterpret_cast<const float*>(sm + s * kLqStageBytes);
      const float* es = us + kLqBlk * kLqBlk;
      if (c + 1 == b) {  // the newest errors: block b - 1, straight from the in-order warp
        wait(eready, (b - 1) & 1, 78);
        es = est;
      }
      // operands of k row r + 1 are loaded before the FMAs of row r
      const float* ep = es + (8 * warp) * kLqRows + 8 * rg;
      const float* upp = us + (8 * warp) * kLqBlk + 4 * cg;
      float4 e0 = *reinterpret_cast<const float4*>(ep);
      float4 e1 = *reinterpret_cast<const float4*>(ep + 4);
      float4 u0 = *reinterpret_cast<const float4*>(upp);
      float4 u1 = *reinterpret_cast<const float4*>(upp + 32);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
        const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        if (r + 1 < 8) {
          e0 = *reinterpret_cast<const float4*>(ep + (r + 1) * kLqRows);
          e1 = *reinterpret_cast<const float4*>(ep + (r + 1) * kLqRows + 4);
          u0 = *reinterpret_cast<const float4*>(upp + (r + 1) * kLqBlk);
          u1 = *reinterpret_cast<const float4*>(upp + (r + 1) * kLqBlk + 32);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[i][q] = fmaf(ev[i], uv[q], acc[i][q]);
      }
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&empty[s]);
    }
    float* rw = red + warp * (kLqRows * kLqBlk);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float* dst = rw + (8 * rg + i) * kLqBlk + 4 * cg;
      *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      *reinterpret_cast<float4*>(dst + 32) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
    gemm_sync();
    {
      // thread i sums row i / 8, columns 4 (i % 8) .. + 3 and 32 + 4 (i % 8) .. + 3
      const int row = threadIdx.x >> 3, c4 = 4 * (threadIdx.x & 7);
      float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
#pragma unroll
      for (int w = 0; w < kLqGemm; ++w) {
        const float4 a = *reinterpret_cast<const float4*>(red + w * (kLqRows * kLqBlk) + row * kLqBlk + c4);
        const float4 b4 = *reinterpret_cast<const float4*>(red + w * (kLqRows * kLqBlk) + row * kLqBlk + 32 + c4);
        s0.x += a.x, s0.y += a.y, s0.z += a.z, s0.w += a.w;
        s1.x += b4.x, s1.y += b4.y, s1.z += b4.z, s1.w += b4.w;
      }
      *reinterpret_cast<float4*>(tbuf + row * kLqTPitch + c4) = s0;
      *reinterpret_cast<float4*>(tbuf + row * kLqTPitch + 32 + c4) = s1;
    }
    gemm_sync();  // the partials are read before the next block writes them
    sm100::mbar_arrive(tready);
  }
}

}  // namespace

size_t ldlq_workspace_bytes(int64_t d_out, int64_t d_in) {
  return size_t(ceil_div(d_out, kLqRows)) * kLqRows * size_t(d_in) * 4;
}

cudaError_t launch_ldlq(const float* P, const float* U, int64_t d_out, int64_t d_in,
                        uint8_t* packed, float* E, unsigned int* err, cudaStream_t s,
                        int* launches) {
  *launches = 0;
  if (d_out == 0 || d_in == 0) return cudaSuccess;
  LdlqParams prm{};
  if (!make_tensor_map_2d(&prm.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, U, uint64_t(d_in),
                          uint64_t(d_in), uint64_t(d_in) * 4, kLqBlk, kLqBlk, false))
    return cudaErrorInvalidValue;
  prm.P = P;
  prm.E = E;
  prm.packed = packed;
  prm.N = d_out;
  prm.K = d_in;
  prm.err = err;
  auto kern = ldlq_kernel;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), kLqSmem);
      e != cudaSuccess)
    return e;
  const int64_t grid = ceil_div(d_out, kLqRows);
  kern<<<static_cast<unsigned int>(grid), kLqThreads, kLqSmem, s>>>(prm);
  *launches = 1;
  return cudaGetLastError();
}

}  // namespace lcvq

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
// columns.  For block b (columns j0 .. j0 + 63, j0 = 64 b):
//   1. the part of t from the earlier blocks, T_b = E_{<b} U[<j0, block], is
//      a 32 x 64 x j0 product: warp 8 streams the chunks c < b, each the
//      64 x 64 tile U[64c .., j0 ..] (TMA box) and the CTA's own errors
//      E[64c .., 32 rows] (one 8 KB bulk copy from the workspace, written at
//      the end of block c), through a ring of shared-memory stages; consumer
//      warp w takes k rows 8w .. 8w + 7 of every chunk and all 32 x 64
//      outputs (fp32 FFMA, lane tile 8 rows x 8 columns: 16 values loaded
//      per 64 FMAs, which balances the shared-memory and FMA pipes), and the
//      8 warps' partial tiles are summed in warp order through shared memory;
//   2. the block itself runs in order: warp w takes rows 4w .. 4w + 3, lane l
//      holds t of columns l and l + 32; at step j the owner lane rounds,
//      the error p_j - z_j is broadcast by a shuffle and every later column
//      adds U[j0 + j][col] times it (the diagonal tile, one more stage);
//   3. codes go out 16 bytes per row, the errors to the workspace (8 KB), and
//      an mbarrier tells the producer that chunk b may now be loaded.
// The work is N K (K - 1) / 2 fused multiply-adds, on the CUDA cores in fp32
// (the codes must follow the fp64 rule except within fp32 rounding of a
// rounding boundary).  Every wait is bounded; a warp that gives up records
// LCVQ_ERR_DEVICE_TIMEOUT and the CTA winds down through the same barriers.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lcvq {

namespace {

constexpr int kLqRows = 32;                         // weight rows per CTA
constexpr int kLqBlk = 64;                          // columns per block = k rows per chunk
constexpr int kLqCons = 8;                          // consumer warps
constexpr int kLqSeqRows = kLqRows / kLqCons;       // rows per warp in the in-order part
constexpr int kLqThreads = (kLqCons + 1) * 32;      // + one producer warp
constexpr int kLqStages = 4;
constexpr uint32_t kLqUBytes = kLqBlk * kLqBlk * 4;          // 64 x 64 fp32 tile of U
constexpr uint32_t kLqEBytes = kLqBlk * kLqRows * 4;         // 64 k x 32 rows of errors
constexpr uint32_t kLqStageBytes = kLqUBytes + kLqEBytes;
constexpr uint32_t kLqRedOff = kLqStages * kLqStageBytes;   // [8 warps][32][64] partials
constexpr uint32_t kLqRedBytes = kLqCons * kLqRows * kLqBlk * 4;
constexpr uint32_t kLqEstOff = kLqRedOff + kLqRedBytes;     // [64][32] errors of the block
constexpr uint32_t kLqZOff = kLqEstOff + kLqEBytes;         // [32][16] code bytes of the block
constexpr uint32_t kLqBarOff = kLqZOff + kLqRows * 16;
constexpr size_t kLqSmem = 128 + kLqBarOff + (2 * kLqStages + 1) * 8 + 16;
constexpr long long kLqWaitLimit = 1LL << 32;
static_assert(kLqStageBytes % 128 == 0, "TMA destinations stay 128-byte aligned");
static_assert(kLqEBytes / 16 == 2 * kLqCons * 32, "two float4 of a chunk of errors per consumer thread");
static_assert(kLqSeqRows == 4, "the in-order part stages its errors as one float4 per column");

struct LdlqParams {
  CUtensorMap u;        // U [K][K] fp32, box 64 x 64, no swizzle
  const float* P;       // [N][K] targets
  float* E;             // workspace [ceil(N/32)][K][32]: p - z per CTA, column-major in rows
  uint8_t* packed;      // [N][K/4]
  int64_t N, K;
  unsigned int* err;
};

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(kLqCons * 32) : "memory");
}
// generic-proxy global writes -> visible to later bulk (async-proxy) reads
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}

__global__ void __launch_bounds__(kLqThreads, 1) ldlq_kernel(const __grid_constant__ LdlqParams p) {
  extern __shared__ __align__(128) unsigned char lq_raw[];
  unsigned char* sm = lq_raw + ((128 - (sm100::smem_u32(lq_raw) & 127)) & 127);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kLqBarOff);
  uint64_t* empty = full + kLqStages;
  uint64_t* ebar = empty + kLqStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ebar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t K = p.K;
  const int nb = static_cast<int>(K / kLqBlk);
  const int64_t row0 = int64_t(blockIdx.x) * kLqRows;
  float* Ecta = p.E + int64_t(blockIdx.x) * K * kLqRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLqStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], kLqCons);
    }
    sm100::mbar_init(ebar, kLqCons * 32);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kLqCons) {
    // ------------------------------------------------------------ producer
    if (lane == 0) sm100::tma_prefetch_map(&p.u);
    int seq = 0;  // stages issued
    for (int b = 0; b < nb && !*abort_flag; ++b) {
      for (int c = 0; c <= b; ++c) {
        const int s = seq % kLqStages;
        if (!sm100::mbar_wait(&empty[s], ((seq / kLqStages) & 1) ^ 1, kLqWaitLimit)) {
          if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 70);
          *abort_flag = 1;
          break;
        }
        // the newest chunk of errors exists once block b - 1 has been stored
        if (c == b - 1 && !sm100::mbar_wait(ebar, (b - 1) & 1, kLqWaitLimit)) {
          if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 71);
          *abort_flag = 1;
          break;
        }
        if (lane == 0) {
          unsigned char* st = sm + s * kLqStageBytes;
          const bool diag = c == b;
          sm100::mbar_arrive_expect_tx(&full[s], kLqUBytes + (diag ? 0u : kLqEBytes));
          sm100::tma_load_2d(&p.u, &full[s], st, b * kLqBlk, c * kLqBlk);
          if (!diag)
            sm100::bulk_load(sm100::smem_u32(st + kLqUBytes), Ecta + int64_t(c) * kLqBlk * kLqRows,
                             kLqEBytes, &full[s]);
        }
        __syncwarp();
        ++seq;
      }
    }
    // no copy may outlive the CTA: wait until the last stages issued have landed
    for (int q = seq > kLqStages ? seq - kLqStages : 0; q < seq; ++q) {
      if (!sm100::mbar_wait(&full[q % kLqStages], (q / kLqStages) & 1, kLqWaitLimit)) {
        if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 72);
        break;
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  // product lane tile 8 x 8: rows 8 rg .. 8 rg + 7, columns 4 cg .. 4 cg + 3 and
  // 32 + 4 cg .. 32 + 4 cg + 3, so that every quarter-warp reads 128 contiguous
  // bytes of U and one broadcast 16 bytes of E per shared-memory load
  const int rg = lane >> 3, cg = lane & 7;
  const int sr = kLqSeqRows * warp;  // rows of the in-order part: sr .. sr + 3
  float* red = reinterpret_cast<float*>(sm + kLqRedOff);
  float* est = reinterpret_cast<float*>(sm + kLqEstOff);
  uint8_t* zst = sm + kLqZOff;
  int seq = 0;  // stages consumed
  for (int b = 0; b < nb; ++b) {
    const int64_t j0 = int64_t(b) * kLqBlk;
    float pv[kLqSeqRows][2];
#pragma unroll
    for (int r = 0; r < kLqSeqRows; ++r) {
      const int64_t gr = row0 + sr + r;
#pragma unroll
      for (int h = 0; h < 2; ++h) pv[r][h] = gr < p.N ? __ldg(p.P + gr * K + j0 + lane + 32 * h) : 0.f;
    }

    // 1. T_b = E_{<b} U[<j0, block]: this warp's k rows of every chunk
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[i][q] = 0.f;
    for (int c = 0; c < b; ++c, ++seq) {
      const int s = seq % kLqStages;
      if (!*abort_flag && !sm100::mbar_wait(&full[s], (seq / kLqStages) & 1, kLqWaitLimit)) {
        if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 73);
        *abort_flag = 1;
      }
      const float* us = reinterpret_cast<const float*>(sm + s * kLqStageBytes);
      const float* es = us + kLqBlk * kLqBlk;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int k = 8 * warp + r;
        const float4 e0 = *reinterpret_cast<const float4*>(es + k * kLqRows + 8 * rg);
        const float4 e1 = *reinterpret_cast<const float4*>(es + k * kLqRows + 8 * rg + 4);
        const float4 u0 = *reinterpret_cast<const float4*>(us + k * kLqBlk + 4 * cg);
        const float4 u1 = *reinterpret_cast<const float4*>(us + k * kLqBlk + 32 + 4 * cg);
        const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
        const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[i][q] = fmaf(ev[i], uv[q], acc[i][q]);
      }
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&empty[s]);
    }
    if (b > 0) {
      float* rw = red + warp * (kLqRows * kLqBlk);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float* dst = rw + (8 * rg + i) * kLqBlk + 4 * cg;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        *reinterpret_cast<float4*>(dst + 32) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
      }
    }
    consumers_sync();
    float t[kLqSeqRows][2];
#pragma unroll
    for (int r = 0; r < kLqSeqRows; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float sum = 0.f;
        if (b > 0) {
#pragma unroll
          for (int w = 0; w < kLqCons; ++w) sum += red[w * (kLqRows * kLqBlk) + (sr + r) * kLqBlk + lane + 32 * h];
        }
        t[r][h] = pv[r][h] + sum;
      }

    // 2. the block in order, with the diagonal tile U[j0 .., j0 ..]
    float eo[kLqSeqRows][2];
    uint32_t zo[kLqSeqRows][2];
#pragma unroll
    for (int r = 0; r < kLqSeqRows; ++r) eo[r][0] = eo[r][1] = 0.f, zo[r][0] = zo[r][1] = 0u;
    {
      const int s = seq % kLqStages;
      if (!*abort_flag && !sm100::mbar_wait(&full[s], (seq / kLqStages) & 1, kLqWaitLimit)) {
        if (lane == 0) record_error(p.err, LCVQ_ERR_DEVICE_TIMEOUT, 74);
        *abort_flag = 1;
      }
      const float* dg = reinterpret_cast<const float*>(sm + s * kLqStageBytes);
      // columns 0 .. 31 of the block (held in t[.][0]), then 32 .. 63 (t[.][1])
#pragma unroll 2
      for (int j = 0; j < 32; ++j) {
        const float u0 = dg[j * kLqBlk + lane];
        const float u1 = dg[j * kLqBlk + lane + 32];
#pragma unroll
        for (int r = 0; r < kLqSeqRows; ++r) {
          const float z = fminf(fmaxf(rintf(t[r][0]), 0.f), 3.f);  // NaN -> 0
          const float e = __shfl_sync(0xffffffffu, pv[r][0] - z, j);
          if (lane == j) {
            eo[r][0] = e;
            zo[r][0] = static_cast<uint32_t>(z);
          }
          // only U[i][j] with i < j is read: the columns after j
          if (lane > j) t[r][0] = fmaf(u0, e, t[r][0]);
          t[r][1] = fmaf(u1, e, t[r][1]);
        }
      }
#pragma unroll 2
      for (int j = 0; j < 32; ++j) {
        const float u1 = dg[(32 + j) * kLqBlk + lane + 32];
#pragma unroll
        for (int r = 0; r < kLqSeqRows; ++r) {
          const float z = fminf(fmaxf(rintf(t[r][1]), 0.f), 3.f);
          const float e = __shfl_sync(0xffffffffu, pv[r][1] - z, j);
          if (lane == j) {
            eo[r][1] = e;
            zo[r][1] = static_cast<uint32_t>(z);
          }
          if (lane > j) t[r][1] = fmaf(u1, e, t[r][1]);
        }
      }
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&empty[s]);
      ++seq;
    }

    // 3. stage the block's errors and codes, then store them
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = lane + 32 * h;
      *reinterpret_cast<float4*>(est + col * kLqRows + sr) =
          make_float4(eo[0][h], eo[1][h], eo[2][h], eo[3][h]);
#pragma unroll
      for (int r = 0; r < kLqSeqRows; ++r) {
        uint32_t v = zo[r][h] << (2 * (lane & 3));
        v |= __shfl_xor_sync(0xffffffffu, v, 1);
        v |= __shfl_xor_sync(0xffffffffu, v, 2);
        if ((lane & 3) == 0) zst[(sr + r) * 16 + (col >> 2)] = static_cast<uint8_t>(v);
      }
    }
    consumers_sync();
    const int tid = threadIdx.x;  // 0 .. 255
    float4* edst = reinterpret_cast<float4*>(Ecta + j0 * kLqRows);
    edst[tid] = reinterpret_cast<const float4*>(est)[tid];
    edst[tid + kLqCons * 32] = reinterpret_cast<const float4*>(est)[tid + kLqCons * 32];
    if (tid < kLqRows && row0 + tid < p.N)
      *reinterpret_cast<uint4*>(p.packed + (row0 + tid) * (K / 4) + j0 / 4) =
          reinterpret_cast<const uint4*>(zst)[tid];
    fence_async_global();
    sm100::mbar_arrive(ebar);
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

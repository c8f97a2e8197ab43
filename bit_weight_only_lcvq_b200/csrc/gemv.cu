// Decode-GEMV for few tokens (M <= 32): Y = X W~ with W~ = A z + B streamed as
// packed 2-bit codes (LC-QAT technical summary, Methodology 3: the forward runs
// on INT2 x FP16 matmul operators), one matrix or a group of matrices.
//
// Both kernels here multiply the transformed activations X'' (see xform.cu)
// with the raw codes on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate):
//   * weights are the 16-row A operand, tokens the 8-column B operand, so a
//     weight tile is decoded once and serves every token;
//   * codes are decoded in registers by a single LOP3 per bf16 pair:
//     (word >> s) & 0x00030003 << 2p | 0x43004300 = bf16x2(128 + 4^p z_lo,
//     128 + 4^p z_hi); the power of two and the 128 offset are folded into X''
//     and the per-row constant `corr`, so decoding costs no float arithmetic;
//   * the MMA's logical k of each lane is mapped onto the lane's own code
//     words (the decoder order of X'' makes the B fragments contiguous loads);
//   * K is cut into chunks of 512 codes; warp w of 8 sums chunks w, w + 8, ...
//     and the 8 partial sums are added in warp order, so every path gives the
//     same bits for a matrix;
//   * programmatic dependent launch: launched right after the X-transform of
//     the same call (early_codes), the split-K kernel issues its code loads
//     before griddepcontrol.wait, so they stream while the transform runs.
//     The X-transform lets it launch only after its own wait has returned, so
//     every kernel that could have written the codes has completed; it touches
//     nothing else before the wait.  Launched on its own (lcvq_gemm_xformed)
//     it waits first.
// gemv_group_kernel (split K, cp.async code rings) serves single matrices and
// small groups; gemv_wide_kernel (128-row tiles, TMA producer warp) serves
// large groups; gemv_tc.cu holds the tcgen05 form for 17..32 tokens.

#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include "codec.cuh"
#include "common.cuh"
#include "gemv_common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lcvq {

namespace {

// ---------------------------------------------------------------------------
// Decode-GEMV over a group of matrices in one persistent launch.
//
// Every matrix of the group is cut into tiles of 16 R weight rows over its
// whole K; tiles are numbered matrix by matrix, and CTA c takes tiles c, c + G,
// c + 2G, ...  (G = grid), so all CTAs sweep the matrices in order and the X''
// of the matrices in flight stays in L2.  Inside a tile, K is cut into chunks
// of kAhead units (kAhead * 128 codes); warp w takes chunks w, w + W, ... .
// The warp's code ring holds one chunk: as it consumes unit j of a chunk it
// loads unit j of its next chunk, which may belong to its next tile, so the
// code stream does not stop at tile boundaries.  Each tile ends with the same
// fixed-order shared-memory sum as a single-matrix launch (double-buffered,
// one barrier per tile); a group of one matrix is exactly the single-matrix
// decode-GEMV.
struct GemvItem {
  const uint8_t* packed;  // [N][K/4]
  const uint16_t* Xpp;    // [M][K] X'' (decoder order), or the int8 digit planes
  const float* corr;      // [M]
  uint16_t* Y;            // [M][N]
  int N, K;
  int tile_end;         // tiles of items 0 .. this one
  const float* inv_s;   // [M]: the int8 path's 1 / scale (null on the bf16 path)
};
template <int kItems>
struct GemvGroup {
  int count, M;
  int early_codes;  // launched right after this call's X-transform: codes may load before the wait
  GemvItem item[kItems];
};

// Code ring in shared memory, per warp: kStages chunks, each ROWS rows x 128 B
// (kAhead units of 32 B per row).  A chunk's 16-byte pieces are copied with
// cp.async by the warp's lanes (8 lanes per row, coalesced), XOR-swizzled by
// (row & 7) so that the lanes' 8-byte reads of one unit spread over the banks.
// Copies in flight hold no registers, so every SM keeps kStages - 1 chunks per
// warp on the way from HBM.
template <int R, int kStages, int kWarps>
__host__ __device__ constexpr size_t group_smem_ring() {
  return size_t(kWarps) * kStages * (16 * R) * 128;
}
template <int NT, int R, int kWarps>
__host__ __device__ constexpr size_t group_smem_part() {
  return size_t(2) * kWarps * (16 * R) * (NT * 8 + 1) * sizeof(float);
}

// kI8: the int8 path (X as the two digit planes of the int8-digit transform,
// u8 x s8 m16n8k32 MMAs accumulating exactly in int32): column c of a token
// tile is token 4 n + c / 2, digit plane c % 2 (hi, lo); otherwise column c is
// token 8 n + c of the bf16 X''.
template <int NT, int R, int kWarps, bool kPrefX, int kMinBlocks, int kStages, int kItems,
          bool kI8 = false>
__global__ void __launch_bounds__(kWarps * 32, kMinBlocks)
    gemv_group_kernel(const __grid_constant__ GemvGroup<kItems> grp) {
  using Acc = typename std::conditional<kI8, int, float>::type;
  constexpr int MP = NT * 8;
  constexpr int ROWS = 16 * R;
  constexpr uint32_t kStageBytes = ROWS * 128;
  static_assert(kStages >= 2, "ring of at least two chunks");
  // dynamic shared memory: [kWarps][kStages][ROWS][128 B] code ring, then
  // [2][kWarps][ROWS][MP + 1] fp32 partial tiles
  extern __shared__ __align__(128) unsigned char gsm[];
  auto part = reinterpret_cast<float(*)[kWarps][ROWS][MP + 1]>(
      gsm + group_smem_ring<R, kStages, kWarps>());

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = grp.M;
  const int T = grp.item[grp.count - 1].tile_end;
  const int G = static_cast<int>(gridDim.x);
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(gsm)) +
                        static_cast<uint32_t>(warp) * kStages * kStageBytes;

  struct Cur {
    int tile, item, chunk;
  };
  auto seek = [&](Cur c) {
    while (c.tile < T) {
      while (c.tile >= grp.item[c.item].tile_end) ++c.item;
      const int nch = static_cast<int>(ceil_div(ceil_div(grp.item[c.item].K, kUnit), kAhead));
      if (c.chunk < nch) return c;
      c.tile += G;
      c.chunk = warp;
    }
    return c;
  };
  auto advance = [&](Cur c) {
    c.chunk += kWarps;
    return seek(c);
  };
  auto tile_begin = [&](int item) { return item == 0 ? 0 : grp.item[item - 1].tile_end; };

  // copy chunk c into stage s (zero-filled outside the matrix; no copy at all
  // past the last tile); always one commit group
  auto issue = [&](const Cur& c, int s) {
    if (c.tile < T) {
      const GemvItem& it = grp.item[c.item];
      const int64_t row0 = int64_t(c.tile - tile_begin(c.item)) * ROWS;
      const int64_t Kb = it.K / 4;
      const int64_t cb = int64_t(c.chunk) * (kAhead * 32);  // chunk's first byte in a row
#pragma unroll
      for (int i = 0; i < ROWS / 4; ++i) {
        const int p = lane + 32 * i;
        const int row = p >> 3, c16 = p & 7;
        const int64_t grow = row0 + row;
        const int64_t col = cb + 16 * c16;
        const bool ok = grow < it.N && col < Kb;
        const uint8_t* src = ok ? it.packed + grow * Kb + col : it.packed;
        cp_async16_zfill(ring + s * kStageBytes + row * 128 + ((c16 ^ (row & 7)) << 4), src, ok);
      }
    }
    cp_async_commit();
  };
  // X'' fragments of unit j of chunk c: word q, token tile n -> two 16-byte halves
  // X of a chunk for this lane: the byte address of its first position in the
  // row (bf16: 32 positions of X''; int8: 32 positions of its digit plane) of
  // each token tile, and how many positions of K remain from there (<= 0: none)
  struct XPos {
    const unsigned char* base[NT];
    int remt;
  };
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) tokok[n] = (kI8 ? n * 4 + (g >> 1) : n * 8 + g) < M;
  auto xpos = [&](const Cur& c) {
    XPos p;
    const bool any = c.tile < T;
    const GemvItem& it = grp.item[any ? c.item : 0];
    const int64_t k0 = int64_t(c.chunk) * (kAhead * kUnit);
    p.remt = any ? static_cast<int>(it.K - k0) - 32 * t : 0;
    const unsigned char* xb = reinterpret_cast<const unsigned char*>(it.Xpp);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      if constexpr (kI8) {
        // chunk c's hi plane at byte 2 k0 of the row, its lo plane n_c bytes on
        const int64_t nc = it.K - k0 < kAhead * kUnit ? it.K - k0 : kAhead * kUnit;
        p.base[n] = xb + (tokok[n] ? int64_t(n * 4 + (g >> 1)) * 2 * it.K : 0) + 2 * k0 +
                    ((g & 1) ? nc : 0) + 32 * t;
      } else {
        p.base[n] = xb + 2 * ((tokok[n] ? int64_t(n * 8 + g) * it.K : 0) + k0 + 32 * t);
      }
    }
    return p;
  };
  // X fragments of unit j: word q, token tile n -> two 16-byte halves (bf16)
  // or one 16-byte block of digits (int8)
  auto load_x = [&](const XPos& p, int j, uint4 (&xb)[2][NT][2]) {
    const bool kok = j * kUnit < p.remt;
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        // written by the X-transform: ordinary loads, not the read-only path
        if (kok && tokok[n]) {
          if constexpr (kI8) {
            xb[q][n][0] = ld_global_v4(p.base[n] + j * kUnit + 16 * q);
            xb[q][n][1] = make_uint4(0, 0, 0, 0);
          } else {
            const unsigned char* src = p.base[n] + 2 * (j * kUnit + 16 * q);
            xb[q][n][0] = ld_global_v4(src);
            xb[q][n][1] = ld_global_v4(src + 16);
          }
        } else {
          xb[q][n][0] = make_uint4(0, 0, 0, 0);
          xb[q][n][1] = make_uint4(0, 0, 0, 0);
        }
      }
  };
  // this lane's code bytes of unit j in a stage row (SW128: chunk ^ (row & 7))
  uint32_t coff[kAhead];
#pragma unroll
  for (int j = 0; j < kAhead; ++j)
    coff[j] = static_cast<uint32_t>((((2 * j + (t >> 1)) ^ g) << 4) + ((t & 1) << 3));

  // prologue: the first kStages - 1 chunks (codes only), before the wait
  // when the X-transform of this call precedes the kernel
  if (!grp.early_codes) griddep_wait();
  Cur cur = seek(Cur{static_cast<int>(blockIdx.x), 0, warp});
  Cur iss = cur;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    issue(iss, s);
    iss = advance(iss);
  }
  Cur nxt = advance(cur);

  if (grp.early_codes) griddep_wait();  // X'' and corr of the X-transform are visible from here

  XPos pcur = xpos(cur), pnxt = xpos(nxt);
  uint4 xcur[2][NT][2], xnxt[2][NT][2];
  load_x(pcur, 0, xcur);

  int stage = 0;  // stage of cur
  int eitem = 0;  // item of the tile in the epilogue
  int buf = 0;
  for (int tile = static_cast<int>(blockIdx.x); tile < T; tile += G, buf ^= 1) {
    Acc acc[R][NT][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][n][e] = Acc(0);

    while (cur.tile == tile) {  // this warp's chunks of the tile
      cp_async_wait<kStages - 2>();  // this lane's copies of chunk `cur` have landed
      __syncwarp();                  // ... and every lane's; the stage refilled below is free
      {
        int s_iss = stage + kStages - 1;
        if (s_iss >= kStages) s_iss -= kStages;
        issue(iss, s_iss);
        iss = advance(iss);
      }
      const int rem = pcur.remt + 32 * t;  // positions of K left from this chunk on
      const uint32_t sbase = ring + stage * kStageBytes;
#pragma unroll
      for (int j = 0; j < kAhead; ++j) {
        if constexpr (kPrefX) {
          if (j + 1 < kAhead) load_x(pcur, j + 1, xnxt);
          else load_x(pnxt, 0, xnxt);
        }
        if (j * kUnit < rem) {  // warp-uniform
          // this lane's two code words of unit j for rows r*16 + g + 8h
          uint2 cw[R][2];
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              cw[r][h] = lds_v2(sbase + (r * 16 + g + 8 * h) * 128 + coff[j]);
          if constexpr (kI8) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {  // word q of each row: 16 codes, 2 k32 tiles
              uint32_t rp[R][2][4];
#pragma unroll
              for (int r = 0; r < R; ++r)
#pragma unroll
                for (int h = 0; h < 2; ++h) dec_word_u8(q == 0 ? cw[r][h].x : cw[r][h].y, rp[r][h]);
#pragma unroll
              for (int mm = 0; mm < 2; ++mm)
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                  const uint32_t b0 = word_of(xcur[q][n][0], 2 * mm);
                  const uint32_t b1 = word_of(xcur[q][n][0], 2 * mm + 1);
#pragma unroll
                  for (int r = 0; r < R; ++r)
                    mma_u8s8_16832(acc[r][n], rp[r][0][2 * mm], rp[r][1][2 * mm],
                                   rp[r][0][2 * mm + 1], rp[r][1][2 * mm + 1], b0, b1);
                }
            }
          } else {
#pragma unroll
          for (int q = 0; q < 2; ++q) {  // word q of each row: 16 codes, 4 k16 tiles
            uint32_t w0[R][2], w6[R][2], w12[R][2];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                w0[r][h] = q == 0 ? cw[r][h].x : cw[r][h].y;
                w6[r][h] = w0[r][h] >> 6;
                w12[r][h] = w0[r][h] >> 12;
              }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              uint32_t a[R][2][2];
#pragma unroll
              for (int r = 0; r < R; ++r)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  a[r][h][0] = dec_pair_rt(2 * jj, w0[r][h], w6[r][h], w12[r][h]);
                  a[r][h][1] = dec_pair_rt(2 * jj + 1, w0[r][h], w6[r][h], w12[r][h]);
                }
#pragma unroll
              for (int n = 0; n < NT; ++n) {
                const uint32_t b0 = word_of(xcur[q][n][jj >> 1], (2 * jj) & 3);
                const uint32_t b1 = word_of(xcur[q][n][jj >> 1], (2 * jj + 1) & 3);
#pragma unroll
                for (int r = 0; r < R; ++r)
                  mma_bf16_16816(acc[r][n], a[r][0][0], a[r][1][0], a[r][0][1], a[r][1][1], b0,
                                 b1);
              }
            }
          }
          }
        }
        if constexpr (kPrefX) {
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              xcur[q][n][0] = xnxt[q][n][0];
              xcur[q][n][1] = xnxt[q][n][1];
            }
        } else {
          if (j + 1 < kAhead) load_x(pcur, j + 1, xcur);
          else load_x(pnxt, 0, xcur);
        }
      }
      cur = nxt;
      pcur = pnxt;
      nxt = advance(nxt);
      pnxt = xpos(nxt);
      if (++stage == kStages) stage = 0;
    }

    // the CTA's last tile: the next kernel may start launching
    if (tile + G >= T) griddep_launch_dependents();

#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int lr = r * 16 + g;
        const int tk = n * 8 + 2 * t;  // int8: token 4 n + t, digit planes hi / lo
        if constexpr (kI8) {
          part[buf][warp][lr][tk] = __int_as_float(acc[r][n][0]);
          part[buf][warp][lr][tk + 1] = __int_as_float(acc[r][n][1]);
          part[buf][warp][lr + 8][tk] = __int_as_float(acc[r][n][2]);
          part[buf][warp][lr + 8][tk + 1] = __int_as_float(acc[r][n][3]);
        } else {
          part[buf][warp][lr][tk] = acc[r][n][0];
          part[buf][warp][lr][tk + 1] = acc[r][n][1];
          part[buf][warp][lr + 8][tk] = acc[r][n][2];
          part[buf][warp][lr + 8][tk + 1] = acc[r][n][3];
        }
      }
    __syncthreads();
    while (tile >= grp.item[eitem].tile_end) ++eitem;
    const GemvItem& it = grp.item[eitem];
    const int64_t row0 = int64_t(tile - tile_begin(eitem)) * ROWS;
    // sum the warps' K chunks in warp order, add the per-row constant, store
    // (int8: each class's exact integer sums scaled by its own 1 / s)
    for (int e = threadIdx.x; e < ROWS * M; e += kWarps * 32) {
      const int lr = e % ROWS, tok = e / ROWS;
      const int64_t grow = row0 + lr;
      float y;
      if constexpr (kI8) {  // warp w's chunks are class w: its own scale
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
          sum = i8_add_class(sum, __float_as_int(part[buf][w][lr][2 * tok]),
                             __float_as_int(part[buf][w][lr][2 * tok + 1]),
                             ld_global_f32(it.inv_s + tok * kWarps + w));
        y = sum + ld_global_f32(it.corr + tok);
      } else {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum += part[buf][w][lr][tok];
        y = sum + ld_global_f32(it.corr + tok);
      }
      if (grow < it.N) it.Y[int64_t(tok) * it.N + grow] = f32_to_bf16(y);
    }
  }
  cp_async_wait<0>();  // no copy may outlive the CTA (only empty groups remain)
}

// ---------------------------------------------------------------------------
// Decode-GEMV over a large group: wide tiles, one producer warp.
//
// A tile is 128 weight rows of one matrix over its whole K; consumer warp w
// (w < 8) owns rows 16 w .. 16 w + 15 of it and runs the whole K, so no tile
// ends in a CTA-wide sum.  Warp 8 produces: it streams the tile's K chunks
// (kAhead units = 512 codes per row: one 128-row x 128-byte TMA box with the
// 128-byte swizzle; and the matching 512 positions of X'' for every token, one
// 1D bulk copy per token) into a ring of kStages shared-memory stages, each
// stage's arrival counted on its `full` mbarrier; the consumers
// release a stage on its `empty` mbarrier.  X'' is thus read once per 128 rows
// instead of once per 16.
//
// Same sums as the split kernel, bit for bit: chunk c of a tile is the split
// kernel's chunk of warp c mod 8, so a consumer keeps 8 accumulators, adds
// chunk c into accumulator c mod 8 in the same unit and MMA order, and ends
// with the split kernel's fixed-order sum over the 8 accumulators.
//
// Every wait is bounded (the workspace's wait limit, default ~2 s); a warp
// that gives up records LCVQ_ERR_DEVICE_TIMEOUT in the group's error word and
// raises the CTA's abort flag, the others wind down, and the producer waits
// for the copies it issued before the CTA exits.
constexpr int kWideConsumers = 8;
constexpr int kWideThreads = (kWideConsumers + 1) * 32;
constexpr int kWideRows = 16 * kWideConsumers;
constexpr uint32_t kWideXPitch = 1040;    // 1024 X'' bytes per token + 16

template <int kItems>
struct GemvWideGroup {
  CUtensorMap codes[kItems];  // per item: [N rows][K/4 bytes], box 128 x 128 B, SW128
  int count, M;
  unsigned int* err;
  GemvItem item[kItems];  // tile_end in 128-row tiles
};

template <int NT, int kStages>
struct WideLayout {
  static constexpr uint32_t kCodeBytes = kWideRows * 128;  // one SW128 box
  static constexpr uint32_t kXBytes = NT * 8 * kWideXPitch;
  static constexpr uint32_t kStageBytes = (kCodeBytes + kXBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kBarOff = kStages * kStageBytes;
  static constexpr size_t kSmem = 1024 + size_t(kBarOff) + 2 * kStages * 8 + 16;  // + alignment
};

// kI8: the int8 path, as for gemv_group_kernel
template <int NT, int kStages, int kMinBlocks, int kItems, bool kI8 = false>
__global__ void __launch_bounds__(kWideThreads, kMinBlocks)
    gemv_wide_kernel(const __grid_constant__ GemvWideGroup<kItems> grp) {
  using Acc = typename std::conditional<kI8, int, float>::type;
  using L = WideLayout<NT, kStages>;
  extern __shared__ __align__(1024) unsigned char wsm_raw[];
  // SW128 boxes need 1024-byte aligned destinations
  unsigned char* wsm = wsm_raw + ((1024 - (sm100::smem_u32(wsm_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(wsm + L::kBarOff);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  const uint32_t sbase = sm100::smem_u32(wsm);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = grp.M;
  const int T = grp.item[grp.count - 1].tile_end;
  const int G = static_cast<int>(gridDim.x);
  auto tile_begin = [&](int item) { return item == 0 ? 0 : grp.item[item - 1].tile_end; };
  auto nchunks = [&](int K) { return static_cast<int>(ceil_div(ceil_div(K, kUnit), kAhead)); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], kWideConsumers);
    }
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();

  griddep_wait();  // X'' and corr written by the X-transforms are visible from here
  const long long lim = wait_limit(grp.err);
  // the abort flag as one decision per warp: the lanes of a warp go on to
  // warp-wide instructions together
  auto warp_abort = [&]() { return __shfl_sync(0xffffffffu, *abort_flag, 0) != 0; };

  if (warp == kWideConsumers) {
    // ------------------------------------------------------------ producer
    int seq = 0, item = 0, filled = 0;
    for (int tile = static_cast<int>(blockIdx.x); tile < T && !warp_abort(); tile += G) {
      while (tile >= grp.item[item].tile_end) ++item;
      const GemvItem& it = grp.item[item];
      const int64_t row0 = int64_t(tile - tile_begin(item)) * kWideRows;
      const int nch = nchunks(it.K);
      for (int c = 0; c < nch; ++c, ++seq) {
        const int s = seq % kStages;
        if (!__all_sync(0xffffffffu, sm100::mbar_wait(&empty[s], ((seq / kStages) & 1) ^ 1, lim))) {
          if (lane == 0) record_error(grp.err, LCVQ_ERR_DEVICE_TIMEOUT, 50);
          *abort_flag = 1;
          break;
        }
        const int64_t xk = int64_t(c) * (kAhead * kUnit);  // chunk's first position
        const uint32_t xbytes = static_cast<uint32_t>(it.K - xk < 512 ? (it.K - xk) * 2 : 1024);
        const uint32_t st = sbase + s * L::kStageBytes;
        if (lane == 0) {
          // the full box is counted, including the zero fill past N rows or K/4 bytes
          sm100::mbar_arrive_expect_tx(&full[s], L::kCodeBytes + static_cast<uint32_t>(M) * xbytes);
          sm100::tma_load_2d(&grp.codes[item], &full[s], wsm + s * L::kStageBytes,
                             c * (kAhead * 32), static_cast<int>(row0));
        }
        __syncwarp();
        if constexpr (kI8) {
          // int8 digits: the hi and lo planes (n_c bytes each) of token lane / 2,
          // the lo plane 16 bytes past the hi plane's end so that the lanes
          // reading the two planes hit different banks
          if (lane < 2 * M) {
            const uint32_t nc = xbytes / 2, pl = static_cast<uint32_t>(lane & 1);
            const unsigned char* src = reinterpret_cast<const unsigned char*>(it.Xpp) +
                                       int64_t(lane >> 1) * 2 * it.K + 2 * xk + pl * nc;
            sm100::bulk_load(st + L::kCodeBytes + (lane >> 1) * kWideXPitch + pl * (nc + 16), src,
                             nc, &full[s]);
          }
        } else if (lane < M) {
          sm100::bulk_load(st + L::kCodeBytes + lane * kWideXPitch,
                           it.Xpp + int64_t(lane) * it.K + xk, xbytes, &full[s]);
        }
        ++filled;
      }
    }
    // drain: every stage filled above has been consumed, so its copies landed
    for (int k = 0; k < kStages && !warp_abort(); ++k, ++seq) {
      const int s = seq % kStages;
      if (!__all_sync(0xffffffffu, sm100::mbar_wait(&empty[s], ((seq / kStages) & 1) ^ 1, lim))) {
        if (lane == 0) record_error(grp.err, LCVQ_ERR_DEVICE_TIMEOUT, 51);
        *abort_flag = 1;
      }
    }
    if (warp_abort() && lane == 0) {
      // gave up: wait for the last kStages fills to land, so no copy writes
      // shared memory after the CTA exits (the default limit: copies in flight
      // finish in microseconds)
      for (int n = filled - 1; n >= 0 && n >= filled - kStages; --n)
        sm100::mbar_wait(&full[n % kStages], (n / kStages) & 1, kDefaultWaitLimit);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;
  // per-lane constants: the SW128 offset of this lane's 8 code bytes of unit j
  // (16-byte chunk 2 j + t/2 of rows g, g + 8 sits at chunk ^ g), and the
  // offset and validity of its X'' token rows
  uint32_t coff[kAhead];
#pragma unroll
  for (int j = 0; j < kAhead; ++j)
    coff[j] = static_cast<uint32_t>(((2 * j + (t >> 1)) ^ g) << 4) + ((t & 1) << 3);
  // (int8: column g of token tile n is token 4 n + g/2, digit plane g % 2; a
  // chunk's lo plane starts n_c bytes after its hi plane)
  uint32_t xoff[NT];
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok = kI8 ? n * 4 + (g >> 1) : n * 8 + g;
    tokok[n] = tok < M;
    xoff[n] = static_cast<uint32_t>(tok * kWideXPitch + (kI8 ? 32 * t : 64 * t));
  }
  int seq = 0, item = 0;
  for (int tile = static_cast<int>(blockIdx.x); tile < T && !warp_abort(); tile += G) {
    while (tile >= grp.item[item].tile_end) ++item;
    const GemvItem& it = grp.item[item];
    const int K = it.K;
    const int nch = nchunks(K);
    Acc acc[kWideConsumers][NT][4];
#pragma unroll
    for (int v = 0; v < kWideConsumers; ++v)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[v][n][e] = Acc(0);

    bool ok = true;
    for (int c0 = 0; c0 < nch && ok; c0 += kWideConsumers) {
#pragma unroll
      for (int v = 0; v < kWideConsumers; ++v) {  // chunk c0 + v -> accumulator v
        const int c = c0 + v;
        if (c >= nch) break;
        const int s = seq % kStages;
        if (!__all_sync(0xffffffffu, sm100::mbar_wait(&full[s], (seq / kStages) & 1, lim))) {
          if (lane == 0) record_error(grp.err, LCVQ_ERR_DEVICE_TIMEOUT, 52);
          *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t st = sbase + s * L::kStageBytes;
        const uint32_t crow = st + (warp * 16 + g) * 128;  // rows g and g + 8: (row & 7) = g
        const uint32_t xst = st + L::kCodeBytes;
        const int rem = K - c * (kAhead * kUnit);   // positions of K left from this chunk on
        const int remt = rem - 32 * t;              // ... from this lane's first position on
        // int8: this lane's digit plane (the lo plane starts 16 bytes after the
        // chunk's n_c hi bytes)
        const uint32_t plane =
            (kI8 && (g & 1)) ? static_cast<uint32_t>(rem < 512 ? rem : 512) + 16u : 0u;
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
          if (j * kUnit >= rem) break;  // warp-uniform: past the end of K
          const bool kok = j * kUnit < remt;
          uint2 cw[2];
          cw[0] = lds_v2(crow + coff[j]);
          cw[1] = lds_v2(crow + 8 * 128 + coff[j]);
          if constexpr (kI8) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {  // word q of rows g, g + 8: 2 k32 tiles
              uint4 xq[NT];
#pragma unroll
              for (int n = 0; n < NT; ++n)
                xq[n] = (kok && tokok[n]) ? lds_v4(xst + xoff[n] + plane + j * kUnit + 16 * q)
                                          : make_uint4(0, 0, 0, 0);
              uint32_t r0[4], r1[4];
              dec_word_u8(q == 0 ? cw[0].x : cw[0].y, r0);
              dec_word_u8(q == 0 ? cw[1].x : cw[1].y, r1);
#pragma unroll
              for (int mm = 0; mm < 2; ++mm)
#pragma unroll
                for (int n = 0; n < NT; ++n)
                  mma_u8s8_16832(acc[v][n], r0[2 * mm], r1[2 * mm], r0[2 * mm + 1], r1[2 * mm + 1],
                                 word_of(xq[n], 2 * mm), word_of(xq[n], 2 * mm + 1));
            }
          } else {
          uint4 xb[2][NT][2];
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              if (kok && tokok[n]) {
                const uint32_t xa = xst + xoff[n] + (j * kUnit + 16 * q) * 2;
                xb[q][n][0] = lds_v4(xa);
                xb[q][n][1] = lds_v4(xa + 16);
              } else {
                xb[q][n][0] = make_uint4(0, 0, 0, 0);
                xb[q][n][1] = make_uint4(0, 0, 0, 0);
              }
            }
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t w0[2], w6[2], w12[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              w0[h] = q == 0 ? cw[h].x : cw[h].y;
              w6[h] = w0[h] >> 6;
              w12[h] = w0[h] >> 12;
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const uint32_t a00 = dec_pair_rt(2 * jj, w0[0], w6[0], w12[0]);
              const uint32_t a10 = dec_pair_rt(2 * jj, w0[1], w6[1], w12[1]);
              const uint32_t a01 = dec_pair_rt(2 * jj + 1, w0[0], w6[0], w12[0]);
              const uint32_t a11 = dec_pair_rt(2 * jj + 1, w0[1], w6[1], w12[1]);
#pragma unroll
              for (int n = 0; n < NT; ++n) {
                const uint32_t b0 = word_of(xb[q][n][jj >> 1], (2 * jj) & 3);
                const uint32_t b1 = word_of(xb[q][n][jj >> 1], (2 * jj + 1) & 3);
                mma_bf16_16816(acc[v][n], a00, a10, a01, a11, b0, b1);
              }
            }
          }
          }
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&empty[s]);
        ++seq;
      }
    }
    if (!ok) break;

    // the split kernel's fixed-order sum over the 8 K partitions, plus corr
    const int64_t row0 = int64_t(tile - tile_begin(item)) * kWideRows + warp * 16;
    if constexpr (kI8) {  // accumulator v holds class v: the split kernel's class sum
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int rh = 0; rh < 2; ++rh) {
          const int64_t row = row0 + g + 8 * rh;
          const int tok = n * 4 + t;
          if (row < it.N && tok < M) {
            float sum = 0.f;
#pragma unroll
            for (int v = 0; v < kWideConsumers; ++v)
              sum = i8_add_class(sum, acc[v][n][2 * rh], acc[v][n][2 * rh + 1],
                                 ld_global_f32(it.inv_s + tok * kWideConsumers + v));
            it.Y[int64_t(tok) * it.N + row] = f32_to_bf16(sum + ld_global_f32(it.corr + tok));
          }
        }
    } else {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t row = row0 + g + 8 * (e >> 1);
        const int tok = n * 8 + 2 * t + (e & 1);
        float sum = 0.f;
#pragma unroll
        for (int v = 0; v < kWideConsumers; ++v) sum += acc[v][n][e];
        if (row < it.N && tok < M)
          it.Y[int64_t(tok) * it.N + row] = f32_to_bf16(sum + ld_global_f32(it.corr + tok));
      }
    }
  }
  // the last CTA-wide point: consumers are done with every stage
  griddep_launch_dependents();
}

// stages of the wide-tile kernel per token-tile count
#ifndef LCVQ_WS1
#define LCVQ_WS1 4
#endif
#ifndef LCVQ_WS2
#define LCVQ_WS2 6
#endif

// code-ring depth (chunks per warp) per token-tile count
#ifndef LCVQ_GS1
#define LCVQ_GS1 4
#endif
#ifndef LCVQ_GS2
#define LCVQ_GS2 4
#endif
#ifndef LCVQ_GS4
#define LCVQ_GS4 3
#endif

// CTAs of a kernel that one device holds at once (cached per kernel and device)
int64_t resident_ctas(const void* kern, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int64_t> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(kern, dev);
  auto f = cache.find(key);
  if (f != cache.end()) return f->second;
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const int64_t v = int64_t(per_sm) * sms;
  cache[key] = v;
  return v;
}

template <int NT, int R, int kWarps, bool kPrefX, int kMinBlocks, int kStages, int kItems,
          bool kI8 = false>
cudaError_t launch_group_t(const GemvGroup<kItems>& grp, cudaStream_t s) {
  auto kern = gemv_group_kernel<NT, R, kWarps, kPrefX, kMinBlocks, kStages, kItems, kI8>;
  constexpr size_t smem = group_smem_ring<R, kStages, kWarps>() + group_smem_part<NT, R, kWarps>();
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
      e != cudaSuccess)
    return e;
  const int64_t tiles = grp.item[grp.count - 1].tile_end;
  const int64_t resident = resident_ctas(reinterpret_cast<const void*>(kern), kWarps * 32, smem);
  if (resident <= 0) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < resident ? tiles : resident), 1, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, grp);
}

// tile rows of the CTA shape used for M tokens
constexpr int kRowsSmallM = 16, kRowsLargeM = 32;
int group_rows(int64_t M) { return M <= 8 ? kRowsSmallM : kRowsLargeM; }

// CTA shapes measured best on the 4096 x 4096 workload (graph replays over
// rotated weights): M <= 8: 16 rows, 2 CTAs per SM; M <= 16: 32 rows, one CTA
// per SM with room for the X'' prefetch; M <= 32: 32 rows, no prefetch.
template <int kItems>
cudaError_t launch_group(const GemvGroup<kItems>& grp, cudaStream_t s) {
  if (grp.item[0].inv_s != nullptr)  // the int8 path (M <= kI8MaxM: one token tile)
    return launch_group_t<1, 1, 8, true, 2, LCVQ_GS1, kItems, true>(grp, s);
  if (grp.M <= 8) return launch_group_t<1, 1, 8, true, 2, LCVQ_GS1, kItems>(grp, s);
  if (grp.M <= 16) return launch_group_t<2, 2, 8, true, 1, LCVQ_GS2, kItems>(grp, s);
  return launch_group_t<4, 2, 8, false, 1, LCVQ_GS4, kItems>(grp, s);
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* Xpp, const float* corr, int64_t M, const uint8_t* packed,
                        int64_t d_out, int64_t d_in, uint16_t* Y, bool after_xform,
                        cudaStream_t s, int* launches, const float* inv_s) {
  // a single matrix is a group of one (the same kernel, so the same bits)
  GemvGroup<1> grp{};
  grp.count = 1;
  grp.M = static_cast<int>(M);
  grp.early_codes = after_xform ? 1 : 0;
  grp.item[0] = GemvItem{packed, Xpp, corr, Y, static_cast<int>(d_out), static_cast<int>(d_in),
                         static_cast<int>(ceil_div(d_out, group_rows(M))), inv_s};
  cudaError_t e = launch_group(grp, s);
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

namespace {
template <int NT, int kStages, int kMinBlocks, int kItems, bool kI8 = false>
cudaError_t launch_wide_t(const GemvWideGroup<kItems>& grp, cudaStream_t s) {
  auto kern = gemv_wide_kernel<NT, kStages, kMinBlocks, kItems, kI8>;
  constexpr size_t smem = WideLayout<NT, kStages>::kSmem;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
      e != cudaSuccess)
    return e;
  const int64_t tiles = grp.item[grp.count - 1].tile_end;
  const int64_t resident = resident_ctas(reinterpret_cast<const void*>(kern), kWideThreads, smem);
  if (resident <= 0) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < resident ? tiles : resident), 1, 1);
  cfg.blockDim = dim3(kWideThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, grp);
}
}  // namespace

#ifndef LCVQ_WIDE_MIN_TILES
#define LCVQ_WIDE_MIN_TILES 296
#endif

cudaError_t launch_gemv_grouped(const GemvJob* jobs, int count, int64_t M, cudaStream_t s,
                                int* launches, unsigned int* err) {
  // enough 128-row tiles to fill the device: the wide-tile kernel (M <= 16)
  int64_t wide_tiles = 0;
  for (int i = 0; i < count; ++i) wide_tiles += ceil_div(jobs[i].d_out, kWideRows);
  // 17..32 tokens: the tcgen05 form (four token tiles of mma.sync cost more
  // than the tensor cores' A-operand streaming rate)
  if (M > 16 && wide_tiles >= LCVQ_WIDE_MIN_TILES && gemv_tc_usable(M))
    return launch_gemv_tc_grouped(jobs, count, M, err, s, launches);
  if (wide_tiles >= LCVQ_WIDE_MIN_TILES) {
    for (int first = 0; first < count; first += kMaxGroupItems) {
      const int n = count - first < kMaxGroupItems ? count - first : kMaxGroupItems;
      GemvWideGroup<kMaxGroupItems> grp{};
      grp.count = n;
      grp.M = static_cast<int>(M);
      grp.err = err;
      int tiles = 0;
      for (int i = 0; i < n; ++i) {
        const GemvJob& j = jobs[first + i];
        tiles += static_cast<int>(ceil_div(j.d_out, kWideRows));
        grp.item[i] = GemvItem{j.packed, j.Xpp, j.corr, j.Y, static_cast<int>(j.d_out),
                               static_cast<int>(j.d_in), tiles, j.inv_s};
        if (!make_tensor_map_2d(&grp.codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, j.packed,
                                uint64_t(j.d_in / 4), uint64_t(j.d_out), uint64_t(j.d_in / 4),
                                kAhead * 32, kWideRows, true))
          return cudaErrorInvalidValue;
      }
      cudaError_t e = jobs[0].inv_s != nullptr
                          ? launch_wide_t<1, LCVQ_WS1, 2, kMaxGroupItems, true>(grp, s)
                      : M <= 8 ? launch_wide_t<1, LCVQ_WS1, 2, kMaxGroupItems>(grp, s)
                               : launch_wide_t<2, LCVQ_WS2, 1, kMaxGroupItems>(grp, s);
      ++*launches;
      if (e != cudaSuccess) return e;
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const int rows = group_rows(M);
  for (int first = 0; first < count; first += kMaxGroupItems) {
    const int n = count - first < kMaxGroupItems ? count - first : kMaxGroupItems;
    GemvGroup<kMaxGroupItems> grp{};
    grp.count = n;
    grp.M = static_cast<int>(M);
    grp.early_codes = 1;  // after launch_xform_grouped
    int tiles = 0;
    for (int i = 0; i < n; ++i) {
      const GemvJob& j = jobs[first + i];
      tiles += static_cast<int>(ceil_div(j.d_out, rows));
      grp.item[i] = GemvItem{j.packed, j.Xpp, j.corr, j.Y, static_cast<int>(j.d_out),
                             static_cast<int>(j.d_in), tiles, j.inv_s};
    }
    cudaError_t e = launch_group(grp, s);
    ++*launches;
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_xformed(const uint16_t* Xpp, const float* corr, int64_t M,
                                const uint8_t* packed, int64_t d_out, int64_t d_in, uint16_t* Y,
                                unsigned int* err, bool after_xform, cudaStream_t s,
                                int* launches) {
  if (M <= 32)
    return launch_gemv(Xpp, corr, M, packed, d_out, d_in, Y, after_xform, s, launches, nullptr);
  return launch_tc_forward(Xpp, true, corr, M, packed, d_out, d_in, 8, nullptr, nullptr, Y, err, s,
                           launches);
}

}  // namespace lcvq

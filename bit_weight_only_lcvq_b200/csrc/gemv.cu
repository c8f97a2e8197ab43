// Decode-GEMV for few tokens (M <= 32): Y = X W~ with W~ = A z + B streamed as
// packed 2-bit codes (LC-QAT technical summary, Methodology 3: the forward runs
// on INT2 x FP16 matmul operators).
//
// The kernel multiplies the transformed activations X'' (see xform.cu) with the
// raw codes on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   * weights are the 16-row A operand, tokens the 8-column B operand, so a
//     weight tile is decoded once and serves every token;
//   * codes go from HBM straight into registers (one 128-bit load per row and
//     lane per 256 codes) and are decoded by a single LOP3 per bf16 pair:
//     (word >> s) & 0x00030003 << 2p | 0x43004300 = bf16x2(128 + 4^p z_lo,
//     128 + 4^p z_hi); the power of two and the 128 offset are folded into X''
//     and the per-row constant `corr`, so decoding costs no float arithmetic;
//   * the MMA's logical k of each lane is mapped onto the lane's own code
//     words (the decoder order of X'' makes the B fragments contiguous loads);
//   * a CTA owns 16 R rows over the whole K (8 warps split K, fixed-order
//     shared-memory sum), so no partial sum leaves the CTA and the result is
//     deterministic;
//   * programmatic dependent launch: the code loads do not depend on the
//     X-transform, so they are issued before griddepcontrol.wait and stream
//     while the prologue runs.  The kernel touches nothing else before the
//     wait, and the X-transform waits for every earlier kernel before it lets
//     this one launch, so the early reads never race a producer of the codes.

#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace lcvq {

namespace {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 (128 + 4^p z_c, 128 + 4^p z_{c+8}) of pair c of a 16-code word, given
// the word and its shifts by 6 and 12.
template <int C>
__device__ __forceinline__ uint32_t dec_pair(uint32_t w0, uint32_t w6, uint32_t w12) {
  constexpr int P = C % 3;
  const uint32_t src = (C < 3) ? w0 : ((C < 6) ? w6 : w12);
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n"  // (a & b) | c
      : "=r"(r)
      : "r"(src), "n"(0x00030003u << (2 * P)), "n"(0x43004300u));
  return r;
}

// same as dec_pair<C> for a C that is a compile-time constant after unrolling
__device__ __forceinline__ uint32_t dec_pair_rt(int c, uint32_t w0, uint32_t w6, uint32_t w12) {
  switch (c) {
    case 0: return dec_pair<0>(w0, w6, w12);
    case 1: return dec_pair<1>(w0, w6, w12);
    case 2: return dec_pair<2>(w0, w6, w12);
    case 3: return dec_pair<3>(w0, w6, w12);
    case 4: return dec_pair<4>(w0, w6, w12);
    case 5: return dec_pair<5>(w0, w6, w12);
    case 6: return dec_pair<6>(w0, w6, w12);
    default: return dec_pair<7>(w0, w6, w12);
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

// CTA: kWarps warps on 16 R weight rows over the whole K, so no partial sum
// leaves the CTA.  Warp w takes K slice w.  A "unit" is 128 codes of each of the
// CTA's rows: lane (g, t) holds 2 words of rows g and g + 8 of every row
// block (8 B each); a warp keeps up to kAhead units of loads in flight.
// Launch order with the X-transform (programmatic dependent launch): the code
// loads are issued before griddepcontrol.wait, so they overlap the prologue;
// X'' and corr are read only after it.
constexpr int kUnit = 128;  // codes per row per unit (32 B)
constexpr int kAhead = 4;

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];\n"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// kPrefX: keep the next unit's X'' fragments in flight (costs registers);
// kMinBlocks: CTAs per SM the register budget must allow.
template <int NT, int R, int kWarps, bool kPrefX, int kMinBlocks>
__global__ void __launch_bounds__(kWarps * 32, kMinBlocks)
    gemv_kernel(const uint16_t* __restrict__ Xpp, const float* __restrict__ corr, int M,
                const uint8_t* __restrict__ packed, int64_t N, int64_t K,
                uint16_t* __restrict__ Y) {
  constexpr int MP = NT * 8;
  constexpr int ROWS = 16 * R;
  __shared__ float part[kWarps][ROWS][MP + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row0 = int64_t(blockIdx.x) * ROWS;
  const int64_t Kb = K / 4;
  const int64_t nunits = ceil_div(K, kUnit);
  const int64_t u0 = nunits * warp / kWarps, u1 = nunits * (warp + 1) / kWarps;

  const uint8_t* rowp[R][2];
  bool rowok[R][2];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t row = row0 + r * 16 + g + 8 * h;
      rowok[r][h] = row < N;
      rowp[r][h] = packed + (rowok[r][h] ? row : 0) * Kb + 8 * t;
    }

  auto load_unit = [&](int64_t u, uint2 (&cw)[R][2]) {
    const bool kok = u < u1 && u * kUnit + 32 * t < K;  // K % 64 == 0: whole lane chunks
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        cw[r][h] = (kok && rowok[r][h]) ? ld_stream_v2(rowp[r][h] + u * 32) : make_uint2(0, 0);
  };

  uint2 ring[kAhead][R][2];
#pragma unroll
  for (int j = 0; j < kAhead; ++j) load_unit(u0 + j, ring[j]);

  griddep_wait();  // X'' and corr written by the X-transform are visible from here

  const uint16_t* xrow[NT];
  bool tokok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int tok = n * 8 + g;
    tokok[n] = tok < M;
    xrow[n] = Xpp + int64_t(tokok[n] ? tok : 0) * K + 32 * t;
  }

  float acc[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

  // X'' fragments of one unit: word q, token tile n -> two 16-byte halves
  auto load_x = [&](int64_t u, uint4 (&xb)[2][NT][2]) {
    const bool kok = u < u1 && u * kUnit + 32 * t < K;
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (kok && tokok[n]) {
          const uint4* src = reinterpret_cast<const uint4*>(xrow[n] + u * kUnit + 16 * q);
          xb[q][n][0] = __ldg(src);
          xb[q][n][1] = __ldg(src + 1);
        } else {
          xb[q][n][0] = make_uint4(0, 0, 0, 0);
          xb[q][n][1] = make_uint4(0, 0, 0, 0);
        }
      }
  };
  uint4 xcur[2][NT][2], xnxt[2][NT][2];
  load_x(u0, xcur);

  for (int64_t base = u0; base < u1; base += kAhead) {
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int64_t u = base + j;
      if (u >= u1) break;
      if constexpr (kPrefX) load_x(u + 1, xnxt);
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // word q of each row: 16 codes, 4 k16 tiles
        uint32_t w0[R][2], w6[R][2], w12[R][2];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            w0[r][h] = q == 0 ? ring[j][r][h].x : ring[j][r][h].y;
            w6[r][h] = w0[r][h] >> 6;
            w12[r][h] = w0[r][h] >> 12;
          }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {  // k16 tile: pairs 2jj, 2jj+1 of word q
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
              mma_bf16_16816(acc[r][n], a[r][0][0], a[r][1][0], a[r][0][1], a[r][1][1], b0, b1);
          }
        }
      }
      load_unit(u + kAhead, ring[j]);  // refill the slot just consumed
      if constexpr (kPrefX) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            xcur[q][n][0] = xnxt[q][n][0];
            xcur[q][n][1] = xnxt[q][n][1];
          }
      } else {
        load_x(u + 1, xcur);
      }
    }
  }

  // every CTA has passed its main loop: the next kernel may start launching
  griddep_launch_dependents();

#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int lr = r * 16 + g;
      const int tk = n * 8 + 2 * t;
      part[warp][lr][tk] = acc[r][n][0];
      part[warp][lr][tk + 1] = acc[r][n][1];
      part[warp][lr + 8][tk] = acc[r][n][2];
      part[warp][lr + 8][tk + 1] = acc[r][n][3];
    }
  __syncthreads();
  // sum the 8 K slices in slice order, add the per-row constant, store
  for (int e = threadIdx.x; e < ROWS * M; e += kWarps * 32) {
    const int lr = e % ROWS, tok = e / ROWS;
    const int64_t grow = row0 + lr;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sum += part[w][lr][tok];
    if (grow < N) Y[int64_t(tok) * N + grow] = f32_to_bf16(sum + corr[tok]);
  }
}

template <int NT, int R, int kWarps, bool kPrefX, int kMinBlocks>
cudaError_t launch_gemv_t(const uint16_t* Xpp, const float* corr, int M, const uint8_t* packed,
                          int64_t N, int64_t K, uint16_t* Y, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(N, 16 * R)), 1, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, R, kWarps, kPrefX, kMinBlocks>, Xpp, corr, M,
                            packed, N, K, Y);
}

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
  const uint16_t* Xpp;    // [M][K] X'' (decoder order)
  const float* corr;      // [M]
  uint16_t* Y;            // [M][N]
  int N, K;
  int tile_end;  // tiles of items 0 .. this one
};
template <int kItems>
struct GemvGroup {
  int count, M;
  GemvItem item[kItems];
};

template <int NT, int R, int kWarps, bool kPrefX, int kMinBlocks, int kItems>
__global__ void __launch_bounds__(kWarps * 32, kMinBlocks)
    gemv_group_kernel(const __grid_constant__ GemvGroup<kItems> grp) {
  constexpr int MP = NT * 8;
  constexpr int ROWS = 16 * R;
  // [2][kWarps][ROWS][MP + 1] partial tiles (dynamic: above the static limit for NT = 4)
  extern __shared__ float part_smem[];
  auto part = reinterpret_cast<float(*)[kWarps][ROWS][MP + 1]>(part_smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = grp.M;
  const int T = grp.item[grp.count - 1].tile_end;
  const int G = static_cast<int>(gridDim.x);

  // a chunk of this warp: tile, its item, chunk index inside the tile
  struct Cur {
    int tile, item, chunk;
  };
  // first chunk of this warp at or after c (c.chunk is a candidate index)
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

  auto load_unit = [&](const Cur& c, int j, uint2 (&cw)[R][2]) {
    bool any = c.tile < T;
    const GemvItem& it = grp.item[any ? c.item : 0];
    const int64_t u = int64_t(c.chunk) * kAhead + j;
    const bool kok = any && u * kUnit + 32 * t < it.K;
    const int64_t row0 = int64_t(c.tile - tile_begin(c.item)) * ROWS;
    const int64_t Kb = it.K / 4;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = row0 + r * 16 + g + 8 * h;
        cw[r][h] = (kok && row < it.N) ? ld_stream_v2(it.packed + row * Kb + 8 * t + u * 32)
                                       : make_uint2(0, 0);
      }
  };
  // X'' fragments of unit j of chunk c: word q, token tile n -> two 16-byte halves
  auto load_x = [&](const Cur& c, int j, uint4 (&xb)[2][NT][2]) {
    const bool any = c.tile < T;
    const GemvItem& it = grp.item[any ? c.item : 0];
    const int64_t u = int64_t(c.chunk) * kAhead + j;
    const bool kok = any && u * kUnit + 32 * t < it.K;
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tok = n * 8 + g;
        if (kok && tok < M) {
          const uint4* src =
              reinterpret_cast<const uint4*>(it.Xpp + int64_t(tok) * it.K + u * kUnit + 32 * t + 16 * q);
          xb[q][n][0] = __ldg(src);
          xb[q][n][1] = __ldg(src + 1);
        } else {
          xb[q][n][0] = make_uint4(0, 0, 0, 0);
          xb[q][n][1] = make_uint4(0, 0, 0, 0);
        }
      }
  };

  Cur cur = seek(Cur{static_cast<int>(blockIdx.x), 0, warp});
  uint2 ring[kAhead][R][2];
#pragma unroll
  for (int j = 0; j < kAhead; ++j) load_unit(cur, j, ring[j]);
  Cur nxt = advance(cur);

  griddep_wait();  // X'' and corr written by the X-transform are visible from here

  uint4 xcur[2][NT][2], xnxt[2][NT][2];
  load_x(cur, 0, xcur);

  int eitem = 0;  // item of the tile in the epilogue
  int buf = 0;
  for (int tile = static_cast<int>(blockIdx.x); tile < T; tile += G, buf ^= 1) {
    float acc[R][NT][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

    while (cur.tile == tile) {  // this warp's chunks of the tile
      const int Kc = grp.item[cur.item].K;
#pragma unroll
      for (int j = 0; j < kAhead; ++j) {
        if constexpr (kPrefX) {
          if (j + 1 < kAhead) load_x(cur, j + 1, xnxt);
          else load_x(nxt, 0, xnxt);
        }
        if ((int64_t(cur.chunk) * kAhead + j) * kUnit < Kc) {  // warp-uniform
#pragma unroll
          for (int q = 0; q < 2; ++q) {  // word q of each row: 16 codes, 4 k16 tiles
            uint32_t w0[R][2], w6[R][2], w12[R][2];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                w0[r][h] = q == 0 ? ring[j][r][h].x : ring[j][r][h].y;
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
        load_unit(nxt, j, ring[j]);  // refill the slot with the next chunk's unit
        if constexpr (kPrefX) {
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              xcur[q][n][0] = xnxt[q][n][0];
              xcur[q][n][1] = xnxt[q][n][1];
            }
        } else {
          if (j + 1 < kAhead) load_x(cur, j + 1, xcur);
          else load_x(nxt, 0, xcur);
        }
      }
      cur = nxt;
      nxt = advance(nxt);
    }

    // the CTA's last tile: the next kernel may start launching
    if (tile + G >= T) griddep_launch_dependents();

#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int lr = r * 16 + g;
        const int tk = n * 8 + 2 * t;
        part[buf][warp][lr][tk] = acc[r][n][0];
        part[buf][warp][lr][tk + 1] = acc[r][n][1];
        part[buf][warp][lr + 8][tk] = acc[r][n][2];
        part[buf][warp][lr + 8][tk + 1] = acc[r][n][3];
      }
    __syncthreads();
    while (tile >= grp.item[eitem].tile_end) ++eitem;
    const GemvItem& it = grp.item[eitem];
    const int64_t row0 = int64_t(tile - tile_begin(eitem)) * ROWS;
    // sum the warps' K chunks in warp order, add the per-row constant, store
    for (int e = threadIdx.x; e < ROWS * M; e += kWarps * 32) {
      const int lr = e % ROWS, tok = e / ROWS;
      const int64_t grow = row0 + lr;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += part[buf][w][lr][tok];
      if (grow < it.N) it.Y[int64_t(tok) * it.N + grow] = f32_to_bf16(sum + it.corr[tok]);
    }
  }
}

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

template <int NT, int R, int kWarps, bool kPrefX, int kMinBlocks, int kItems>
cudaError_t launch_group_t(const GemvGroup<kItems>& grp, cudaStream_t s) {
  auto kern = gemv_group_kernel<NT, R, kWarps, kPrefX, kMinBlocks, kItems>;
  constexpr size_t smem = size_t(2) * kWarps * (16 * R) * (NT * 8 + 1) * sizeof(float);
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
  if (grp.M <= 8) return launch_group_t<1, 1, 8, true, 2, kItems>(grp, s);
  if (grp.M <= 16) return launch_group_t<2, 2, 8, true, 1, kItems>(grp, s);
  return launch_group_t<4, 2, 8, false, 1, kItems>(grp, s);
}

}  // namespace

#ifndef LCVQ_GEMV_GROUPED
#define LCVQ_GEMV_GROUPED 1
#endif

cudaError_t launch_gemv(const uint16_t* Xpp, const float* corr, int64_t M, const uint8_t* packed,
                        int64_t d_out, int64_t d_in, uint16_t* Y, cudaStream_t s,
                        int* launches) {
  cudaError_t e;
  const int m = static_cast<int>(M);
  if (LCVQ_GEMV_GROUPED) {
    GemvGroup<1> grp{};
    grp.count = 1;
    grp.M = m;
    grp.item[0] = GemvItem{packed, Xpp, corr, Y, static_cast<int>(d_out), static_cast<int>(d_in),
                           static_cast<int>(ceil_div(d_out, group_rows(M)))};
    e = launch_group(grp, s);
  } else if (M <= 8) {
    e = launch_gemv_t<1, 1, 8, true, 2>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  } else if (M <= 16) {
    e = launch_gemv_t<2, 2, 8, true, 1>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  } else {
    e = launch_gemv_t<4, 2, 8, false, 1>(Xpp, corr, m, packed, d_out, d_in, Y, s);
  }
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemv_grouped(const GemvJob* jobs, int count, int64_t M, cudaStream_t s,
                                int* launches) {
  const int rows = group_rows(M);
  for (int first = 0; first < count; first += kMaxGroupItems) {
    const int n = count - first < kMaxGroupItems ? count - first : kMaxGroupItems;
    GemvGroup<kMaxGroupItems> grp{};
    grp.count = n;
    grp.M = static_cast<int>(M);
    int tiles = 0;
    for (int i = 0; i < n; ++i) {
      const GemvJob& j = jobs[first + i];
      tiles += static_cast<int>(ceil_div(j.d_out, rows));
      grp.item[i] = GemvItem{j.packed, j.Xpp, j.corr, j.Y, static_cast<int>(j.d_out),
                             static_cast<int>(j.d_in), tiles};
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
                                unsigned int* err, cudaStream_t s, int* launches) {
  if (M <= 32) return launch_gemv(Xpp, corr, M, packed, d_out, d_in, Y, s, launches);
  return launch_tc_forward(Xpp, true, corr, M, packed, d_out, d_in, 8, nullptr, nullptr, Y, err, s,
                           launches);
}

}  // namespace lcvq

// Decode-GEMV over a group of matrices on the 5th-generation tensor cores,
// with the decoded weights in tensor memory.  Y_i = X_i W~_i for M <= 32
// tokens (LC-QAT technical summary, Methodology 3: the forward on INT2 x FP16
// matmul operators), in the algebraic form of xform.cu: Y = X'' v^T + corr,
// v = 128 + 4^p z decoded by one LOP3 per bf16 pair.
//
// The weights are the MMA's M dimension (tiles of 128 rows over the whole K)
// and the tokens its N dimension (32, zero-filled past M), so the tensor core,
// not the decode, scales with the token count.  Decoding 2-bit codes into
// bf16 multiplies their bytes by 8; through shared memory that expansion would
// cap the kernel at shared-memory bandwidth, so the decoders write the bf16 A
// tiles straight into tensor memory (tcgen05.st) and the MMA reads A from
// there (tcgen05.mma with A in TMEM, B = X'' from shared memory).
//
//   warp 0        TMA producer of code chunks (one box of 128 rows x 128 B =
//                 512 codes per row, 128-byte swizzle) into a shared-memory ring
//   warp 1        TMEM allocator + single-thread MMA issuer
//   warp 2        TMA producer of X'' boxes (32 tokens x 64 positions, SW128)
//   warps 3..18   decoders: warp w owns TMEM lanes 32 (w % 4) .. + 31 (rows)
//                 and k-block (w - 3) / 4 of every code chunk, so a chunk's
//                 four k-blocks are decoded at once per lane quarter
//   warps 19..22  epilogue: TMEM -> registers, + corr, -> Y (bf16)
//
// TMEM columns: kAStages A slots of 64 columns (a k-block: 128 bf16 per row),
// then two 32-column D buffers (tile i's epilogue overlaps tile i+1's MMAs).
// Every wait is bounded (the workspace's wait limit, default ~2 s); a role
// that gives up records LCVQ_ERR_DEVICE_TIMEOUT in the group's error word,
// raises the CTA's abort flag, and the others wind down; the producers wait
// for their copies in flight and the MMA issuer drains its MMAs before the
// TMEM is released.
#include <cudaTypedefs.h>

#include <map>
#include <mutex>

#include "codec.cuh"
#include "common.cuh"
#include "gemv_common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lcvq {

using namespace sm100;

namespace {

constexpr int kTcRows = 128;        // weight rows per tile (MMA M)
constexpr int kTcTok = 32;          // token columns (MMA N)
constexpr int kTcKB = 128;          // positions per k-block (A slot, MMA group)
constexpr int kSub = 4;             // k-blocks per code chunk
constexpr int kTcCodeBytes = kTcRows * kTcKB * kSub / 4;  // 16 KB of codes per chunk
constexpr int kTcXBytes = kTcTok * kTcKB * 2;          // 8 KB of X'' per k-block
constexpr int kCStages = 4;         // code ring (64 KB)
constexpr int kAStages = 6;         // A (TMEM) + X'' (shared) ring
constexpr int kTmemCols = 512;
constexpr uint32_t kDCol0 = kAStages * 64;            // first D column
constexpr int kDecPerQuarter = 4;   // decoder warps per TMEM lane quarter (= kSub)
constexpr int kDecWarps = 4 * kDecPerQuarter;
constexpr int kTcThreads = 32 * (3 + kDecWarps + 4);
constexpr int kTcItems = 48;        // matrices per launch (2 tensor maps each)

static_assert(kDCol0 + 2 * kTcTok <= kTmemCols, "TMEM budget");
static_assert(kDecPerQuarter == kSub, "one decoder warp per k-block of a chunk and lane quarter");

struct TcItem {
  const float* corr;  // [M]
  uint16_t* Y;        // [M][N]
  int N, K;
  int tile_end;       // 128-row tiles of items 0 .. this one
};
struct TcGroup {
  CUtensorMap codes[kTcItems];  // [N rows][K/4 bytes], box 128 B x 128 rows
  CUtensorMap xpp[kTcItems];    // [M rows][K] bf16, box 64 x 32, 128-byte swizzle
  int count, M;
  unsigned int* err;
  TcItem item[kTcItems];
};

// shared memory: 1024 alignment slack | X'' ring | code ring | barriers
constexpr size_t kTcSmem = 1024 + size_t(kAStages) * kTcXBytes + size_t(kCStages) * kTcCodeBytes +
                           1024;


__device__ __forceinline__ void tc_fail(const TcGroup& g, volatile int* abort_flag, unsigned site) {
  record_error(g.err, LCVQ_ERR_DEVICE_TIMEOUT, site);
  *abort_flag = 1;
}

__global__ void __launch_bounds__(kTcThreads, 1) gemv_tc_kernel(const __grid_constant__ TcGroup grp) {
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;                                  // kAStages x 8 KB (SW128 boxes)
  uint8_t* sC = sX + kAStages * kTcXBytes;             // kCStages x 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + kCStages * kTcCodeBytes);
  uint64_t* cfull = bars;                              // codes landed (TMA)
  uint64_t* cempty = cfull + kCStages;                 // codes read (decoders)
  uint64_t* xfull = cempty + kCStages;                 // X'' landed (TMA)
  uint64_t* afull = xfull + kAStages;                  // A slot written (decoders)
  uint64_t* aempty = afull + kAStages;                 // A slot and X'' read (MMA commit)
  uint64_t* tfull = aempty + kAStages;                 // D buffer complete (MMA commit)
  uint64_t* tempty = tfull + 2;                        // D buffer read (epilogue)
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = grp.item[grp.count - 1].tile_end;
  const int G = static_cast<int>(gridDim.x);
  auto tile_begin = [&](int item) { return item == 0 ? 0 : grp.item[item - 1].tile_end; };
  // k-blocks of a tile, whole chunks (the box past K reads zeros)
  auto kblocks = [&](int item) {
    return kSub * static_cast<int>(ceil_div(grp.item[item].K, kTcKB * kSub));
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCStages; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], 4 * kSub);        // every decoder warp of the chunk
    }
    for (int a = 0; a < kAStages; ++a) {
      mbar_init(&xfull[a], 1);
      mbar_init(&afull[a], 4);
      mbar_init(&aempty[a], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const long long lim = wait_limit(grp.err);
  // the abort flag as one decision per warp, for the roles whose lanes go on to
  // warp-wide instructions together
  auto warp_abort = [&]() { return __shfl_sync(0xffffffffu, *abort_flag, 0) != 0; };

  if (warp == 0) {
    // ------------------------------------------------------------ code producer
    // codes are not written by the kernels this one may overlap: no wait needed
    if (lane == 0) {
      int g = 0, item = 0;
      for (int tile = static_cast<int>(blockIdx.x); tile < T && !*abort_flag; tile += G) {
        while (tile >= grp.item[item].tile_end) ++item;
        const int row0 = (tile - tile_begin(item)) * kTcRows;
        const int nch = kblocks(item) / kSub;
        for (int ch = 0; ch < nch; ++ch, ++g) {  // g counts chunks here
          const int s = g % kCStages;
          if (!mbar_wait(&cempty[s], ((g / kCStages) & 1) ^ 1, lim)) {
            tc_fail(grp, abort_flag, 60);
            break;
          }
          mbar_arrive_expect_tx(&cfull[s], kTcCodeBytes);
          tma_load_2d(&grp.codes[item], &cfull[s], sC + s * kTcCodeBytes, ch * (kTcKB * kSub / 4),
                      row0);
        }
      }
      if (*abort_flag)  // the copies in flight land before the CTA exits
        for (int n = g - 1; n >= 0 && n >= g - kCStages; --n)
          mbar_wait(&cfull[n % kCStages], (n / kCStages) & 1, kDefaultWaitLimit);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ X'' producer
    griddep_wait();  // X'' and corr written by the X-transform are visible from here
    if (lane == 0) {
      int g = 0, item = 0;
      for (int tile = static_cast<int>(blockIdx.x); tile < T && !*abort_flag; tile += G) {
        while (tile >= grp.item[item].tile_end) ++item;
        const int nkb = kblocks(item);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int a = g % kAStages;
          if (!mbar_wait(&aempty[a], ((g / kAStages) & 1) ^ 1, lim)) {
            tc_fail(grp, abort_flag, 61);
            break;
          }
          mbar_arrive_expect_tx(&xfull[a], kTcXBytes);
          tma_load_2d(&grp.xpp[item], &xfull[a], sX + a * kTcXBytes, kb * kTcKB, 0);
          tma_load_2d(&grp.xpp[item], &xfull[a], sX + a * kTcXBytes + kTcXBytes / 2,
                      kb * kTcKB + kTcKB / 2, 0);
        }
      }
      if (*abort_flag)  // the copies in flight land before the CTA exits
        for (int n = g - 1; n >= 0 && n >= g - kAStages; --n)
          mbar_wait(&xfull[n % kAStages], (n / kAStages) & 1, kDefaultWaitLimit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTcRows, kTcTok, false, false);
      int g = 0, item = 0, local = 0;
      bool issued = false;
      for (int tile = static_cast<int>(blockIdx.x); tile < T && !*abort_flag; tile += G, ++local) {
        while (tile >= grp.item[item].tile_end) ++item;
        const int buf = local & 1;
        if (!mbar_wait(&tempty[buf], ((local >> 1) & 1) ^ 1, lim)) {
          tc_fail(grp, abort_flag, 62);
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + kDCol0 + buf * kTcTok;
        const int nkb = kblocks(item);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int a = g % kAStages;
          const uint32_t par = (g / kAStages) & 1;
          if (!mbar_wait(&afull[a], par, lim) || !mbar_wait(&xfull[a], par, lim)) {
            tc_fail(grp, abort_flag, 63);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xs = smem_u32(sX + a * kTcXBytes);
#pragma unroll
          for (int sb = 0; sb < 2; ++sb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(dcol, tmem + a * 64 + sb * 32 + kk * 8,
                     sdesc_sw128(xs + sb * (kTcXBytes / 2) + kk * 32, 16, 1024), idesc,
                     (kb | sb | kk) != 0 ? 1u : 0u);
          issued = true;
          mma_commit(&aempty[a]);
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
      }
      if (issued) {  // no MMA may still run when the TMEM is released
        mma_commit(drain);
        // the default limit: TMEM may be released only after the running MMAs
        if (!mbar_wait(drain, 0, kDefaultWaitLimit)) tc_fail(grp, abort_flag, 64);
      }
    }
  } else if (warp < 3 + kDecWarps) {
    // ------------------------------------------------------------ decoders
    const int q = warp & 3;                 // TMEM lane quarter = rows 32 q .. 32 q + 31
    const int slot = (warp - 3) >> 2;       // k-blocks g with g % kDecPerQuarter == slot
    const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
    int g = 0, item = 0;
    for (int tile = static_cast<int>(blockIdx.x); tile < T && !warp_abort(); tile += G) {
      while (tile >= grp.item[item].tile_end) ++item;
      const int nkb = kblocks(item);
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb, ++g) {
        if (g % kDecPerQuarter != slot) continue;
        const int c = g / kSub;  // code chunk of this k-block (kDecPerQuarter == kSub)
        const int s = c % kCStages, a = g % kAStages;
        const bool landed = mbar_wait(&cfull[s], (c / kCStages) & 1, lim) &&
                            mbar_wait(&aempty[a], ((g / kAStages) & 1) ^ 1, lim);
        if (!__all_sync(0xffffffffu, landed)) {  // one outcome per warp
          tc_fail(grp, abort_flag, 65);
          ok = false;
          break;
        }
        // this row's 128 codes of the k-block: 16-byte chunks 2 slot and 2 slot + 1
        // of its 128-byte chunk row, stored at chunk ^ (row & 7) (128-byte swizzle)
        const int row = 32 * q + lane;
        const uint8_t* crow = sC + s * kTcCodeBytes + row * (kTcKB * kSub / 4);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4 cw =
              *reinterpret_cast<const uint4*>(crow + (((2 * slot + half) ^ (row & 7)) << 4));
          uint32_t v[32];
          dec_word8(cw.x, v);
          dec_word8(cw.y, v + 8);
          dec_word8(cw.z, v + 16);
          dec_word8(cw.w, v + 24);
          tmem_st32(tmem + lanes + a * 64 + half * 32, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&cempty[s]);
          mbar_arrive(&afull[a]);
        }
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    griddep_wait();  // corr is written by the X-transform
    const int q = warp & 3;
    const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
    const int M = grp.M;
    int item = 0, local = 0;
    for (int tile = static_cast<int>(blockIdx.x); tile < T && !warp_abort(); tile += G, ++local) {
      while (tile >= grp.item[item].tile_end) ++item;
      const TcItem& it = grp.item[item];
      const int buf = local & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (local >> 1) & 1, lim))) {
        tc_fail(grp, abort_flag, 66);
        break;
      }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tmem + lanes + kDCol0 + buf * kTcTok, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      const int64_t row = int64_t(tile - tile_begin(item)) * kTcRows + 32 * q + lane;
      if (row < it.N) {
#pragma unroll
        for (int tok = 0; tok < kTcTok; ++tok)
          if (tok < M)
            it.Y[int64_t(tok) * it.N + row] =
                f32_to_bf16(__uint_as_float(r[tok]) + ld_global_f32(it.corr + tok));
      }
    }
    if (threadIdx.x == 32 * (3 + kDecWarps)) griddep_launch_dependents();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// one CTA per SM: each allocates all 512 TMEM columns, so a second CTA on an
// SM would only wait for the first to finish
int tc_resident() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  auto f = cache.find(dev);
  if (f != cache.end()) return f->second;
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_tc_kernel, kTcThreads, kTcSmem) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm < 1)
    return 0;
  cache[dev] = sms;
  return sms;
}

}  // namespace

bool gemv_tc_usable(int64_t M) { return M >= 1 && M <= kTcTok; }

cudaError_t launch_gemv_tc_grouped(const GemvJob* jobs, int count, int64_t M, unsigned int* err,
                                   cudaStream_t s, int* launches) {
  if (!gemv_tc_usable(M)) return cudaErrorInvalidValue;
  if (cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(gemv_tc_kernel), kTcSmem);
      e != cudaSuccess)
    return e;
  const int resident = tc_resident();
  if (resident <= 0) return cudaErrorInvalidConfiguration;
  for (int first = 0; first < count; first += kTcItems) {
    const int n = count - first < kTcItems ? count - first : kTcItems;
    TcGroup grp{};
    grp.count = n;
    grp.M = static_cast<int>(M);
    grp.err = err;
    int tiles = 0;
    for (int i = 0; i < n; ++i) {
      const GemvJob& j = jobs[first + i];
      tiles += static_cast<int>(ceil_div(j.d_out, kTcRows));
      grp.item[i] = TcItem{j.corr, j.Y, static_cast<int>(j.d_out), static_cast<int>(j.d_in), tiles};
      if (!make_tensor_map_2d(&grp.codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, j.packed,
                              uint64_t(j.d_in / 4), uint64_t(j.d_out), uint64_t(j.d_in / 4),
                              kTcKB * kSub / 4, kTcRows, true) ||
          !make_tensor_map_2d(&grp.xpp[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, j.Xpp,
                              uint64_t(j.d_in), uint64_t(M), uint64_t(j.d_in) * 2, kTcKB / 2,
                              kTcTok, true))
        return cudaErrorInvalidValue;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles < resident ? tiles : resident), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = kTcSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_tc_kernel, grp);
    ++*launches;
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace lcvq

// Prologue of the algebraic form of the forward (LC-QAT technical summary,
// Methodology 3: the forward is recast onto INT2 x FP16 matmul operators).
//
// For every activation row x and every d-vector g:
//     sum_k x_k W~[n][k] = sum_g x_g^T (A z_g + B)
//                        = sum_k X'_k z_k + sum_g x_g^T B
// with X'[g d + j] = sum_i x[g d + i] A[i][j].  Centering the codes
// (zc = z - 3/2, W~ = A zc + B', B' = B + 3/2 A 1) gives the same sum as
// sum_k X'_k zc_k + s', s' = sum_g x_g^T B'.
//
// The tensor-core main loops multiply X'' (below) with codes that are decoded
// by one LOP3 each into the bf16 value 128 + 4^p z, p = p(position) in {0,1,2}
// (the code lands in mantissa bits 2p..2p+1 of a bf16 whose exponent says 128).
// So the B operand is X'' = bf16(X') * 4^-p (exact power-of-two scaling) and
//     acc = sum_k X''_k (128 + 4^p z_k) = sum_k X'r_k z_k + 128 sum_k X''_k,
// where X'r = bf16(X').  The per-row constant
//     corr = s' - 3/2 sum_k X'r_k - 128 sum_k X''_k
// makes acc + corr = sum_k X'r_k zc_k + s': the centred form, whose only
// rounding is that of X' to bf16 (relative 2^-9 per term, against codes of
// magnitude <= 3/2).  The sums are formed in fp64.
//
// K order ("decoder order"): inside every block of 16 consecutive k, the decoder
// turns one 32-bit word of codes into 8 bf16x2 pairs, pair c holding positions
// c and c + 8 (the same bit offset in the two 16-bit halves).  X'' is stored in
// that order: element 2c of the block is position c, element 2c+1 is c + 8;
// p(c) = c mod 3.
#include "common.cuh"
#include "internal.h"
#include "xform.cuh"

namespace lcvq {

constexpr int kXfThreads = 256;

// One launch transforms the rows of up to kItems matrices' activations: CTA
// (m, i) does row m of item i (a single call is a group of one).
struct XformItem {
  const uint16_t* X;  // [M][d_in] bf16
  const float* A;     // [D*D]
  const float* B;     // [D]
  uint16_t* Xpp;      // [M][d_in] out (bf16 X'', or the int8 digit planes)
  float* corr;        // [M] out
  float* inv_s;       // [M] out (int8 digits only: 1 / the row's scale)
  int64_t d_in;
};
template <int kItems>
struct XformGroup {
  XformItem item[kItems];
};

template <int D, int kItems>
__global__ void __launch_bounds__(kXfThreads)
    xform_kernel(const __grid_constant__ XformGroup<kItems> grp) {
  const XformItem& it = grp.item[blockIdx.y];
  // X, A and B may come from the kernel just before this one: read them with
  // ld_global_*, never through the read-only path
  const uint16_t* X = it.X;
  const float* A = it.A;
  const float* B = it.B;
  uint16_t* __restrict__ Xpp = it.Xpp;
  float* __restrict__ corr = it.corr;
  const int64_t d_in = it.d_in;
  __shared__ float sA[D * D];
  __shared__ float sB[D];
  __shared__ float sBp[D];
  __shared__ double red[3][kXfThreads / 32];
  // Programmatic dependent launch.  This kernel waits for every earlier kernel
  // before it touches anything (X may be the previous layer's output), and only
  // then lets the decode-GEMV that follows launch: that GEMV reads packed codes
  // before its own wait, which is safe because every kernel that could have
  // written them has completed by the time this wait returns, and this kernel
  // writes none.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int64_t m = blockIdx.x;
  const uint16_t* xr = X + m * d_in;
  uint16_t* orow = Xpp + m * d_in;
  // warp w takes the chunks c = w, w + 8, ... (the classes of the corr sum);
  // lane l transforms block l of the chunk.  The first chunk's activations
  // are loaded together with A and B.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nblk = d_in / 16;
  const int64_t nchunk = ceil_div(d_in, kCorrChunk);
  uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0;
  {
    const int64_t b = int64_t(warp) * (kCorrChunk / 16) + lane;
    if (warp < nchunk && b < nblk) {
      p0 = ld_global_v4(xr + 16 * b);
      p1 = ld_global_v4(xr + 16 * b + 8);
    }
  }
  if (threadIdx.x < D * D) sA[threadIdx.x] = ld_global_f32(A + threadIdx.x);
  if (threadIdx.x < D) sB[threadIdx.x] = ld_global_f32(B + threadIdx.x);
  __syncthreads();
  if (threadIdx.x < D) sBp[threadIdx.x] = shifted_offset<D>(sA + threadIdx.x * D, sB[threadIdx.x]);
  __syncthreads();

  double s_b = 0.0, s_xr = 0.0, s_xpp = 0.0;  // this class's running sums (lane 0)
  for (int64_t c = warp; c < nchunk; c += kCorrClasses) {
    const int64_t b = c * (kCorrChunk / 16) + lane;
    float sb = 0.f, sxr = 0.f, sxpp = 0.f;
    if (b < nblk) {
      uint4 u0 = p0, u1 = p1;
      if (c != warp) {
        u0 = ld_global_v4(xr + 16 * b);
        u1 = ld_global_v4(xr + 16 * b + 8);
      }
      uint32_t o[8];
      xform_block<D>(u0, u1, sA, sBp, o, sb, sxr, sxpp);
      uint4* dst = reinterpret_cast<uint4*>(orow + 16 * b);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    const double tb = chunk_tree_sum(double(sb));
    const double txr = chunk_tree_sum(double(sxr));
    const double txpp = chunk_tree_sum(double(sxpp));
    if (lane == 0) {
      s_b += tb;
      s_xr += txr;
      s_xpp += txpp;
    }
  }
  static_assert(kXfThreads / 32 == kCorrClasses, "one warp per chunk class");
  if (lane == 0) {
    red[0][warp] = s_b;
    red[1][warp] = s_xr;
    red[2][warp] = s_xpp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0, c = 0.0;
    for (int w = 0; w < kCorrClasses; ++w) {
      a += red[0][w];
      b += red[1][w];
      c += red[2][w];
    }
    corr[m] = static_cast<float>(a - 1.5 * b - 128.0 * c);
  }
}

// ---------------------------------------------------------------------------
// The int8-digit form of X' for few tokens (the decode-GEMV's int8 path).
//
// Per row m and chunk class r (the chunks c = r, r + 8, ... of 512 positions,
// warp r's share), X' = x A (fp32, the same fused multiply-adds as the bf16
// form) is scaled by a power of two chosen from the class's largest |X'|:
//     s_{m,r} = 2^k, the largest with max |X'| s <= 32639,
// rounded to integers q = rint(X' s) (|q| <= 32639) and split into two signed
// byte digits q = 256 hi + lo with hi = (q + 128) >> 8, lo = q - 256 hi, both in
// [-128, 127].  The GEMV multiplies the raw codes z (u8) with the digits on the
// integer tensor-core MMA, exactly: sum_k q_k z_k = 256 sum hi z + sum lo z per
// class.  Then
//     Y = sum_k (q_k / s_k) (z_k - 3/2) + s' = sum_r (sum_{k in r} q_k z_k) / s_r + corr,
//     corr = s' - 3/2 sum_r (sum_{k in r} q_k) / s_r,
// with s' = sum_g x_g . B' summed in the order of the bf16 form and the q sums
// exact; inv_s[m][r] = 1/s_{m,r} (exact).  A class with no finite largest
// |X'| (non-finite activations) gives corr = NaN.
// Layout per row: 2 d_in bytes; chunk c (512 positions, n_c = min(512,
// d_in - 512 c) of them) at byte 1024 c holds the hi plane (n_c bytes), then
// the lo plane (n_c bytes).  Within each 16-position block byte 4 p + i holds
// position 4 i + p, the order in which the GEMV's decoder extracts codes from
// a 32-bit code word (shift by 2 p, mask each byte).
constexpr int kI8Max = 32639;  // 127 * 256 + 127

constexpr int kI8Keep = 4;  // chunks per warp whose X' stays in registers between the passes

template <int D, int kItems>
__global__ void __launch_bounds__(kXfThreads)
    xform_i8_kernel(const __grid_constant__ XformGroup<kItems> grp) {
  const XformItem& it = grp.item[blockIdx.y];
  // X, A and B may come from the kernel just before this one: ld_global_*
  const uint16_t* X = it.X;
  const float* A = it.A;
  const float* B = it.B;
  const int64_t d_in = it.d_in;
  __shared__ float sA[D * D];
  __shared__ float sB[D];
  __shared__ float sBp[D];
  __shared__ double red[2][kXfThreads / 32];
  // programmatic dependent launch: as xform_kernel
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int64_t m = blockIdx.x;
  const uint16_t* xr = X + m * d_in;
  uint8_t* orow = reinterpret_cast<uint8_t*>(it.Xpp) + m * 2 * d_in;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nblk = d_in / 16;
  const int64_t nchunk = ceil_div(d_in, kCorrChunk);
  // warp w takes the chunks c = w, w + 8, ...; lane l block l of a chunk.  The
  // activations of the warp's first kI8Keep chunks load together with A and B.
  auto block_of = [&](int64_t c) { return c * (kCorrChunk / 16) + lane; };
  uint4 xin[kI8Keep][2];
#pragma unroll
  for (int ci = 0; ci < kI8Keep; ++ci) {
    const int64_t c = warp + int64_t(kCorrClasses) * ci, b = block_of(c);
    xin[ci][0] = xin[ci][1] = make_uint4(0, 0, 0, 0);
    if (c < nchunk && b < nblk) {
      xin[ci][0] = ld_global_v4(xr + 16 * b);
      xin[ci][1] = ld_global_v4(xr + 16 * b + 8);
    }
  }
  if (threadIdx.x < D * D) sA[threadIdx.x] = ld_global_f32(A + threadIdx.x);
  if (threadIdx.x < D) sB[threadIdx.x] = ld_global_f32(B + threadIdx.x);
  __syncthreads();
  if (threadIdx.x < D) sBp[threadIdx.x] = shifted_offset<D>(sA + threadIdx.x * D, sB[threadIdx.x]);
  __syncthreads();

  // pass 1: X' (kept in registers for the first kI8Keep chunks) and the
  // class's largest |X'| (NaN propagates through the comparisons)
  float xk[kI8Keep][16], sbk[kI8Keep];
  float mx = 0.f;
  auto take_max = [&](const float (&xp)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float a = fabsf(xp[e]);
      mx = (a > mx || a != a) ? a : mx;
    }
  };
#pragma unroll
  for (int ci = 0; ci < kI8Keep; ++ci) {
    const int64_t c = warp + int64_t(kCorrClasses) * ci;
    sbk[ci] = 0.f;
    if (c < nchunk && block_of(c) < nblk) {
      xprime_block<D>(xin[ci][0], xin[ci][1], sA, sBp, xk[ci], sbk[ci]);
      take_max(xk[ci]);
    }
  }
  for (int64_t c = warp + int64_t(kCorrClasses) * kI8Keep; c < nchunk; c += kCorrClasses) {
    const int64_t b = block_of(c);
    if (b < nblk) {
      float xp[16], sb;
      xprime_block<D>(ld_global_v4(xr + 16 * b), ld_global_v4(xr + 16 * b + 8), sA, sBp, xp, sb);
      take_max(xp);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, mx, off);
    mx = (o > mx || o != o) ? o : mx;
  }
  // s = 2^k, the largest with mx s <= 32639 (from the exponent bits; k = 0 for
  // an empty class, sc = 0 marks a non-finite one)
  int k = 0;
  const bool finite = mx <= 3.402823466e38f;
  if (finite && mx > 0.f) {
    const uint32_t bits = __float_as_uint(mx);
    const int e = bits >= 0x00800000u ? int(bits >> 23) - 127 : -127;  // subnormal: below 2^-126
    k = 14 - e;  // mx 2^k in [2^14, 2^15) for a normal mx
    if (k > 126) k = 126;
    if (mx * __uint_as_float(uint32_t(k + 127) << 23) > float(kI8Max)) --k;
  }
  const float sc = finite ? __uint_as_float(uint32_t(k + 127) << 23) : 0.f;
  const float inv = __uint_as_float(uint32_t(127 - k) << 23);
  if (lane == 0) it.inv_s[m * kCorrClasses + warp] = inv;

  // pass 2: digits, and the parts of corr (s' in the order of xform_kernel;
  // sum q exactly)
  double s_b = 0.0, s_q = 0.0;  // this class's running sums (lane 0)
  auto emit = [&](int64_t c, const float (&xp)[16], float sb) {
    int qsum = 0;
    if (block_of(c) < nblk) {
      uint32_t wh[4] = {0, 0, 0, 0}, wl[4] = {0, 0, 0, 0};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int q = sc > 0.f ? __float2int_rn(xp[e] * sc) : 0;
        const int h = (q + 128) >> 8;
        const int l = q - h * 256;
        qsum += q;
        const int p = e & 3, i = e >> 2;  // position e = 4 i + p -> byte 4 p + i
        wh[p] |= (uint32_t(h) & 0xFFu) << (8 * i);
        wl[p] |= (uint32_t(l) & 0xFFu) << (8 * i);
      }
      const int64_t nc = d_in - c * kCorrChunk < kCorrChunk ? d_in - c * kCorrChunk : kCorrChunk;
      uint8_t* dst = orow + c * 2 * kCorrChunk + 16 * lane;
      *reinterpret_cast<uint4*>(dst) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
      *reinterpret_cast<uint4*>(dst + nc) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    }
    const double tb = chunk_tree_sum(double(sb));
    const double tq = chunk_tree_sum(double(qsum));
    if (lane == 0) {
      s_b += tb;
      s_q += tq;
    }
  };
#pragma unroll
  for (int ci = 0; ci < kI8Keep; ++ci) {
    const int64_t c = warp + int64_t(kCorrClasses) * ci;
    if (c < nchunk) emit(c, xk[ci], sbk[ci]);
  }
  for (int64_t c = warp + int64_t(kCorrClasses) * kI8Keep; c < nchunk; c += kCorrClasses) {
    const int64_t b = block_of(c);
    float xp[16], sb = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) xp[e] = 0.f;
    if (b < nblk)
      xprime_block<D>(ld_global_v4(xr + 16 * b), ld_global_v4(xr + 16 * b + 8), sA, sBp, xp, sb);
    emit(c, xp, sb);
  }
  if (lane == 0) {
    red[0][warp] = s_b;
    red[1][warp] = finite ? s_q * double(inv) : __longlong_as_double(0x7FF8000000000000LL);  // exact
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // the class parts in class order
    double a = 0.0, q = 0.0;
    for (int w = 0; w < kCorrClasses; ++w) {
      a += red[0][w];
      q += red[1][w];
    }
    it.corr[m] = static_cast<float>(a - 1.5 * q);
  }
}

namespace {
template <int kItems>
cudaError_t launch_xform_group(const XformGroup<kItems>& grp, int count, int64_t M, int d,
                               bool i8, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M), static_cast<unsigned>(count), 1);
  cfg.blockDim = dim3(kXfThreads, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (i8) {
    switch (d) {
      case 1: return cudaLaunchKernelEx(&cfg, xform_i8_kernel<1, kItems>, grp);
      case 2: return cudaLaunchKernelEx(&cfg, xform_i8_kernel<2, kItems>, grp);
      case 4: return cudaLaunchKernelEx(&cfg, xform_i8_kernel<4, kItems>, grp);
      default: return cudaLaunchKernelEx(&cfg, xform_i8_kernel<8, kItems>, grp);
    }
  }
  switch (d) {
    case 1: return cudaLaunchKernelEx(&cfg, xform_kernel<1, kItems>, grp);
    case 2: return cudaLaunchKernelEx(&cfg, xform_kernel<2, kItems>, grp);
    case 4: return cudaLaunchKernelEx(&cfg, xform_kernel<4, kItems>, grp);
    default: return cudaLaunchKernelEx(&cfg, xform_kernel<8, kItems>, grp);
  }
}
}  // namespace

cudaError_t launch_xform(const uint16_t* X, int64_t M, int64_t d_in, int d, const float* A,
                         const float* B, uint16_t* Xpp, float* corr, cudaStream_t s,
                         int* launches) {
  XformGroup<1> grp{};
  grp.item[0] = XformItem{X, A, B, Xpp, corr, nullptr, d_in};
  cudaError_t e = launch_xform_group(grp, 1, M, d, false, s);
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_xform_i8(const uint16_t* X, int64_t M, int64_t d_in, int d, const float* A,
                            const float* B, uint8_t* X8, float* corr, float* inv_s, cudaStream_t s,
                            int* launches) {
  XformGroup<1> grp{};
  grp.item[0] = XformItem{X, A, B, reinterpret_cast<uint16_t*>(X8), corr, inv_s, d_in};
  cudaError_t e = launch_xform_group(grp, 1, M, d, true, s);
  ++*launches;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_xform_grouped(const XformJob* jobs, int count, int64_t M, int d,
                                 cudaStream_t s, int* launches) {
  for (int first = 0; first < count; first += kMaxGroupItems) {
    const int n = count - first < kMaxGroupItems ? count - first : kMaxGroupItems;
    XformGroup<kMaxGroupItems> grp{};
    for (int i = 0; i < n; ++i) {
      const XformJob& j = jobs[first + i];
      grp.item[i] = XformItem{j.X, j.A, j.B, j.Xpp, j.corr, j.inv_s, j.d_in};
    }
    cudaError_t e = launch_xform_group(grp, n, M, d, jobs[first].inv_s != nullptr, s);
    ++*launches;
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// r[m] = sum_n dY[m][n]: the rank-1 term of the dX epilogue (the B part of
// W~ = A z + B contributes B_i r[m] to dX[m][g d + i]).
__global__ void __launch_bounds__(256) rowsum_kernel(const uint16_t* __restrict__ dY, int64_t n,
                                                     float* __restrict__ r) {
  __shared__ double red[8];
  const uint16_t* row = dY + int64_t(blockIdx.x) * n;
  double s = 0.0;
  for (int64_t j = threadIdx.x * 8; j < n; j += 256 * 8) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + j));
    s += double(bf16_lo(u.x)) + double(bf16_hi(u.x)) + double(bf16_lo(u.y)) + double(bf16_hi(u.y)) +
         double(bf16_lo(u.z)) + double(bf16_hi(u.z)) + double(bf16_lo(u.w)) + double(bf16_hi(u.w));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_down_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    r[blockIdx.x] = static_cast<float>(t);
  }
}

cudaError_t launch_rowsum(const uint16_t* dY, int64_t M, int64_t n, float* r, cudaStream_t s,
                          int* launches) {
  rowsum_kernel<<<static_cast<unsigned>(M), 256, 0, s>>>(dY, n, r);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace lcvq

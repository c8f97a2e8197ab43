// C ABI of liblcvq: argument validation, workspace layout and dispatch.
// Every entry point validates all of its arguments before it launches
// anything, so a failing call has no side effect.
#include <atomic>
#include <cmath>
#include <vector>
#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"
#include "internal.h"
#include "trace.h"

using namespace lcvq;

namespace lcvq {

cudaError_t set_max_dynamic_smem(const void* func, size_t bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;  // (function, device) already raised
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({func, dev})) return cudaSuccess;
  // raise to the device maximum once, so any size up to it needs no further call
  int max_optin = 0;
  if (cudaError_t e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
      e != cudaSuccess)
    return e;
  if (bytes > size_t(max_optin)) return cudaErrorInvalidValue;
  cudaFuncAttributes fa{};
  if (cudaError_t e = cudaFuncGetAttributes(&fa, func); e != cudaSuccess) return e;
  const int dyn_max = max_optin - static_cast<int>(fa.sharedSizeBytes);
  if (cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max);
      e != cudaSuccess)
    return e;
  done.insert({func, dev});
  return cudaSuccess;
}

}  // namespace lcvq

namespace {

thread_local int g_last_launches = 0;

}  // namespace

namespace lcvq {
void set_last_launches(int n) { g_last_launches = n; }
}  // namespace lcvq

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other

lcvq_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LCVQ_ERR_UNSUPPORTED;
  int v = g_dev_ok[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return LCVQ_ERR_CUDA;
    v = (major == 10 && minor == 0) ? 1 : 2;
    g_dev_ok[dev].store(v, std::memory_order_relaxed);
  }
  return v == 1 ? LCVQ_OK : LCVQ_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
constexpr int64_t kMaxGemmDim = int64_t(1) << 30;
constexpr int64_t kMaxLdlqDim = int64_t(1) << 20;  // U is d_in^2 floats
constexpr int64_t kMaxFitHDin = int64_t(1) << 16;  // the Gram is ~12 d_in^2 bytes
constexpr int64_t kMaxFitHDout = int64_t(1) << 20; // integer code sums stay exact in fp32
bool valid_d(int d) { return d == 1 || d == 2 || d == 4 || d == 8; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- workspace layouts ----
struct GemmWs {
  size_t xpp_off, corr_off, total;
};
GemmWs gemm_ws(lcvq_dtype dtype, int64_t M, int64_t d_in) {
  GemmWs w{};
  size_t off = kWsHeaderBytes;
  if (dtype == LCVQ_BF16) {
    w.xpp_off = off;
    off = round_up(off + size_t(M) * size_t(d_in) * 2, 256);
    w.corr_off = off;  // corr [M], then the int8 path's inv_s [M][8]
    off = round_up(off + size_t(M) * 36, 256);
  }
  w.total = off;
  return w;
}
struct BwdWs {
  size_t rsum_off, part_off, num_parts, total;
};
BwdWs bwd_ws(int64_t M, int64_t d_out, int64_t d_in, int d) {
  BwdWs w{};
  const int64_t simt_parts = simt_dw_num_tiles(d_out, d_in);
  const int64_t tc_parts = kNumSMsB200 * 2;  // >= any persistent grid on one device
  w.num_parts = size_t(simt_parts > tc_parts ? simt_parts : tc_parts);
  w.rsum_off = kWsHeaderBytes;
  w.part_off = round_up(w.rsum_off + size_t(M) * 4, 256);
  w.total = round_up(w.part_off + w.num_parts * size_t(d * d + d) * 4, 256);
  return w;
}

lcvq_status finish(cudaError_t e, int launches) {
  if (e != cudaSuccess) return LCVQ_ERR_CUDA;
  g_last_launches = launches;
  return LCVQ_OK;
}

}  // namespace

extern "C" {

const char* lcvq_status_string(lcvq_status s) {
  switch (s) {
    case LCVQ_OK: return "LCVQ_OK";
    case LCVQ_ERR_INVALID_ARG: return "LCVQ_ERR_INVALID_ARG";
    case LCVQ_ERR_UNSUPPORTED: return "LCVQ_ERR_UNSUPPORTED";
    case LCVQ_ERR_ALIGNMENT: return "LCVQ_ERR_ALIGNMENT";
    case LCVQ_ERR_WORKSPACE: return "LCVQ_ERR_WORKSPACE";
    case LCVQ_ERR_CUDA: return "LCVQ_ERR_CUDA";
    case LCVQ_ERR_DEVICE_TIMEOUT: return "LCVQ_ERR_DEVICE_TIMEOUT";
  }
  return "LCVQ_ERR_UNKNOWN";
}

int lcvq_last_launch_count(void) { return g_last_launches; }

lcvq_status lcvq_assign_pack(const float* Wp, int64_t d_out, int64_t d_in, int d,
                             uint8_t* packed, uint8_t* mask_bits, void* stream) {
  LCVQ_API_RANGE();
  if (d_out < 0 || d_in < 0 || !valid_d(d)) return LCVQ_ERR_INVALID_ARG;
  if (d_in % 8 != 0 || d_in % d != 0) return LCVQ_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d_out == 0 || d_in == 0) return LCVQ_OK;
  if (Wp == nullptr || packed == nullptr) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(Wp) || !aligned16(packed) || (mask_bits && !aligned16(mask_bits)))
    return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  cudaError_t e = launch_assign_pack(Wp, d_out * d_in, packed, mask_bits,
                                     static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

lcvq_status lcvq_decode(const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                        const float* A, const float* B, void* W, lcvq_dtype w_dtype,
                        void* stream) {
  LCVQ_API_RANGE();
  if (d_out < 0 || d_in < 0 || !valid_d(d)) return LCVQ_ERR_INVALID_ARG;
  if (d_in % 16 != 0) return LCVQ_ERR_INVALID_ARG;
  if (w_dtype != LCVQ_F32 && w_dtype != LCVQ_BF16) return LCVQ_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d_out == 0 || d_in == 0) return LCVQ_OK;
  if (!packed || !A || !B || !W) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(W) || !aligned16(A) || !aligned16(B))
    return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  cudaError_t e = launch_decode(packed, d_out, d_in, d, A, B, W, w_dtype == LCVQ_BF16,
                                static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

size_t lcvq_workspace_size(lcvq_op op, lcvq_dtype dtype, int64_t M, int64_t d_out, int64_t d_in,
                           int d) {
  if (M < 0 || d_out < 0 || d_in < 0 || !valid_d(d)) return 0;
  if (dtype != LCVQ_F32 && dtype != LCVQ_BF16) return 0;
  if (op == LCVQ_OP_GEMM) return gemm_ws(dtype, M, d_in).total;
  if (op == LCVQ_OP_GEMM_BACKWARD) return bwd_ws(M, d_out, d_in, d).total;
  if (op == LCVQ_OP_FIT_AFFINE) return kWsHeaderBytes + fit_partials_bytes(d_out, d_in, d);
  if (op == LCVQ_OP_ASSIGN_LDLQ) return kWsHeaderBytes + ldlq_workspace_bytes(d_out, d_in);
  if (op == LCVQ_OP_FIT_AFFINE_H) return kWsHeaderBytes + fith_scratch_bytes(d_out, d_in, d);
  return 0;
}

lcvq_status lcvq_fit_affine_h(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                              int d, const float* H, float* A, float* B, void* workspace,
                              size_t ws_bytes, void* stream) {
  LCVQ_API_RANGE();
  g_last_launches = 0;
  if (d_out < 0 || d_in < 0 || !valid_d(d) || d_in % 64 != 0) return LCVQ_ERR_INVALID_ARG;
  if (d_in > kMaxFitHDin || d_out > kMaxFitHDout) return LCVQ_ERR_INVALID_ARG;
  if (!A || !B || !workspace) return LCVQ_ERR_INVALID_ARG;
  const bool empty = d_out == 0 || d_in == 0;
  if (!empty && (!W0 || !packed || !H)) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(workspace) || !aligned16(A) || !aligned16(B) ||
      (!empty && (!aligned16(W0) || !aligned16(packed) || !aligned16(H))))
    return LCVQ_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeaderBytes + fith_scratch_bytes(d_out, d_in, d)) return LCVQ_ERR_WORKSPACE;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = launch_fit_affine_h(W0, packed, empty ? 0 : d_out, empty ? 0 : d_in, d, H, A, B,
                                      ws + kWsHeaderBytes, reinterpret_cast<unsigned int*>(ws),
                                      static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

lcvq_status lcvq_assign_ldlq(const float* P, const float* U, int64_t d_out, int64_t d_in, int d,
                             uint8_t* packed, void* workspace, size_t ws_bytes, void* stream) {
  LCVQ_API_RANGE();
  g_last_launches = 0;
  if (d_out < 0 || d_in < 0 || !valid_d(d)) return LCVQ_ERR_INVALID_ARG;
  if (d_in % 64 != 0 || d_in % d != 0 || d_in > kMaxLdlqDim || d_out > kMaxGemmDim)
    return LCVQ_ERR_INVALID_ARG;
  if (!workspace) return LCVQ_ERR_INVALID_ARG;
  if (d_out == 0 || d_in == 0) return LCVQ_OK;
  if (!P || !U || !packed) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(P) || !aligned16(U) || !aligned16(packed) || !aligned16(workspace))
    return LCVQ_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeaderBytes + ldlq_workspace_bytes(d_out, d_in)) return LCVQ_ERR_WORKSPACE;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = launch_ldlq(P, U, d_out, d_in, packed, reinterpret_cast<float*>(ws + kWsHeaderBytes),
                              reinterpret_cast<unsigned int*>(ws), static_cast<cudaStream_t>(stream),
                              &launches);
  return finish(e, launches);
}

lcvq_status lcvq_dge_scale(float* dWp, const float* Wp, int64_t n, float k, void* stream) {
  LCVQ_API_RANGE();
  g_last_launches = 0;
  if (n < 0 || n % 4 != 0 || !(k > 0.f) || !std::isfinite(k)) return LCVQ_ERR_INVALID_ARG;
  if (n == 0) return LCVQ_OK;
  if (!dWp || !Wp) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(dWp) || !aligned16(Wp)) return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  cudaError_t e = launch_dge_scale(dWp, Wp, n, k, static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

lcvq_status lcvq_fit_affine(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                            int d, const float* h, float* A, float* B, void* workspace,
                            size_t ws_bytes, void* stream) {
  LCVQ_API_RANGE();
  g_last_launches = 0;
  if (d_out < 0 || d_in < 0 || !valid_d(d) || d_in % 16 != 0) return LCVQ_ERR_INVALID_ARG;
  if (!A || !B || !workspace) return LCVQ_ERR_INVALID_ARG;
  const bool empty = d_out == 0 || d_in == 0;
  if (!empty && (!W0 || !packed)) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(workspace) || (!empty && (!aligned16(W0) || !aligned16(packed))) ||
      (h && !aligned16(h)))
    return LCVQ_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeaderBytes + fit_partials_bytes(d_out, d_in, d)) return LCVQ_ERR_WORKSPACE;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  double* partials = reinterpret_cast<double*>(static_cast<char*>(workspace) + kWsHeaderBytes);
  cudaError_t e = launch_fit_affine(W0, packed, empty ? 0 : d_out, empty ? 0 : d_in, d, h, A, B,
                                    partials, static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

static lcvq_status validate_gemm_shapes(lcvq_dtype dtype, int64_t M, int64_t d_out, int64_t d_in,
                                        int d) {
  if (M < 0 || d_out < 0 || d_in < 0 || !valid_d(d)) return LCVQ_ERR_INVALID_ARG;
  if (dtype != LCVQ_F32 && dtype != LCVQ_BF16) return LCVQ_ERR_INVALID_ARG;
  if (d_in % 64 != 0 || d_out % 8 != 0) return LCVQ_ERR_INVALID_ARG;
  // the GEMV kernels index rows and columns in 32 bits
  if (M > INT32_MAX || d_out > kMaxGemmDim || d_in > kMaxGemmDim) return LCVQ_ERR_INVALID_ARG;
  return LCVQ_OK;
}

lcvq_status lcvq_gemm(const void* X, lcvq_dtype dtype, int64_t M, const uint8_t* packed,
                      int64_t d_out, int64_t d_in, int d, const float* A, const float* B,
                      void* Y, lcvq_form form, void* workspace, size_t ws_bytes, void* stream) {
  LCVQ_API_RANGE();
  if (lcvq_status st = validate_gemm_shapes(dtype, M, d_out, d_in, d); st != LCVQ_OK) return st;
  if (form != LCVQ_FORM_AUTO && form != LCVQ_FORM_DECODE && form != LCVQ_FORM_ALGEBRAIC)
    return LCVQ_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (M == 0 || d_out == 0) return LCVQ_OK;
  if (!Y) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(Y)) return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t esz = dtype == LCVQ_BF16 ? 2 : 4;
  if (d_in == 0) {
    if (cudaMemsetAsync(Y, 0, size_t(M) * size_t(d_out) * esz, s) != cudaSuccess)
      return LCVQ_ERR_CUDA;
    return LCVQ_OK;
  }
  if (!X || !packed || !A || !B || !workspace) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(packed) || !aligned16(A) || !aligned16(B) ||
      !aligned16(workspace))
    return LCVQ_ERR_ALIGNMENT;
  const GemmWs w = gemm_ws(dtype, M, d_in);
  if (ws_bytes < w.total) return LCVQ_ERR_WORKSPACE;

  int launches = 0;
  cudaError_t e = cudaSuccess;
  char* ws = static_cast<char*>(workspace);
  unsigned int* err = reinterpret_cast<unsigned int*>(ws);
  if (dtype == LCVQ_BF16 && M <= kI8MaxM) {
    // few tokens: the int8 path (X' as two signed byte digits per position,
    // the integer tensor-core MMA, exact integer sums per chunk class)
    uint8_t* X8 = reinterpret_cast<uint8_t*>(ws + w.xpp_off);
    float* corr = reinterpret_cast<float*>(ws + w.corr_off);
    float* inv_s = corr + M;
    e = launch_xform_i8(static_cast<const uint16_t*>(X), M, d_in, d, A, B, X8, corr, inv_s, s,
                        &launches);
    if (e == cudaSuccess)
      e = launch_gemv(reinterpret_cast<const uint16_t*>(X8), corr, M, packed, d_out, d_in,
                      static_cast<uint16_t*>(Y), true, s, &launches, inv_s);
  } else if (dtype == LCVQ_BF16 && (M <= 32 || form != LCVQ_FORM_DECODE)) {
    uint16_t* Xpp = reinterpret_cast<uint16_t*>(ws + w.xpp_off);
    float* corr = reinterpret_cast<float*>(ws + w.corr_off);
    e = launch_xform(static_cast<const uint16_t*>(X), M, d_in, d, A, B, Xpp, corr, s, &launches);
    if (e == cudaSuccess)
      e = launch_gemm_xformed(Xpp, corr, M, packed, d_out, d_in, static_cast<uint16_t*>(Y), err,
                              true, s, &launches);
  } else if (dtype == LCVQ_BF16) {  // decode form on the tensor cores
    e = launch_tc_forward(static_cast<const uint16_t*>(X), false, nullptr, M, packed, d_out, d_in,
                          d, A, B, static_cast<uint16_t*>(Y), err, s, &launches);
  } else {
    e = launch_simt_forward(X, dtype == LCVQ_BF16, M, packed, d_out, d_in, d, A, B, Y, s,
                            &launches);
  }
  return finish(e, launches);
}

}  // extern "C"

namespace {

constexpr int64_t kGroupMaxDim = int64_t(1) << 28;

// byte offsets of item i's X'' and corr in a grouped workspace; total bytes
// (0 if any item is invalid)
size_t grouped_ws(const lcvq_gemm_item* items, int count, int64_t M, int d,
                  std::vector<size_t>* xpp_off, std::vector<size_t>* corr_off) {
  if (items == nullptr || count < 1 || M < 1 || M > 32 || !valid_d(d)) return 0;
  size_t off = kWsHeaderBytes;
  for (int i = 0; i < count; ++i) {
    const lcvq_gemm_item& it = items[i];
    if (it.d_out < 1 || it.d_in < 1 || it.d_out >= kGroupMaxDim || it.d_in >= kGroupMaxDim ||
        it.d_in % 64 != 0 || it.d_out % 8 != 0)
      return 0;
    if (xpp_off) xpp_off->push_back(off);
    off = round_up(off + size_t(M) * size_t(it.d_in) * 2, 256);
    if (corr_off) corr_off->push_back(off);
    off = round_up(off + size_t(M) * 36, 256);  // corr [M], then the int8 path's inv_s [M][8]
  }
  return off;
}

}  // namespace

extern "C" {

size_t lcvq_workspace_size_grouped(const lcvq_gemm_item* items, int count, int64_t M, int d) {
  return grouped_ws(items, count, M, d, nullptr, nullptr);
}

lcvq_status lcvq_gemm_grouped(const lcvq_gemm_item* items, int count, int64_t M, int d,
                              void* workspace, size_t ws_bytes, void* stream) {
  LCVQ_API_RANGE();
  g_last_launches = 0;
  std::vector<size_t> xoff, coff;
  const size_t need = grouped_ws(items, count, M, d, &xoff, &coff);
  if (need == 0) return LCVQ_ERR_INVALID_ARG;
  if (!workspace) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return LCVQ_ERR_ALIGNMENT;
  if (ws_bytes < need) return LCVQ_ERR_WORKSPACE;
  for (int i = 0; i < count; ++i) {
    const lcvq_gemm_item& it = items[i];
    if (!it.X || !it.packed || !it.A || !it.B || !it.Y) return LCVQ_ERR_INVALID_ARG;
    if (!aligned16(it.X) || !aligned16(it.packed) || !aligned16(it.A) || !aligned16(it.B) ||
        !aligned16(it.Y))
      return LCVQ_ERR_ALIGNMENT;
  }
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  std::vector<XformJob> xj(count);
  std::vector<GemvJob> gj(count);
  for (int i = 0; i < count; ++i) {
    const lcvq_gemm_item& it = items[i];
    uint16_t* Xpp = reinterpret_cast<uint16_t*>(ws + xoff[i]);
    float* corr = reinterpret_cast<float*>(ws + coff[i]);
    float* inv_s = M <= kI8MaxM ? corr + M : nullptr;  // set: the int8 path, as lcvq_gemm
    xj[i] = XformJob{static_cast<const uint16_t*>(it.X), it.A, it.B, Xpp, corr, it.d_in, inv_s};
    gj[i] = GemvJob{it.packed, Xpp, corr, static_cast<uint16_t*>(it.Y), it.d_out, it.d_in, inv_s};
  }
  int launches = 0;
  // per chunk of matrices: their X-transforms, then their decode-GEMV
  cudaError_t e = cudaSuccess;
  for (int first = 0; first < count && e == cudaSuccess; first += kMaxGroupItems) {
    const int n = count - first < kMaxGroupItems ? count - first : kMaxGroupItems;
    e = launch_xform_grouped(xj.data() + first, n, M, d, s, &launches);
    if (e == cudaSuccess)
      e = launch_gemv_grouped(gj.data() + first, n, M, s, &launches,
                              reinterpret_cast<unsigned int*>(ws));
  }
  return finish(e, launches);
}

lcvq_status lcvq_xform(const void* X, lcvq_dtype dtype, int64_t M, int64_t d_in, int d,
                       const float* A, const float* B, void* Xpp, float* corr, void* stream) {
  LCVQ_API_RANGE();
  if (lcvq_status st = validate_gemm_shapes(dtype, M, 8, d_in, d); st != LCVQ_OK) return st;
  if (dtype != LCVQ_BF16) return LCVQ_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (M == 0 || d_in == 0) return LCVQ_OK;
  if (!X || !A || !B || !Xpp || !corr) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Xpp) || !aligned16(corr))
    return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  cudaError_t e = launch_xform(static_cast<const uint16_t*>(X), M, d_in, d, A, B,
                               static_cast<uint16_t*>(Xpp), corr,
                               static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

lcvq_status lcvq_gemm_xformed(const void* Xpp, const float* corr, int64_t M,
                              const uint8_t* packed, int64_t d_out, int64_t d_in, void* Y,
                              void* stream) {
  LCVQ_API_RANGE();
  if (lcvq_status st = validate_gemm_shapes(LCVQ_BF16, M, d_out, d_in, 8); st != LCVQ_OK) return st;
  g_last_launches = 0;
  if (M == 0 || d_out == 0) return LCVQ_OK;
  if (!Xpp || !corr || !packed || !Y) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(Xpp) || !aligned16(corr) || !aligned16(packed) || !aligned16(Y))
    return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  int launches = 0;
  // launched on its own: whatever ran before may have written the codes
  cudaError_t e = launch_gemm_xformed(static_cast<const uint16_t*>(Xpp), corr, M, packed, d_out,
                                      d_in, static_cast<uint16_t*>(Y), nullptr, false,
                                      static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

lcvq_status lcvq_gemm_backward(const void* X, const void* dY, lcvq_dtype dtype, int64_t M,
                               const uint8_t* packed, const uint8_t* mask_bits, int64_t d_out,
                               int64_t d_in, int d, const float* A, const float* B, void* dX,
                               float* dA, float* dB, float* dWp, void* workspace,
                               size_t ws_bytes, void* stream) {
  LCVQ_API_RANGE();
  if (lcvq_status st = validate_gemm_shapes(dtype, M, d_out, d_in, d); st != LCVQ_OK) return st;
  g_last_launches = 0;
  if (!dA || !dB) return LCVQ_ERR_INVALID_ARG;
  if (dWp != nullptr && mask_bits == nullptr) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(dA) || !aligned16(dB) || (dWp && !aligned16(dWp)) || (dX && !aligned16(dX)) ||
      (mask_bits && !aligned16(mask_bits)))
    return LCVQ_ERR_ALIGNMENT;
  if (lcvq_status st = check_device(); st != LCVQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t esz = dtype == LCVQ_BF16 ? 2 : 4;
  if (M == 0 || d_out == 0 || d_in == 0) {
    // no tokens / no weights: all gradients are empty sums
    if (cudaMemsetAsync(dA, 0, size_t(d) * d * 4, s) != cudaSuccess) return LCVQ_ERR_CUDA;
    if (cudaMemsetAsync(dB, 0, size_t(d) * 4, s) != cudaSuccess) return LCVQ_ERR_CUDA;
    if (dWp && d_out > 0 && d_in > 0 &&
        cudaMemsetAsync(dWp, 0, size_t(d_out) * size_t(d_in) * 4, s) != cudaSuccess)
      return LCVQ_ERR_CUDA;
    if (dX && M > 0 && d_in > 0 &&
        cudaMemsetAsync(dX, 0, size_t(M) * size_t(d_in) * esz, s) != cudaSuccess)
      return LCVQ_ERR_CUDA;
    return LCVQ_OK;
  }
  if (!X || !dY || !packed || !A || !B || !workspace) return LCVQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(packed) || !aligned16(A) || !aligned16(B) ||
      !aligned16(workspace))
    return LCVQ_ERR_ALIGNMENT;
  const BwdWs w = bwd_ws(M, d_out, d_in, d);
  if (ws_bytes < w.total) return LCVQ_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  unsigned int* err = reinterpret_cast<unsigned int*>(ws);
  float* partials = reinterpret_cast<float*>(ws + w.part_off);
  int launches = 0;
  cudaError_t e = cudaSuccess;
  int64_t parts = 0;
  if (dtype == LCVQ_BF16) {
    float* rsum = reinterpret_cast<float*>(ws + w.rsum_off);
    const uint16_t* dYb = static_cast<const uint16_t*>(dY);
    if (dX) {
      e = launch_rowsum(dYb, M, d_out, rsum, s, &launches);
      if (e == cudaSuccess)
        e = launch_tc_backward_dx(dYb, rsum, M, packed, d_out, d_in, d, A, B,
                                  static_cast<uint16_t*>(dX), err, s, &launches);
    }
    int grid = 0;
    if (e == cudaSuccess)
      e = launch_tc_backward_dw(static_cast<const uint16_t*>(X), dYb, M, packed, mask_bits, d_out,
                                d_in, d, A, dWp, partials, &grid, err, s, &launches);
    parts = grid;
  } else {
    if (dX) e = launch_simt_backward_dx(dY, false, M, packed, d_out, d_in, d, A, B, dX, s, &launches);
    if (e == cudaSuccess)
      e = launch_simt_backward_dw(X, dY, false, M, packed, mask_bits, d_out, d_in, d, A, dWp,
                                  partials, s, &launches);
    parts = simt_dw_num_tiles(d_out, d_in);
  }
  if (e == cudaSuccess) e = launch_reduce_partials(partials, parts, d, dA, dB, s, &launches);
  return finish(e, launches);
}

lcvq_status lcvq_check_device_error(void* workspace, void* stream) {
  LCVQ_API_RANGE();
  if (!workspace) return LCVQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int h[2] = {0, 0};
  if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return LCVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LCVQ_ERR_CUDA;
  if (h[0] != 0) {
    const unsigned int zero[2] = {0, 0};
    if (cudaMemcpy(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return LCVQ_ERR_CUDA;
    return h[0] == LCVQ_ERR_DEVICE_TIMEOUT ? LCVQ_ERR_DEVICE_TIMEOUT : LCVQ_ERR_CUDA;
  }
  return LCVQ_OK;
}

}  // extern "C"

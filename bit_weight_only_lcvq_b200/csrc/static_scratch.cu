// lcvq_gemv_static: the decode-GEMV (bf16, M <= 32) with no workspace argument.
//
// Some callers cannot hand the library a workspace: code that runs while a
// CUDA graph is being captured (cudaMalloc is not allowed there), runtimes
// that reserve all device memory up front and forbid later allocations, and
// bindings whose host framework owns the allocator but exposes no scratch
// API to extension code.  This entry point keeps its scratch -- the
// transformed activations X'' and the per-row constants -- in one fixed array
// in the library's own device memory instead.
//
// The array is a file-scope __device__ object of kStaticScratchBytes; every
// GPU that loads the library holds it until the process exits.  Host code may
// not use the array's name as a device address (it is a host-side shadow), so
// the first call on each device, with that device current, asks the runtime
// for the array's device address with cudaGetSymbolAddress and remembers it.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "trace.h"

namespace {

constexpr int64_t kStaticMaxM = 32;
constexpr int64_t kStaticMaxDin = 32768;
constexpr int64_t kStaticMaxDout = int64_t(1) << 30;  // the same bound as lcvq_gemm
constexpr size_t kStaticXppBytes = size_t(kStaticMaxM) * size_t(kStaticMaxDin) * 2;  // 2 MiB
constexpr size_t kStaticScratchBytes = kStaticXppBytes + 256;  // + corr [32], inv_s [<= 4][8]

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_mu;
void* g_ptr[kMaxDev] = {};

// Device address of the array on the current device (set up once per device).
lcvq_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return LCVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return LCVQ_ERR_CUDA;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return LCVQ_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" lcvq_status lcvq_gemv_static(const void* X, int64_t M, const uint8_t* packed,
                                        int64_t d_out, int64_t d_in, int d, const float* A,
                                        const float* B, void* Y, void* stream) {
  LCVQ_API_RANGE();
  lcvq::set_last_launches(0);
  if (M < 0 || d_out < 0 || d_in < 0) return LCVQ_ERR_INVALID_ARG;
  if (!(d == 1 || d == 2 || d == 4 || d == 8)) return LCVQ_ERR_INVALID_ARG;
  if (d_in % 64 != 0 || d_out % 8 != 0) return LCVQ_ERR_INVALID_ARG;
  if (d_out > kStaticMaxDout) return LCVQ_ERR_INVALID_ARG;  // rows are indexed in 32 bits
  if (M > kStaticMaxM || d_in > kStaticMaxDin) return LCVQ_ERR_WORKSPACE;  // beyond the array
  if (M == 0 || d_out == 0) return LCVQ_OK;
  if (!Y) return LCVQ_ERR_INVALID_ARG;
  if (d_in == 0)  // an empty sum: Y = 0 (a memset allocates nothing)
    return cudaMemsetAsync(Y, 0, size_t(M) * size_t(d_out) * 2, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? LCVQ_OK
               : LCVQ_ERR_CUDA;
  if (!X || !packed || !A || !B) return LCVQ_ERR_INVALID_ARG;
  if (!al16(X) || !al16(packed) || !al16(A) || !al16(B) || !al16(Y)) return LCVQ_ERR_ALIGNMENT;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return LCVQ_ERR_CUDA;
  if (major != 10 || minor != 0) return LCVQ_ERR_UNSUPPORTED;
  void* base = nullptr;
  if (lcvq_status st = static_scratch(&base); st != LCVQ_OK) return st;
  // X'' and corr are written in full by the X-transform before the GEMV reads
  // them, so nothing in the array has to start at zero.
  uint16_t* Xpp = static_cast<uint16_t*>(base);
  float* corr = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kStaticXppBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e;
  if (M <= lcvq::kI8MaxM) {  // the int8 path, as lcvq_gemm takes it
    float* inv_s = corr + kStaticMaxM;
    e = lcvq::launch_xform_i8(static_cast<const uint16_t*>(X), M, d_in, d, A, B,
                              reinterpret_cast<uint8_t*>(Xpp), corr, inv_s, s, &launches);
    if (e == cudaSuccess)
      e = lcvq::launch_gemv(Xpp, corr, M, packed, d_out, d_in, static_cast<uint16_t*>(Y), true, s,
                            &launches, inv_s);
  } else {
    e = lcvq::launch_xform(static_cast<const uint16_t*>(X), M, d_in, d, A, B, Xpp, corr, s,
                           &launches);
    if (e == cudaSuccess)
      e = lcvq::launch_gemv(Xpp, corr, M, packed, d_out, d_in, static_cast<uint16_t*>(Y), true, s,
                            &launches);
  }
  if (e != cudaSuccess) return LCVQ_ERR_CUDA;
  lcvq::set_last_launches(launches);
  return LCVQ_OK;
}

// Internal launchers behind the C ABI (host side).  Each returns the CUDA error
// of its launch(es) and adds the number of kernels it launched to *launches.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lcvq {

// cudaFuncAttributeMaxDynamicSharedMemorySize for `func` on the current device,
// set once per (function, device)
cudaError_t set_max_dynamic_smem(const void* func, size_t bytes);

// records the number of kernels the current call launched, for
// lcvq_last_launch_count() (per host thread)
void set_last_launches(int n);

// ---- elementwise ----
cudaError_t launch_assign_pack(const float* Wp, int64_t n_elems, uint8_t* packed,
                               uint8_t* mask_bits, cudaStream_t s, int* launches);
cudaError_t launch_decode(const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                          const float* A, const float* B, void* W, bool w_bf16,
                          cudaStream_t s, int* launches);

// dWp[i] *= phi_k'(Wp[i]) (the DGE factor; 0 outside [0, 3]); n % 4 == 0
cudaError_t launch_dge_scale(float* dWp, const float* Wp, int64_t n, float k, cudaStream_t s,
                             int* launches);

// ---- algebraic-form prologue (bf16 tensor-core paths) ----
// Xpp[M][d_in] bf16: X' = group-wise X A, rounded to bf16, scaled by the
// per-position power of two of the code decoder, in the decoder's K order.
// corr[M] fp32: per-row constant that turns the tensor-core accumulator into Y.
cudaError_t launch_xform(const uint16_t* X, int64_t M, int64_t d_in, int d, const float* A,
                         const float* B, uint16_t* Xpp, float* corr, cudaStream_t s,
                         int* launches);
// The int8-digit form for the decode-GEMV's int8 path (M <= kI8MaxM): per row
// and chunk class r (chunks r, r + 8, ... of 512 positions) a power-of-two
// scale s, q = rint(X' s) as two signed byte digits per position (X8
// [M][2 d_in] bytes: per chunk the hi plane, then the lo plane), inv_s[M][8] =
// 1 / s and corr[M] = s' - 3/2 sum_r (sum of class r's q) / s_r.
constexpr int64_t kI8MaxM = 4;
cudaError_t launch_xform_i8(const uint16_t* X, int64_t M, int64_t d_in, int d, const float* A,
                            const float* B, uint8_t* X8, float* corr, float* inv_s, cudaStream_t s,
                            int* launches);

// ---- decode-GEMV (bf16, M <= 32) ----
// after_xform: launched right after launch_xform of the same call on the same
// stream, so the codes may be read before the kernel's dependency wait.
// inv_s set: the int8 path on launch_xform_i8's digits (Xpp points at them).
cudaError_t launch_gemv(const uint16_t* Xpp, const float* corr, int64_t M, const uint8_t* packed,
                        int64_t d_out, int64_t d_in, uint16_t* Y, bool after_xform,
                        cudaStream_t s, int* launches, const float* inv_s = nullptr);

constexpr int kMaxGroupItems = 128;

// the X-transform of several matrices' activations (common M and d) in
// launches of up to kMaxGroupItems matrices; per matrix, the same bits as
// launch_xform.
struct XformJob {
  const uint16_t* X;
  const float* A;
  const float* B;
  uint16_t* Xpp;  // the int8 digit planes when inv_s is set
  float* corr;
  int64_t d_in;
  float* inv_s;  // null: bf16 X''; else the int8-digit form (every job of a call alike)
};

// decode-GEMV over a group of matrices with a common token count M <= 32, in
// persistent launches of up to kMaxGroupItems matrices each (X'' and corr of
// every matrix already formed by launch_xform or launch_xform_grouped).  For
// M <= 16 each matrix's Y is bit-identical to launch_gemv on that matrix
// alone; large groups with 17 <= M <= 32 run on the tcgen05 form below.
struct GemvJob {
  const uint8_t* packed;
  const uint16_t* Xpp;  // or the int8 digits
  const float* corr;
  uint16_t* Y;
  int64_t d_out, d_in;
  const float* inv_s;  // set: the int8 path (M <= kI8MaxM; every job of a call alike)
};
// err: device error word for the bounded waits of the wide-tile form
cudaError_t launch_gemv_grouped(const GemvJob* jobs, int count, int64_t M, cudaStream_t s,
                                int* launches, unsigned int* err);
cudaError_t launch_xform_grouped(const XformJob* jobs, int count, int64_t M, int d,
                                 cudaStream_t s, int* launches);
// the same on the tcgen05 tensor cores (weights in TMEM as the MMA's A
// operand, tokens as N = 32): launches of up to 48 matrices
bool gemv_tc_usable(int64_t M);
cudaError_t launch_gemv_tc_grouped(const GemvJob* jobs, int count, int64_t M, unsigned int* err,
                                   cudaStream_t s, int* launches);

// integer-code GEMM on X'' (dispatches on M: decode-GEMV for M <= 32, else
// the tcgen05 GEMM); err may be null (no device error word); after_xform as
// for launch_gemv
cudaError_t launch_gemm_xformed(const uint16_t* Xpp, const float* corr, int64_t M,
                                const uint8_t* packed, int64_t d_out, int64_t d_in, uint16_t* Y,
                                unsigned int* err, bool after_xform, cudaStream_t s,
                                int* launches);

// 2D TMA tensor map: `inner` contiguous elements per row, `outer` rows of
// `row_bytes`; box box_inner x box_outer; 128-byte swizzle or none; zero fill
// out of bounds.  False if the driver entry point is missing or rejects it.
bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                        uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                        bool swizzle128);

// ---- least-squares refit of (A, B) given the codes ----
// partials: fit_partials_bytes(d_out, d_in, d) bytes of fp64 scratch
size_t fit_partials_bytes(int64_t d_out, int64_t d_in, int d);
cudaError_t launch_fit_affine(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                              int d, const float* h, float* A, float* B, double* partials,
                              cudaStream_t s, int* launches);

// ---- least-squares refit of (A, B) under the full Hessian H ----
// scratch: fith_scratch_bytes(d_out, d_in, d) bytes (the bf16 operands, the
// fp32 Gram and the fp64 partials of the normal equations)
size_t fith_scratch_bytes(int64_t d_out, int64_t d_in, int d);
cudaError_t launch_fit_affine_h(const float* W0, const uint8_t* packed, int64_t d_out, int64_t d_in,
                                int d, const float* H, float* A, float* B, void* scratch,
                                unsigned int* err, cudaStream_t s, int* launches);

// ---- H-aware sequential code assignment ----
// E: ldlq_workspace_bytes(d_out, d_in) bytes of fp32 scratch (the errors p - z)
size_t ldlq_workspace_bytes(int64_t d_out, int64_t d_in);
cudaError_t launch_ldlq(const float* P, const float* U, int64_t d_out, int64_t d_in,
                        uint8_t* packed, float* E, unsigned int* err, cudaStream_t s,
                        int* launches);

// ---- tcgen05 GEMMs (bf16, persistent, one CTA per SM) ----
int tc_max_grid();
// Xa is X'' (algebraic, with corr) or X (decode form, A z + B decoded on chip)
cudaError_t launch_tc_forward(const uint16_t* Xa, bool algebraic, const float* corr, int64_t M,
                              const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                              const float* A, const float* B, uint16_t* Y, unsigned int* err,
                              cudaStream_t s, int* launches);
cudaError_t launch_tc_backward_dx(const uint16_t* dY, const float* rsum, int64_t M,
                                  const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                                  const float* A, const float* B, uint16_t* dX, unsigned int* err,
                                  cudaStream_t s, int* launches);
// *num_parts receives the number of per-CTA partial rows written
cudaError_t launch_tc_backward_dw(const uint16_t* X, const uint16_t* dY, int64_t M,
                                  const uint8_t* packed, const uint8_t* mask, int64_t d_out,
                                  int64_t d_in, int d, const float* A, float* dWp,
                                  float* partials, int* num_parts, unsigned int* err,
                                  cudaStream_t s, int* launches);
// C[r][c] = sum_n Q[n][r] Q[n][c] for r < cols_p, c < cols_q (fp32 out,
// [cols_p][cols_q]): the tcgen05 Gram of Q's first cols_p columns against all
// of Q (bf16 [rows][cols_q]); cols_p, cols_q multiples of 64
cudaError_t launch_tc_gram(const uint16_t* Q, int64_t rows, int64_t cols_p, int64_t cols_q,
                           float* C, unsigned int* err, cudaStream_t s, int* launches);
// r[m] = sum_n dY[m][n] (fp64 accumulation), bf16 dY
cudaError_t launch_rowsum(const uint16_t* dY, int64_t M, int64_t n, float* r, cudaStream_t s,
                          int* launches);

// ---- CUDA-core paths (any M; fp32 or bf16 activations) ----
cudaError_t launch_simt_forward(const void* X, bool bf16, int64_t M, const uint8_t* packed,
                                int64_t d_out, int64_t d_in, int d, const float* A,
                                const float* B, void* Y, cudaStream_t s, int* launches);
cudaError_t launch_simt_backward_dx(const void* dY, bool bf16, int64_t M, const uint8_t* packed,
                                    int64_t d_out, int64_t d_in, int d, const float* A,
                                    const float* B, void* dX, cudaStream_t s, int* launches);
// G = dY^T X tiles with the fused epilogue: dWp (if non-null) and per-tile
// partials of dA/dB into `partials` ([num_tiles][d*d + d] fp32).
cudaError_t launch_simt_backward_dw(const void* X, const void* dY, bool bf16, int64_t M,
                                    const uint8_t* packed, const uint8_t* mask_bits,
                                    int64_t d_out, int64_t d_in, int d, const float* A,
                                    float* dWp, float* partials, cudaStream_t s, int* launches);
int64_t simt_dw_num_tiles(int64_t d_out, int64_t d_in);

// fixed-order fp64 reduction of [num_parts][d*d + d] fp32 partials into dA, dB
cudaError_t launch_reduce_partials(const float* partials, int64_t num_parts, int d, float* dA,
                                   float* dB, cudaStream_t s, int* launches);

}  // namespace lcvq

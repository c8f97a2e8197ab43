/*
 * lcvq.h - C ABI of liblcvq: the data-parallel hot path of linear-constrained
 * vector quantization (LC-VQ) at 2 bits per weight, for NVIDIA B200 (sm_100a).
 *
 * The method (LC-QAT: Data-Efficient 2-Bit QAT for LLMs via Linear-Constrained
 * Vector Quantization; technical summary, Methodology 1 and 3):
 *   - a weight matrix is cut into d-element vectors along its input dimension;
 *   - each vector is the codeword c = A z + B of a 2-bit code z in {0,1,2,3}^d,
 *     with A (d x d) and B (d) floating-point parameters shared by the whole
 *     matrix (Methodology 1, "linear-constrained parameterization");
 *   - in QAT the float proxy weights W_p are rounded and clamped to the codes
 *     W_z, decoded as A W_z + B and used in the layer's matmul; gradients reach
 *     A, B and (straight-through the rounding) W_p (Methodology 3, "training
 *     pipeline", and the gradient-estimation ablation, which uses STE).
 *
 * Conventions (shared by every call):
 *   - Storage order: weights [d_out][d_in] row-major (the transpose of the
 *     d_in x d_out matrix W~ of decoupleQ eq. (1), Y = X W~); activations
 *     [M][d_in] and [M][d_out] row-major.  So Y[m][n] = sum_k X[m][k] W~[n][k].
 *   - Vectors are d consecutive elements along d_in: element k of row n belongs
 *     to vector k / d, position k % d.  c_i = sum_j A[i*d + j] z_j + B[i]
 *     (A row-major, acting on column vectors).
 *   - Packed codes, format V1: [d_out][d_in/4] bytes; element k of a row sits in
 *     byte k/4 at bits 2(k%4) and 2(k%4)+1 (LSB first).  For d = 8 the two bytes
 *     of one vector read as a little-endian u16 equal its codebook index
 *     sum_j z_j 4^j.
 *   - Clamp mask bits: [d_out][d_in/8] bytes, bit k%8 of byte k/8, set where
 *     0 <= W_p <= 3 (the straight-through pass region).
 *   - Rounding is round-half-to-even; NaN -> 0, +inf -> 3, -inf -> 0; NaN is
 *     outside the mask.
 *
 * Ownership and execution: every pointer is a DEVICE pointer owned by the
 * caller (except where a parameter says "host").  The library allocates no
 * device memory and never synchronizes the stream on the hot path; scratch goes
 * in a caller-provided workspace sized by lcvq_workspace_size().  All calls are
 * asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the legacy
 * default stream).  Outputs are overwritten, never accumulated into.  The
 * decode-GEMV kernels are launched with programmatic dependent launch: a
 * call's first kernel may become resident while earlier work on the stream
 * finishes, but it reads no input before that work has completed, so inputs
 * produced by any earlier kernel or copy on the stream are always seen.
 *
 * Errors: arguments are validated before anything is launched; a failing call
 * launches nothing and returns a status.  Launch failures return
 * LCVQ_ERR_CUDA.  Kernels that wait on mbarriers give up after a bounded number
 * of clock cycles and record LCVQ_ERR_DEVICE_TIMEOUT in the workspace's error
 * word, read by lcvq_check_device_error(); the other roles of the kernel then
 * wind down, copies in flight land and tensor-core work drains before the
 * kernel exits, so the next call on the workspace runs normally.  Nothing
 * aborts, throws or traps.
 *
 * Workspace header (its first 256 bytes, zeroed once by the caller):
 *   bytes 0..3   error word (0, or the first LCVQ_ERR_DEVICE_TIMEOUT)
 *   bytes 4..7   which wait gave up (a small integer naming the wait)
 *   bytes 8..15  int64 wait limit in clock cycles of the tensor-core GEMMs and
 *                the grouped decode-GEMV kernels; 0 (the default) means 2^32
 *                (about 2 s).  A caller may lower it, e.g. to test its own
 *                handling of LCVQ_ERR_DEVICE_TIMEOUT.
 *
 * Requirements: a compute capability 10.0 device (sm_100a); otherwise
 * LCVQ_ERR_UNSUPPORTED.  Pointers 16-byte aligned (LCVQ_ERR_ALIGNMENT).
 * d in {1, 2, 4, 8}.  Shape rules are listed per call.  Thread safety: calls
 * hold no global state except a per-device cache of device properties and
 * kernel attributes, guarded for concurrent first use.
 */
#ifndef LCVQ_H_
#define LCVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LCVQ_FORMAT_V1 1

#if defined(__GNUC__)
#define LCVQ_API __attribute__((visibility("default")))
#else
#define LCVQ_API
#endif

typedef enum {
  LCVQ_OK = 0,
  LCVQ_ERR_INVALID_ARG = 1,    /* null pointer, bad shape, bad enum */
  LCVQ_ERR_UNSUPPORTED = 2,    /* not an sm_100 device, or unsupported d/dtype combination */
  LCVQ_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned */
  LCVQ_ERR_WORKSPACE = 4,      /* workspace missing or smaller than lcvq_workspace_size() */
  LCVQ_ERR_CUDA = 5,           /* a CUDA runtime call or kernel launch failed */
  LCVQ_ERR_DEVICE_TIMEOUT = 6  /* a device-side bounded wait gave up (from lcvq_check_device_error) */
} lcvq_status;

typedef enum {
  LCVQ_F32 = 0,   /* float */
  LCVQ_BF16 = 1   /* bfloat16 bit patterns (uint16_t) */
} lcvq_dtype;

/* Forward formulation for lcvq_gemm (both compute the same Y = X W~):
 *  DECODE:    codes are decoded to bf16 tiles of A z + B on chip and multiplied
 *             with X directly.
 *  ALGEBRAIC: X is first multiplied group-wise by A (X'[m][g d + j] =
 *             sum_i X[m][g d + i] A[i][j]) and dotted with B; the main loop then
 *             multiplies X' with the raw integer codes and adds the per-row
 *             B term:  Y = X' Z^T + s 1^T.  Exact algebra on
 *             sum_k x_k w~_k = sum_g x_g^T (A z_g + B).
 *  AUTO:      the library's choice (ALGEBRAIC on the tensor-core paths). */
typedef enum { LCVQ_FORM_AUTO = 0, LCVQ_FORM_DECODE = 1, LCVQ_FORM_ALGEBRAIC = 2 } lcvq_form;

typedef enum {
  LCVQ_OP_GEMM = 0,
  LCVQ_OP_GEMM_BACKWARD = 1,
  LCVQ_OP_FIT_AFFINE = 2,
  LCVQ_OP_ASSIGN_LDLQ = 3,
  LCVQ_OP_FIT_AFFINE_H = 4
} lcvq_op;

/* Code assignment and 2-bit packing (LC-QAT technical summary, Methodology 1:
 * index selection becomes rounding and clamping; Methodology 3: proxy weights
 * are rounded and clamped to integer weights).
 *   Wp        [d_out][d_in] fp32 proxy weights (read only).
 *   packed    [d_out][d_in/4] out: codes z = clamp(rint(Wp), 0, 3), format V1.
 *   mask_bits [d_out][d_in/8] out, may be NULL: bit set where 0 <= Wp <= 3.
 *   d         vector length (only checked: d_in % d == 0).
 * Shapes: d_in % 8 == 0; d_out, d_in >= 0 (an empty matrix is a no-op). */
LCVQ_API lcvq_status lcvq_assign_pack(const float* Wp, int64_t d_out, int64_t d_in, int d,
                             uint8_t* packed, uint8_t* mask_bits, void* stream);

/* Decode: materialize W~[n][g d + i] = sum_j A[i][j] z[n][g d + j] + B[i]
 * (Methodology 1, c = A z + B; Methodology 3, A W_z + B), computed in fp32 and
 * stored as w_dtype (bf16 rounds to nearest even).
 *   packed [d_out][d_in/4] codes; A [d*d] fp32 row-major; B [d] fp32;
 *   W      [d_out][d_in] out.
 * Shapes: d_in % 16 == 0. */
LCVQ_API lcvq_status lcvq_decode(const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                        const float* A, const float* B, void* W, lcvq_dtype w_dtype,
                        void* stream);

/* Fused decode-and-GEMM  Y = X W~  (Methodology 3: the forward is recast onto
 * INT2 x FP16 matmul operators; decoupleQ eq. (1) for the layer convention).
 *   X [M][d_in] in `dtype`; Y [M][d_out] out in `dtype`.
 *   dtype BF16: tensor-core paths (M <= 32: decode-GEMV; larger M: tcgen05
 *   GEMM), fp32 accumulation.  dtype F32: an fp32 CUDA-core path.
 *   For M <= 4 (bf16) the decode-GEMV takes the int8 path: per token and
 *   chunk class r (the 512-position chunks r, r + 8, ... of K) X' = x A
 *   (fp32) is scaled by a power of two s, the largest with max |X'| s <= 32639
 *   over the class, rounded to q = rint(X' s) and split into two signed byte
 *   digits q = 256 hi + lo; the codes (u8) times the digits (s8) accumulate
 *   exactly on the integer tensor cores, each class's sum is scaled by 1/s
 *   and the classes are added in class order, plus the per-row constant
 *   s' - 3/2 sum_r (sum q_r) / s_r.  The activations' only rounding is that of
 *   X' to q: half a step of 1/s, about 2^-16 of the class's largest |X'|
 *   (bf16's is 2^-9 of each |X'|).  For 5 <= M <= 32 X' is rounded to bf16 (see
 *   lcvq_xform).
 *   form: see lcvq_form (F32 always uses DECODE).
 *   workspace: >= lcvq_workspace_size(LCVQ_OP_GEMM, ...) bytes, 256-byte aligned.
 * Shapes: d_in % 64 == 0, d_out % 8 == 0, M >= 0, d_in and d_out <= 2^30.
 * M == 0 or d_out == 0 is a no-op; d_in == 0 writes Y = 0. */
LCVQ_API lcvq_status lcvq_gemm(const void* X, lcvq_dtype dtype, int64_t M,
                      const uint8_t* packed, int64_t d_out, int64_t d_in, int d,
                      const float* A, const float* B, void* Y, lcvq_form form,
                      void* workspace, size_t ws_bytes, void* stream);

/* The algebraic form in two calls (bf16 only).  For M > 4, lcvq_gemm with
 * LCVQ_FORM_ALGEBRAIC is exactly lcvq_xform followed by lcvq_gemm_xformed (for
 * M <= 4 lcvq_gemm takes its int8 path); the split lets a caller time or reuse
 * the halves.
 *
 * lcvq_xform: X'[m][g d + j] = sum_i X[m][g d + i] A[i][j] is rounded to bf16
 * and stored in the "decoder order" the integer-code GEMM consumes: within each
 * block of 16 consecutive k, element 2c holds position c and element 2c + 1
 * position c + 8 (c = 0..7), each multiplied by 4^-(c mod 3).  corr[m] is the
 * per-row constant  s'[m] - 3/2 sum_k bf16(X')[m][k] - 128 sum_k X''[m][k]
 * with s'[m] = sum_g x_g . (B + 3/2 A 1), formed in fp64 and stored as fp32.
 *   X [M][d_in] bf16;  Xpp [M][d_in] bf16 out;  corr [M] fp32 out.
 * lcvq_gemm_xformed: Y[m][n] = sum_k X''[m][k] v[n][k] + corr[m], where
 * v = 128 + 4^(c mod 3) z is the bf16 value the kernel's one-instruction code
 * decoder produces; this equals sum_k bf16(X')[m][k] (z[n][k] - 3/2) + s'[m],
 * the centred algebraic form of Y = X W~.
 *   Y [M][d_out] bf16 out.
 * Shapes as lcvq_gemm (M >= 1). */
LCVQ_API lcvq_status lcvq_xform(const void* X, lcvq_dtype dtype, int64_t M, int64_t d_in, int d,
                                const float* A, const float* B, void* Xpp, float* corr,
                                void* stream);
LCVQ_API lcvq_status lcvq_gemm_xformed(const void* Xpp, const float* corr, int64_t M,
                                       const uint8_t* packed, int64_t d_out, int64_t d_in,
                                       void* Y, void* stream);

/* Grouped decode-GEMV: Y_i = X_i W~_i for `count` independent matrices.  The
 * pages define the operation per matrix (Methodology 3; decoupleQ eq. (1) for
 * the layer convention); grouping is this library's launch arrangement for
 * many matrices at once (the projections of a layer that read one input, the
 * experts of a layer, or any set of independent decode-time matmuls).  For
 * M <= 16 each Y_i is bit-identical to lcvq_gemm on item i alone (at M <= 4
 * both take the int8 path described at lcvq_gemm).  For 17 <= M <= 32, groups of at least 296 tiles of 128 rows run on the
 * tcgen05 tensor cores (decoded weights in tensor memory) and sum in a
 * different fp32 order: Y_i then agrees with lcvq_gemm within the forward
 * tolerance, not bitwise.
 *   items  host array of `count` descriptors (read during the call only):
 *          X [M][d_in] bf16, packed [d_out][d_in/4] codes, A [d*d] and B [d]
 *          fp32, Y [M][d_out] bf16 out; every pointer 16-byte aligned.
 *   M      common token count, 1 <= M <= 32 (the decode-GEMV regime).
 *   d      common vector length.
 *   workspace: >= lcvq_workspace_size_grouped(items, count, M, d) bytes,
 *          256-byte aligned, first 256 bytes zeroed once (as lcvq_gemm).
 * Shapes per item: d_in % 64 == 0, d_out % 8 == 0, 1 <= d_in, d_out < 2^28.
 * count >= 1.  The call launches 2 * ceil(count / 128) kernels: the
 * X-transforms of up to 128 matrices, then one persistent decode-GEMV over
 * their tiles.  Any invalid item fails the whole call before anything is
 * launched.  The Y_i must not overlap one another or any input. */
typedef struct {
  const void* X;
  const uint8_t* packed;
  const float* A;
  const float* B;
  void* Y;
  int64_t d_out;
  int64_t d_in;
} lcvq_gemm_item;

LCVQ_API lcvq_status lcvq_gemm_grouped(const lcvq_gemm_item* items, int count, int64_t M, int d,
                                       void* workspace, size_t ws_bytes, void* stream);
LCVQ_API size_t lcvq_workspace_size_grouped(const lcvq_gemm_item* items, int count, int64_t M,
                                            int d);

/* Decode-GEMV without a workspace.  The pages have no counterpart: this is a
 * convenience of this library.  It computes exactly what lcvq_gemm computes for
 * bf16 activations and M <= 32 (same kernels, same results), but takes no
 * workspace, because some callers cannot provide one: code running while a
 * CUDA graph is being captured (device allocation is not allowed there),
 * runtimes that reserve all device memory at start-up and forbid later
 * allocations, and extensions whose host framework owns the allocator and
 * offers them no scratch space.
 *   X [M][d_in] bf16, Y [M][d_out] bf16; packed, A, B as lcvq_gemm.
 * Scratch: a fixed 2 MiB + 256 B array inside the library's device memory,
 * held by every GPU that loads the library until the process exits.  Limits:
 * M <= 32 and d_in <= 32768; larger sizes return LCVQ_ERR_WORKSPACE and
 * launch nothing.  Other shape rules as lcvq_gemm.
 * The first call on each device (made with that device current) looks up the
 * array's device address (cudaGetSymbolAddress) and caches it; make that first
 * call before any stream capture begins.  The call allocates no memory.
 * All calls share the one array and it keeps the last call's contents: two
 * calls that may run at the same time on the GPU (different streams, or
 * different host threads on the same device) race on it and must be ordered
 * by the caller. */
LCVQ_API lcvq_status lcvq_gemv_static(const void* X, int64_t M, const uint8_t* packed,
                                      int64_t d_out, int64_t d_in, int d, const float* A,
                                      const float* B, void* Y, void* stream);

/* Straight-through QAT backward of Y = X W~ with W~ = decode(clamp(rint(Wp))).
 * (Methodology 1: gradients flow through the linear map c = A z + B;
 * Methodology 3 and the gradient-estimation ablation: STE through the
 * rounding, zero where the clamp is active.)  Given dY = dL/dY:
 *   dX [M][d_in]  = dY W~                               (may be NULL)
 *   G[n][k]       = sum_m dY[m][n] X[m][k]               (never stored)
 *   dA [d*d]      = sum_{n,g} G[n][g d + i] z[n][g d + j]   (fp32, overwritten)
 *   dB [d]        = sum_{n,g} G[n][g d + i]                 (fp32, overwritten)
 *   dWp [d_out][d_in] = mask * sum_i A[i][j] G[n][g d + i]   (fp32, may be NULL)
 * X, dY, dX in `dtype`.  mask_bits is required when dWp is non-NULL.
 * dA and dB are reduced in a fixed order (bitwise reproducible run to run).
 * Shapes as lcvq_gemm.  M == 0 writes dA = dB = dWp = 0. */
LCVQ_API lcvq_status lcvq_gemm_backward(const void* X, const void* dY, lcvq_dtype dtype, int64_t M,
                               const uint8_t* packed, const uint8_t* mask_bits,
                               int64_t d_out, int64_t d_in, int d,
                               const float* A, const float* B,
                               void* dX, float* dA, float* dB, float* dWp,
                               void* workspace, size_t ws_bytes, void* stream);

/* DGE rescale of the proxy-weight gradient (LC-QAT technical summary,
 * Methodology 3: the paper's backward uses a differentiable gradient
 * estimator (DGE), a smooth curve in place of the rounding, instead of the
 * straight-through estimator).  The pages give no formula; this library takes
 * the tanh staircase through the rounding points on [0, 3]
 *     phi_k(w) = floor(w) + 1/2 + tanh(k (frac(w) - 1/2)) / (2 tanh(k/2)),
 * equal to w at the integers, to rint(w) as k -> inf and to w as k -> 0, and
 * multiplies the gradient by its derivative
 *     phi_k'(w) = k / (2 tanh(k/2)) sech^2(k (frac(w) - 1/2))   (0 outside [0, 3]).
 * Applied to the dWp of lcvq_gemm_backward (the STE gradient, A^T G inside the
 * clamp mask) it gives the DGE gradient: dWp[i] *= phi_k'(Wp[i]).  As k -> 0
 * the factor tends to the clamp mask, i.e. back to the STE.
 *   dWp [n] fp32 in/out;  Wp [n] fp32 proxy weights;  k > 0 the sharpness.
 * Shapes: n % 4 == 0, n >= 0; 16-byte aligned pointers. */
LCVQ_API lcvq_status lcvq_dge_scale(float* dWp, const float* Wp, int64_t n, float k, void* stream);

/* Least-squares refit of the float part (A, B) given the codes (decoupleQ
 * page: eq. (5), the layer objective tr{(W~ - W0)^T H (W~ - W0)}, and section
 * 3.3, where the float part is solved in closed form with the integer part
 * fixed; here for LC-VQ's codewords c = A z + B, LC-QAT technical summary,
 * Methodology 1).  H is taken as its diagonal h: the call minimizes
 *     sum_n sum_k h[k] (W0[n][k] - W~[n][k])^2,   W~ = A z + B per vector,
 * over A and B.  Row i of [A | B] is G_i^+ R_i, where G_i = sum h zt zt^T
 * and R_i = sum h W0 zt run over every vector with zt = [z_0 .. z_{d-1}, 1],
 * taking channel k = g d + i of vector g.  G^+ is the pseudo-inverse:
 * eigenvalues below 1e-12 of the largest count as zero, which gives the
 * minimum-norm solution when G_i is singular (a code position that never
 * varies, or weights that vanish).  The pass forms, per vector position, the
 * codes' Gram (exact) and the targets times the codes (d = 8: tf32 hi/lo tensor-
 * core products; other d: fp32), added into fp64 every 16 terms; h enters in
 * fp64 afterwards.  Every sum has a fixed order and the solve is fp64: the
 * result is bitwise reproducible.
 *   W0     [d_out][d_in] fp32 target weights (e.g. the pretrained matrix).
 *   packed [d_out][d_in/4] codes (format V1).
 *   h      [d_in] fp32 channel weights >= 0 (e.g. diag(X^T X)), or NULL for 1.
 *   A      [d*d] fp32 out (row-major);  B [d] fp32 out.
 *   workspace: >= lcvq_workspace_size(LCVQ_OP_FIT_AFFINE, LCVQ_F32, 0, d_out,
 *   d_in, d) bytes, 256-byte aligned.
 * Shapes: d_in % 16 == 0; an empty matrix gives A = 0, B = 0.  Launches 2
 * kernels. */
LCVQ_API lcvq_status lcvq_fit_affine(const float* W0, const uint8_t* packed, int64_t d_out,
                                     int64_t d_in, int d, const float* h, float* A, float* B,
                                     void* workspace, size_t ws_bytes, void* stream);

/* Least-squares refit of (A, B) under the full input Hessian H (decoupleQ
 * page: eq. (5), the layer objective tr{(W~ - W0)^T H (W~ - W0)} with W~ and
 * W0 of shape d_in x d_out and H = X^T X of the layer's inputs; section 3.3:
 * with the integer part fixed the float part is a quadratic, solved in closed
 * form; LC-QAT technical summary, Methodology 1, for the codewords
 * c = A z + B).  In storage order the call minimizes
 *     sum_n (W~[n] - W0[n])^T H (W~[n] - W0[n]),   W~ = A z + B per vector,
 * over A and B.  With theta = [A | B] (row i = [A[i][0..d-1], B[i]]) and
 * zt = [z_0 .. z_{d-1}, 1] per vector, the normal equations couple every pair
 * of vector positions (g, h):
 *     L[(i,a),(j,b)] = sum_{g,h} H[g d + i][h d + j] sum_n zt[n][g][a] zt[n][h][b]
 *     R[(i,a)]       = sum_g sum_k H[g d + i][k] sum_n zt[n][g][a] W0[n][k]
 * and theta = L^+ R (d (d+1) unknowns): Cholesky when every pivot is above
 * 1e-8 of the largest diagonal entry, otherwise the pseudo-inverse with
 * eigenvalues below 1e-12 of the largest taken as zero (the minimum-norm
 * solution).  With H diagonal this is lcvq_fit_affine with h = diag(H).
 * Arithmetic: the code Gram and the code column sums are exact (bf16 codes,
 * fp32 tensor-core sums); W0 enters the tensor-core contraction W0^T Z as two
 * bf16 terms (within 2^-18 of W0) summed in fp32 over the rows; the
 * contraction with H and the solve are fp64.  Every sum has a fixed order:
 * the result is bitwise reproducible.
 *   W0     [d_out][d_in] fp32 target weights.
 *   packed [d_out][d_in/4] codes (format V1).
 *   H      [d_in][d_in] fp32, symmetric (every entry is read); e.g. X^T X of
 *          calibration activations, usually with a small ridge.
 *   A      [d*d] fp32 out (row-major);  B [d] fp32 out.
 *   workspace: >= lcvq_workspace_size(LCVQ_OP_FIT_AFFINE_H, LCVQ_F32, 0, d_out,
 *   d_in, d) bytes (about 2 d_out d_in * 3 + 12 d_in^2 bytes of scratch),
 *   256-byte aligned, first 256 bytes zeroed once.
 * Shapes: d_in % 64 == 0, d_in <= 65536, d_out <= 2^20; an empty matrix gives
 * A = 0, B = 0.  Launches 5 kernels: the bf16 operand pass, one tcgen05 GEMM
 * of 2 (d_in + 64)(3 d_in + 64) d_out flops, the fp64 contraction with H, the
 * fixed-order sum of its partials and the solve. */
LCVQ_API lcvq_status lcvq_fit_affine_h(const float* W0, const uint8_t* packed, int64_t d_out,
                                       int64_t d_in, int d, const float* H, float* A, float* B,
                                       void* workspace, size_t ws_bytes, void* stream);

/* H-aware sequential code assignment, the PTQ initialisation of the codes
 * (LC-QAT technical summary, Methodology 2: the initial integer weights come
 * from LDLQ, column-wise quantization with sequential compensation of the
 * reconstruction error; decoupleQ page, section 3.3, eq. (8)-(11): round and
 * clip one element, then re-solve the remaining ones without the integer
 * constraint and the box).  For a row with target w0 and the input Hessian H
 * (e.g. X^T X of calibration activations) the layer objective is
 *     1/2 (Abar z + bbar - w0)^T H (Abar z + bbar - w0) = 1/2 (z - p)^T Q (z - p),
 * with Abar = blockdiag(A, .., A), bbar = B per vector, Q = Abar^T H Abar and
 * p = Abar^-1 (w0 - bbar), the row's code-space target (what W_p holds).  The
 * call takes P and the factor U of Q = (I + U) diag(D) (I + U)^T (U strictly
 * upper triangular: the Cholesky factor of Q with its rows and columns
 * reversed, scaled to a unit diagonal), and sets, for every row, in order of
 * increasing column j,
 *     z_j = clamp(rint(t_j), 0, 3),   t_j = p_j + sum_{i<j} U[i][j] (p_i - z_i),
 * which is t_j = the j-th element of the minimiser of eq. (11) once z_0 ..
 * z_{j-1} are fixed.  With Q diagonal (U = 0) this is lcvq_assign_pack.
 * Arithmetic is fp32 (t in a fixed blocked order); a code can differ from the
 * fp64 rule only where t_j lies within fp32 rounding of a rounding boundary.
 *   P      [d_out][d_in] fp32 targets; finite values (a non-finite one makes
 *          the rest of its row unspecified).
 *   U      [d_in][d_in] fp32 row-major; only the entries above the diagonal
 *          are read.
 *   packed [d_out][d_in/4] out: the codes (format V1).
 *   workspace: >= lcvq_workspace_size(LCVQ_OP_ASSIGN_LDLQ, LCVQ_F32, 0, d_out,
 *   d_in, d) bytes (the fp32 errors p - z of every row), 256-byte aligned.
 * Shapes: d_in % 64 == 0, d_in % d == 0, d_in <= 2^20; 16-byte aligned
 * pointers.  Launches 1 kernel of ceil(d_out / 32) CTAs, d_out d_in (d_in - 1) / 2
 * fused multiply-adds. */
LCVQ_API lcvq_status lcvq_assign_ldlq(const float* P, const float* U, int64_t d_out, int64_t d_in,
                                      int d, uint8_t* packed, void* workspace, size_t ws_bytes,
                                      void* stream);

/* Workspace bytes a call with these arguments needs (0 on invalid input).
 * The workspace holds the device error word (its first 256 bytes, which the
 * caller zeroes once before first use), the transformed activations of the
 * algebraic form and the per-block partial sums of dA/dB.  A workspace may be
 * reused by calls that are ordered on one stream; calls that may overlap on the
 * GPU need separate workspaces. */
LCVQ_API size_t lcvq_workspace_size(lcvq_op op, lcvq_dtype dtype, int64_t M, int64_t d_out,
                           int64_t d_in, int d);

/* Synchronizes `stream`, reads and clears the workspace's device error word.
 * Returns LCVQ_OK, LCVQ_ERR_DEVICE_TIMEOUT, or LCVQ_ERR_CUDA. */
LCVQ_API lcvq_status lcvq_check_device_error(void* workspace, void* stream);

/* Static string naming a status. */
LCVQ_API const char* lcvq_status_string(lcvq_status s);

/* Number of kernels the last successful call on this host thread launched
 * (for launch accounting by benchmarks). */
LCVQ_API int lcvq_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LCVQ_H_ */

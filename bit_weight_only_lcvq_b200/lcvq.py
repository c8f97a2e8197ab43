"""Thin Python binding of liblcvq's C ABI (argument marshalling only).

Every step of the hot path runs in the library's CUDA kernels; this module only
turns torch CUDA tensors into pointers and sizes, passes the current stream and
raises on a non-OK status.  There is no fallback: if ``liblcvq.so`` is missing
or fails to load, every call raises.

Names follow the C ABI (``include/lcvq.h``): assign_pack, decode, gemm,
gemm_backward, workspace_size, check_device_error.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblcvq.so")

F32, BF16 = 0, 1
FORMS = {"auto": 0, "decode": 1, "algebraic": 2}
OP_GEMM, OP_GEMM_BACKWARD, OP_FIT_AFFINE, OP_ASSIGN_LDLQ, OP_FIT_AFFINE_H = 0, 1, 2, 3, 4
STATUS = {
    0: "LCVQ_OK",
    1: "LCVQ_ERR_INVALID_ARG",
    2: "LCVQ_ERR_UNSUPPORTED",
    3: "LCVQ_ERR_ALIGNMENT",
    4: "LCVQ_ERR_WORKSPACE",
    5: "LCVQ_ERR_CUDA",
    6: "LCVQ_ERR_DEVICE_TIMEOUT",
}
EXPORTS = (
    "lcvq_assign_pack",
    "lcvq_decode",
    "lcvq_gemm",
    "lcvq_gemm_backward",
    "lcvq_xform",
    "lcvq_gemm_xformed",
    "lcvq_gemv_static",
    "lcvq_gemm_grouped",
    "lcvq_fit_affine",
    "lcvq_fit_affine_h",
    "lcvq_dge_scale",
    "lcvq_assign_ldlq",
    "lcvq_workspace_size",
    "lcvq_workspace_size_grouped",
    "lcvq_check_device_error",
    "lcvq_status_string",
    "lcvq_last_launch_count",
)


class LcvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


_lib = None

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


class GemmItem(ctypes.Structure):
    """lcvq_gemm_item: one matrix of a grouped decode-GEMV."""
    _fields_ = [("X", _vp), ("packed", _vp), ("A", _vp), ("B", _vp), ("Y", _vp),
                ("d_out", _i64), ("d_in", _i64)]


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"liblcvq.so is not built ({LIB_PATH}); run "
                          "python -m bit_weight_only_lcvq_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        L.lcvq_assign_pack.argtypes = [_vp, _i64, _i64, _i32, _vp, _vp, _vp]
        L.lcvq_decode.argtypes = [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _i32, _vp]
        L.lcvq_gemm.argtypes = [_vp, _i32, _i64, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _i32,
                                _vp, _sz, _vp]
        L.lcvq_gemm_backward.argtypes = [_vp, _vp, _i32, _i64, _vp, _vp, _i64, _i64, _i32, _vp,
                                         _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.lcvq_xform.argtypes = [_vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp]
        L.lcvq_gemm_xformed.argtypes = [_vp, _vp, _i64, _vp, _i64, _i64, _vp, _vp]
        L.lcvq_gemv_static.argtypes = [_vp, _i64, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp]
        L.lcvq_gemm_grouped.argtypes = [ctypes.POINTER(GemmItem), _i32, _i64, _i32, _vp, _sz, _vp]
        L.lcvq_workspace_size_grouped.argtypes = [ctypes.POINTER(GemmItem), _i32, _i64, _i32]
        L.lcvq_workspace_size_grouped.restype = _sz
        L.lcvq_fit_affine.argtypes = [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
        L.lcvq_fit_affine_h.argtypes = [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
        L.lcvq_dge_scale.argtypes = [_vp, _vp, _i64, ctypes.c_float, _vp]
        L.lcvq_assign_ldlq.argtypes = [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _sz, _vp]
        L.lcvq_workspace_size.argtypes = [_i32, _i32, _i64, _i64, _i64, _i32]
        L.lcvq_workspace_size.restype = _sz
        L.lcvq_check_device_error.argtypes = [_vp, _vp]
        L.lcvq_status_string.argtypes = [_i32]
        L.lcvq_status_string.restype = ctypes.c_char_p
        L.lcvq_last_launch_count.argtypes = []
        for fn in ("lcvq_assign_pack", "lcvq_decode", "lcvq_gemm", "lcvq_gemm_backward",
                   "lcvq_xform", "lcvq_gemm_xformed", "lcvq_gemv_static", "lcvq_gemm_grouped",
                   "lcvq_fit_affine", "lcvq_fit_affine_h", "lcvq_dge_scale", "lcvq_assign_ldlq",
                   "lcvq_check_device_error",
                   "lcvq_last_launch_count"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t):
    """Device address of a CUDA tensor (None stays None).  Every array the
    C ABI takes is device memory, so a host tensor is refused here rather than
    handed to a kernel as an address it cannot read."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"lcvq: expected a CUDA tensor, got one on {t.device}")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(dt) -> int:
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {dt}")


def _check(fn: str, st: int):
    if st != 0:
        raise LcvqError(fn, st)


def last_launch_count() -> int:
    return lib().lcvq_last_launch_count()


def workspace_size(op: int, dtype, M: int, d_out: int, d_in: int, d: int) -> int:
    return int(lib().lcvq_workspace_size(op, _dtype_code(dtype), M, d_out, d_in, d))


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A workspace tensor (zeroed, so its error word starts clear)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def assign_pack(Wp: torch.Tensor, d: int, *, with_mask: bool = True, packed=None, mask=None,
                stream=None):
    """Codes z = clamp(rint(Wp), 0, 3) packed 4 per byte, and the clamp mask bits."""
    d_out, d_in = Wp.shape
    if packed is None:
        packed = torch.empty((d_out, d_in // 4), dtype=torch.uint8, device=Wp.device)
    if with_mask and mask is None:
        mask = torch.empty((d_out, d_in // 8), dtype=torch.uint8, device=Wp.device)
    _check("lcvq_assign_pack", lib().lcvq_assign_pack(
        _ptr(Wp), d_out, d_in, d, _ptr(packed), _ptr(mask) if with_mask else None,
        _stream(stream)))
    return packed, (mask if with_mask else None)


def decode(packed: torch.Tensor, d_in: int, A: torch.Tensor, B: torch.Tensor, d: int, *,
           dtype=torch.bfloat16, out=None, stream=None) -> torch.Tensor:
    """Materialized W~ = A z + B, shape [d_out][d_in]."""
    d_out = packed.shape[0]
    if out is None:
        out = torch.empty((d_out, d_in), dtype=dtype, device=packed.device)
    _check("lcvq_decode", lib().lcvq_decode(_ptr(packed), d_out, d_in, d, _ptr(A), _ptr(B),
                                            _ptr(out), _dtype_code(out.dtype), _stream(stream)))
    return out


def gemm(X: torch.Tensor, packed: torch.Tensor, d_in: int, A: torch.Tensor, B: torch.Tensor,
         d: int, *, form: str = "auto", workspace=None, out=None, stream=None) -> torch.Tensor:
    """Y = X W~ (X [M][d_in], Y [M][d_out] in X's dtype)."""
    M = X.shape[0]
    d_out = packed.shape[0]
    if out is None:
        out = torch.empty((M, d_out), dtype=X.dtype, device=X.device)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_GEMM, X.dtype, M, d_out, d_in, d), X.device)
    _check("lcvq_gemm", lib().lcvq_gemm(
        _ptr(X), _dtype_code(X.dtype), M, _ptr(packed), d_out, d_in, d, _ptr(A), _ptr(B),
        _ptr(out), FORMS[form], _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def gemm_backward(X: torch.Tensor, dY: torch.Tensor, packed: torch.Tensor, mask: torch.Tensor,
                  d_in: int, A: torch.Tensor, B: torch.Tensor, d: int, *, want_dx: bool = True,
                  want_dwp: bool = True, workspace=None, outs=None, stream=None) -> dict:
    """STE backward: returns dict(dX, dA, dB, dWp) (dX / dWp None when not wanted)."""
    M = X.shape[0]
    d_out = packed.shape[0]
    dev = X.device
    o = dict(outs or {})
    if want_dx and o.get("dX") is None:
        o["dX"] = torch.empty((M, d_in), dtype=X.dtype, device=dev)
    if want_dwp and o.get("dWp") is None:
        o["dWp"] = torch.empty((d_out, d_in), dtype=torch.float32, device=dev)
    if o.get("dA") is None:
        o["dA"] = torch.empty((d, d), dtype=torch.float32, device=dev)
    if o.get("dB") is None:
        o["dB"] = torch.empty((d,), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_GEMM_BACKWARD, X.dtype, M, d_out, d_in, d), dev)
    _check("lcvq_gemm_backward", lib().lcvq_gemm_backward(
        _ptr(X), _ptr(dY), _dtype_code(X.dtype), M, _ptr(packed), _ptr(mask), d_out, d_in, d,
        _ptr(A), _ptr(B), _ptr(o.get("dX") if want_dx else None), _ptr(o["dA"]), _ptr(o["dB"]),
        _ptr(o.get("dWp") if want_dwp else None), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    if not want_dx:
        o["dX"] = None
    if not want_dwp:
        o["dWp"] = None
    return o


def xform(X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, d: int, *, xpp=None, corr=None,
          stream=None):
    """First half of the algebraic form: (X'' in decoder order, per-row corr)."""
    M, d_in = X.shape
    if xpp is None:
        xpp = torch.empty((M, d_in), dtype=torch.bfloat16, device=X.device)
    if corr is None:
        corr = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check("lcvq_xform", lib().lcvq_xform(_ptr(X), _dtype_code(X.dtype), M, d_in, d, _ptr(A),
                                          _ptr(B), _ptr(xpp), _ptr(corr), _stream(stream)))
    return xpp, corr


def gemm_xformed(xpp: torch.Tensor, corr: torch.Tensor, packed: torch.Tensor, *, out=None,
                 stream=None) -> torch.Tensor:
    """Second half: the integer-code GEMM Y = X'' v^T + corr."""
    M, d_in = xpp.shape
    d_out = packed.shape[0]
    if out is None:
        out = torch.empty((M, d_out), dtype=torch.bfloat16, device=xpp.device)
    _check("lcvq_gemm_xformed", lib().lcvq_gemm_xformed(
        _ptr(xpp), _ptr(corr), M, _ptr(packed), d_out, d_in, _ptr(out), _stream(stream)))
    return out


def gemv_static(X: torch.Tensor, packed: torch.Tensor, d_in: int, A: torch.Tensor,
                B: torch.Tensor, d: int, *, out=None, stream=None) -> torch.Tensor:
    """Decode-GEMV (bf16, M <= 32) that takes no workspace: its scratch lives in a
    fixed array inside the library, for callers that cannot allocate device
    memory (see lcvq_gemv_static in include/lcvq.h)."""
    M = X.shape[0]
    d_out = packed.shape[0]
    if out is None:
        out = torch.empty((M, d_out), dtype=torch.bfloat16, device=X.device)
    _check("lcvq_gemv_static", lib().lcvq_gemv_static(
        _ptr(X), M, _ptr(packed), d_out, d_in, d, _ptr(A), _ptr(B), _ptr(out), _stream(stream)))
    return out


def set_wait_limit(workspace: torch.Tensor, cycles: int) -> None:
    """Writes the workspace header's wait limit (bytes 8..15, int64 clock
    cycles; 0 = the library's default).  Ordered on the current stream."""
    workspace[8:16].view(torch.int64).fill_(int(cycles))


def check_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronizes the stream and returns the workspace's device error status."""
    return int(lib().lcvq_check_device_error(_ptr(workspace), _stream(stream)))


def _group_items(jobs, outs):
    arr = (GemmItem * len(jobs))()
    for i, (X, packed, A, B, d_in) in enumerate(jobs):
        arr[i] = GemmItem(_ptr(X), _ptr(packed), _ptr(A), _ptr(B), _ptr(outs[i]),
                          packed.shape[0], d_in)
    return arr


def workspace_size_grouped(jobs, M: int, d: int) -> int:
    """Workspace bytes for gemm_grouped over jobs = [(X, packed, A, B, d_in), ...]."""
    arr = (GemmItem * len(jobs))()
    for i, (X, packed, A, B, d_in) in enumerate(jobs):
        arr[i] = GemmItem(None, None, None, None, None, packed.shape[0], d_in)
    return int(lib().lcvq_workspace_size_grouped(arr, len(jobs), M, d))


def gemm_grouped(jobs, d: int, *, workspace=None, outs=None, stream=None):
    """Grouped decode-GEMV: Y_i = X_i W~_i for jobs = [(X, packed, A, B, d_in), ...]
    sharing the token count M <= 32 and d.  Returns the list of Y_i."""
    M = jobs[0][0].shape[0]
    if outs is None:
        outs = [torch.empty((M, packed.shape[0]), dtype=torch.bfloat16, device=X.device)
                for X, packed, _, _, _ in jobs]
    arr = _group_items(jobs, outs)
    if workspace is None:
        workspace = new_workspace(workspace_size_grouped(jobs, M, d), jobs[0][0].device)
    _check("lcvq_gemm_grouped", lib().lcvq_gemm_grouped(
        arr, len(jobs), M, d, _ptr(workspace), workspace.numel(), _stream(stream)))
    return outs


def fit_affine(W0: torch.Tensor, packed: torch.Tensor, d: int, *, h=None, workspace=None,
               A=None, B=None, stream=None):
    """Least-squares (A, B) for target weights W0 given the codes, with optional
    per-input-channel weights h (see lcvq_fit_affine).  Returns (A, B)."""
    d_out, d_in = W0.shape
    dev = W0.device
    if A is None:
        A = torch.empty((d, d), dtype=torch.float32, device=dev)
    if B is None:
        B = torch.empty(d, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_FIT_AFFINE, torch.float32, 0, d_out, d_in, d),
                                  dev)
    _check("lcvq_fit_affine", lib().lcvq_fit_affine(
        _ptr(W0), _ptr(packed), d_out, d_in, d, _ptr(h), _ptr(A), _ptr(B), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return A, B


def fit_affine_h(W0: torch.Tensor, packed: torch.Tensor, d: int, H: torch.Tensor, *,
                 workspace=None, A=None, B=None, stream=None):
    """Least-squares (A, B) for target weights W0 given the codes under the full
    input Hessian H [d_in][d_in] (see lcvq_fit_affine_h).  Returns (A, B)."""
    d_out, d_in = W0.shape
    dev = W0.device
    if A is None:
        A = torch.empty((d, d), dtype=torch.float32, device=dev)
    if B is None:
        B = torch.empty(d, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_FIT_AFFINE_H, torch.float32, 0, d_out, d_in, d),
                                  dev)
    _check("lcvq_fit_affine_h", lib().lcvq_fit_affine_h(
        _ptr(W0), _ptr(packed), d_out, d_in, d, _ptr(H), _ptr(A), _ptr(B), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return A, B


def assign_ldlq(P: torch.Tensor, U: torch.Tensor, d: int, *, workspace=None, packed=None,
                stream=None) -> torch.Tensor:
    """Codes of the H-aware sequential assignment of the code-space targets P
    [d_out][d_in] with the strictly upper factor U [d_in][d_in] of the
    code-space Hessian (see lcvq_assign_ldlq).  Returns packed [d_out][d_in/4]."""
    d_out, d_in = P.shape
    dev = P.device
    if packed is None:
        packed = torch.empty((d_out, d_in // 4), dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_ASSIGN_LDLQ, torch.float32, 0, d_out, d_in, d),
                                  dev)
    _check("lcvq_assign_ldlq", lib().lcvq_assign_ldlq(
        _ptr(P), _ptr(U), d_out, d_in, d, _ptr(packed), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return packed


def dge_scale(dWp: torch.Tensor, Wp: torch.Tensor, k: float, *, stream=None) -> torch.Tensor:
    """In place: dWp *= phi_k'(Wp), turning the STE gradient of gemm_backward into
    the DGE gradient (see lcvq_dge_scale).  Returns dWp."""
    _check("lcvq_dge_scale", lib().lcvq_dge_scale(_ptr(dWp), _ptr(Wp), dWp.numel(), float(k),
                                                  _stream(stream)))
    return dWp

"""ctypes wrapper of the C++ fp64 oracle (``oracle/lcvq_oracle.cpp``).
TEST INFRASTRUCTURE ONLY: the same rule as ``oracle/lcvq_oracle.py`` applies
(only ``tests/``, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline legs
may use it; the library never does).

The functions take and return numpy arrays with the same names and meanings
as the numpy oracle's (assign, pack_codes, unpack_codes, pack_mask,
unpack_mask, decode, forward, backward, ldlq_assign, fit_affine, fit_affine_h,
dge_phi, dge_derivative), so every pin written for one runs on the other.  Floating inputs are widened to fp64 (exact for fp32/bf16 values).

``build()`` compiles the shared library with g++ (plain C++17, -O2, no
fast-math, no fused multiply-add contraction); ``lib()`` builds it on first use
when it is missing or older than its source.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lcvq_oracle.cpp")
SO = os.path.join(HERE, "liblcvq_oracle.so")
CXX = os.environ.get("CXX", "g++")
FLAGS = ["-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]

_lib = None
_vp, _i64, _i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int


def build(force: bool = False) -> str:
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < os.path.getmtime(SRC):
        tmp = SO + f".tmp{os.getpid()}"
        r = subprocess.run([CXX, *FLAGS, SRC, "-o", tmp], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"g++ failed for the C++ oracle:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, SO)
    return SO


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.lco_assign.argtypes = [_vp, _i64, _vp, _vp]
        for nm in ("lco_pack_codes", "lco_unpack_codes", "lco_pack_mask", "lco_unpack_mask"):
            getattr(L, nm).argtypes = [_vp, _i64, _i64, _vp]
        for nm in ("lco_decode_z8", "lco_decode_zf"):
            getattr(L, nm).argtypes = [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _i32]
        for nm in ("lco_forward_z8", "lco_forward_zf", "lco_forward_packed"):
            getattr(L, nm).argtypes = [_vp, _i64, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _i32]
        for nm in ("lco_backward_z8", "lco_backward_zf"):
            getattr(L, nm).argtypes = [_vp, _vp, _i64, _vp, _vp, _i64, _i64, _i32, _vp, _vp,
                                       _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32]
        L.lco_ldlq_assign.argtypes = [_vp, _i64, _i64, _vp, _vp, _i32]
        L.lco_fit_affine.argtypes = [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp]
        L.lco_fit_affine_h.argtypes = [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp]
        for nm in ("lco_dge_phi", "lco_dge_derivative"):
            getattr(L, nm).argtypes = [_vp, _i64, ctypes.c_double, _vp]
            getattr(L, nm).restype = None
        for f in (L.lco_assign, L.lco_pack_codes, L.lco_decode_z8, L.lco_forward_z8,
                  L.lco_ldlq_assign, L.lco_fit_affine, L.lco_fit_affine_h):
            f.restype = None
        _lib = L
    return _lib


def default_threads() -> int:
    return os.cpu_count() or 1


def _p(a: np.ndarray):
    return a.ctypes.data_as(_vp)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _codes(z):
    """u8 codes pass as they are; anything else (the STE surrogate's clamped
    proxy weights) as fp64 values."""
    z = np.asarray(z)
    if z.dtype == np.uint8:
        return np.ascontiguousarray(z), "z8"
    return _f64(z), "zf"


# ---------------------------------------------------------------- assign / pack
def assign(Wp):
    w = _f64(Wp)
    z = np.empty(w.shape, dtype=np.uint8)
    m = np.empty(w.shape, dtype=np.uint8)
    lib().lco_assign(_p(w), w.size, _p(z), _p(m))
    return z, m.astype(bool)


def pack_codes(z):
    z = np.ascontiguousarray(np.asarray(z, dtype=np.uint8))
    n, k = z.shape
    assert k % 4 == 0
    out = np.empty((n, k // 4), dtype=np.uint8)
    lib().lco_pack_codes(_p(z), n, k, _p(out))
    return out


def unpack_codes(packed, d_in: int):
    p = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    z = np.empty((p.shape[0], d_in), dtype=np.uint8)
    lib().lco_unpack_codes(_p(p), p.shape[0], d_in, _p(z))
    return z


def pack_mask(mask):
    m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    n, k = m.shape
    assert k % 8 == 0
    out = np.empty((n, k // 8), dtype=np.uint8)
    lib().lco_pack_mask(_p(m), n, k, _p(out))
    return out


def unpack_mask(bits, d_in: int):
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint8))
    m = np.empty((b.shape[0], d_in), dtype=np.uint8)
    lib().lco_unpack_mask(_p(b), b.shape[0], d_in, _p(m))
    return m.astype(bool)


# ---------------------------------------------------------------- decode / forward / backward
def decode(z, A, B, threads: int | None = None):
    A, B = _f64(A), _f64(B)
    d = A.shape[0]
    zz, kind = _codes(z)
    n, k = zz.shape
    W = np.empty((n, k))
    getattr(lib(), f"lco_decode_{kind}")(_p(zz), n, k, d, _p(A), _p(B), _p(W),
                                          threads or default_threads())
    return W


def forward(X, z, A, B, threads: int | None = None):
    """(Y, D_Y): Y[m, n] = sum_k X[m, k] W~[n, k], D_Y = sum_k |X| |W~|."""
    X, A, B = _f64(X), _f64(A), _f64(B)
    d = A.shape[0]
    zz, kind = _codes(z)
    n, k = zz.shape
    M = X.shape[0]
    assert X.shape[1] == k
    Y = np.empty((M, n))
    D = np.empty((M, n))
    getattr(lib(), f"lco_forward_{kind}")(_p(X), M, _p(zz), n, k, d, _p(A), _p(B), _p(Y), _p(D),
                                           threads or default_threads())
    return Y, D


def forward_packed(X, packed, d_in: int, A, B, threads: int | None = None):
    """forward() with the codes given in format V1 ``[d_out][d_in/4]`` (the
    oracle's own unpacking, row by row)."""
    X, A, B = _f64(X), _f64(A), _f64(B)
    d = A.shape[0]
    p = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    n = p.shape[0]
    assert p.shape[1] * 4 == d_in and X.shape[1] == d_in
    M = X.shape[0]
    Y = np.empty((M, n))
    D = np.empty((M, n))
    lib().lco_forward_packed(_p(X), M, _p(p), n, d_in, d, _p(A), _p(B), _p(Y), _p(D),
                             threads or default_threads())
    return Y, D


def backward(X, dY, z, mask, A, B, threads: int | None = None):
    """dX, dA, dB, dWp of the straight-through backward and their normalisers
    (keys as the numpy oracle's)."""
    X, dY, A, B = _f64(X), _f64(dY), _f64(A), _f64(B)
    d = A.shape[0]
    zz, kind = _codes(z)
    n, k = zz.shape
    M = X.shape[0]
    mk = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    out = dict(dX=np.empty((M, k)), D_dX=np.empty((M, k)), dA=np.empty((d, d)),
               D_dA=np.empty((d, d)), dB=np.empty(d), D_dB=np.empty(d), dWp=np.empty((n, k)),
               D_dWp=np.empty((n, k)))
    getattr(lib(), f"lco_backward_{kind}")(
        _p(X), _p(dY), M, _p(zz), _p(mk), n, k, d, _p(A), _p(B), _p(out["dX"]), _p(out["D_dX"]),
        _p(out["dA"]), _p(out["D_dA"]), _p(out["dB"]), _p(out["D_dB"]), _p(out["dWp"]),
        _p(out["D_dWp"]), threads or default_threads())
    return out


# ---------------------------------------------------------------- H-aware sequential assignment
def ldlq_assign(P, U, threads: int | None = None):
    """Codes Z (u8, N x K) of the sequential rule, every row of the targets P
    (N x K) on its own, elements in increasing k; only the strictly upper
    triangle of U (K x K) is read."""
    P, U = _f64(P), _f64(U)
    n, k = P.shape
    assert U.shape == (k, k)
    Z = np.empty((n, k), dtype=np.uint8)
    lib().lco_ldlq_assign(_p(P), n, k, _p(U), _p(Z), threads or default_threads())
    return Z


# ---------------------------------------------------------------- least-squares refits of (A, B)
def fit_affine(W0, z, d: int, h=None):
    """(A, B) minimizing sum_n sum_k h_k (W0[n, k] - W~[n, k])^2 given the codes
    (h = 1 when None); the minimum-norm solution where a Gram is singular."""
    W0 = _f64(W0)
    zz = np.ascontiguousarray(np.asarray(z, dtype=np.uint8))
    n, k = W0.shape
    hv = None if h is None else _f64(h)
    A = np.empty((d, d))
    B = np.empty(d)
    lib().lco_fit_affine(_p(W0), _p(zz), n, k, d, None if hv is None else _p(hv), _p(A), _p(B))
    return A, B


def fit_affine_h(W0, z, d: int, H):
    """(A, B) minimizing sum_n (W~[n] - W0[n])^T H (W~[n] - W0[n]) given the codes."""
    W0, H = _f64(W0), _f64(H)
    zz = np.ascontiguousarray(np.asarray(z, dtype=np.uint8))
    n, k = W0.shape
    assert H.shape == (k, k)
    A = np.empty((d, d))
    B = np.empty(d)
    lib().lco_fit_affine_h(_p(W0), _p(zz), n, k, d, _p(H), _p(A), _p(B))
    return A, B


# ---------------------------------------------------------------- DGE curve (a reading)
def dge_phi(w, k):
    """The smooth rounding curve phi_k on [0, 3] (clamped outside)."""
    x = _f64(w)
    out = np.empty(x.shape)
    lib().lco_dge_phi(_p(x), x.size, float(k), _p(out))
    return out


def dge_derivative(Wp, k):
    """phi_k'(Wp): the factor DGE puts where the STE puts the clamp mask."""
    x = _f64(Wp)
    out = np.empty(x.shape)
    lib().lco_dge_derivative(_p(x), x.size, float(k), _p(out))
    return out

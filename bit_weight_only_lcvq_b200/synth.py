"""Seeded synthetic inputs for the LC-VQ workloads.

This module only draws random numbers and shapes them into the five
workloads; it holds none of the method's arithmetic (no rounding to codes,
no packing, no decode, no matmul).  Both the fp64 oracle (through the tests)
and the CUDA path (through the tests and the benchmark) take their inputs
from here, so both sides always see the same bytes.

Every tensor has its own stream: ``numpy.random.PCG64`` seeded with
``0x1C0A0000 + 16 * workload + tensor_id``.  Floating inputs are drawn in
fp64, then rounded once to the storage type (fp32, or bf16 with
round-to-nearest-even).  bf16 tensors are returned as fp32 arrays whose
values are exactly representable in bf16; :func:`bf16_bits` gives the raw
16-bit patterns the GPU consumes.

Workloads (shapes in storage order: weights ``[d_out][d_in]``,
activations ``[M][d_in]``):

1. ``single_layer``  d_in=d_out=512, d=4, M=16, fp32.
2. ``decode_gemv``   d_in=d_out=4096, d=8, M in {1,4,16}, bf16 X with 1% of
   input channels scaled by 20.
3. ``prefill``       d_in=4096, d_out=11008, d=8, M=2048, bf16.
4. ``qat_step``      d_in=14336, d_out=4096, d=8, M=8192, bf16, W_p ~ N(1.5,1),
   dY ~ N(0, 0.1^2).
5. ``stack``         32 layers x {q,k,v,o 4096x4096; gate,up 4096->11008;
   down 11008->4096}, d=8, random packed codes, M in {1,8,32}.
"""

from __future__ import annotations

import numpy as np

SEED_BASE = 0x1C0A0000

# tensor ids inside one workload
T_WP, T_A, T_X, T_DY, T_OUTLIER, T_CODES = 0, 1, 2, 3, 4, 5

WORKLOADS = {
    1: dict(name="single_layer", d_in=512, d_out=512, d=4, M=(16,), dtype="f32"),
    2: dict(name="decode_gemv", d_in=4096, d_out=4096, d=8, M=(1, 4, 16), dtype="bf16"),
    3: dict(name="prefill", d_in=4096, d_out=11008, d=8, M=(2048,), dtype="bf16"),
    4: dict(name="qat_step", d_in=14336, d_out=4096, d=8, M=(8192,), dtype="bf16"),
    5: dict(name="stack", d=8, M=(1, 8, 32), dtype="bf16", layers=32),
}

# (name, d_in, d_out) of one decoder layer of the 7B-shaped stack
STACK_PROJS = (
    ("q", 4096, 4096),
    ("k", 4096, 4096),
    ("v", 4096, 4096),
    ("o", 4096, 4096),
    ("gate", 4096, 11008),
    ("up", 4096, 11008),
    ("down", 11008, 4096),
)


def rng(workload: int, tensor_id: int, sub: int = 0) -> np.random.Generator:
    """Independent stream for one tensor of one workload (``sub`` separates
    the matrices of the stack)."""
    seed = SEED_BASE + 16 * workload + tensor_id + (sub << 32)
    return np.random.Generator(np.random.PCG64(seed))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to the nearest bf16 value (ties to even) and
    return it as fp32.  Finite inputs only."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of an fp32 array whose values are
    already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("array holds values that are not bf16-representable")
    return (u >> np.uint32(16)).astype(np.uint16)


def from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """fp32 values of raw bf16 bit patterns (exact widening)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def _store(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    return round_to_bf16(x32) if dtype == "bf16" else x32


def affine_single_layer(d: int, g: np.random.Generator):
    """A = 0.02 (I + 0.1 N(0,1) off-diagonal), B = -1.5 A 1 (fp64, then fp32)."""
    off = 0.1 * g.standard_normal((d, d))
    np.fill_diagonal(off, 0.0)
    A = 0.02 * (np.eye(d) + off)
    B = -1.5 * A.sum(axis=1)
    return A.astype(np.float32), B.astype(np.float32)


def affine_diag_dominant(d: int, g: np.random.Generator):
    """A = diag(0.02 |N(1, 0.2)|) + 0.002 N(0,1) off-diagonal, B = -1.5 A 1."""
    diag = 0.02 * np.abs(g.normal(1.0, 0.2, size=d))
    off = 0.002 * g.standard_normal((d, d))
    np.fill_diagonal(off, 0.0)
    A = np.diag(diag) + off
    B = -1.5 * A.sum(axis=1)
    return A.astype(np.float32), B.astype(np.float32)


def wp_uniform(d_out: int, d_in: int, g: np.random.Generator) -> np.ndarray:
    """Proxy weights ~ U[-0.5, 3.5] (uniform codes), fp32 ``[d_out][d_in]``."""
    return g.uniform(-0.5, 3.5, size=(d_out, d_in)).astype(np.float32)


def wp_normal(d_out: int, d_in: int, g: np.random.Generator) -> np.ndarray:
    """Proxy weights ~ N(1.5, 1), fp32 ``[d_out][d_in]``."""
    return g.normal(1.5, 1.0, size=(d_out, d_in)).astype(np.float32)


def x_outliers(M: int, d_in: int, g_x: np.random.Generator, g_ch: np.random.Generator,
               dtype: str = "bf16") -> np.ndarray:
    """X ~ N(0,1) with round(0.01 d_in) input channels (a seeded choice)
    scaled by 20 before the cast to the storage type."""
    x = g_x.standard_normal((M, d_in))
    n_out = int(round(0.01 * d_in))
    ch = g_ch.permutation(d_in)[:n_out]
    x[:, ch] *= 20.0
    return _store(x, dtype)


def normal(shape, std: float, g: np.random.Generator, dtype: str) -> np.ndarray:
    return _store(std * g.standard_normal(shape), dtype)


def random_packed(d_out: int, d_in: int, g: np.random.Generator) -> np.ndarray:
    """Uniformly random packed code bytes ``[d_out][d_in/4]`` (4 codes/byte)."""
    return g.integers(0, 256, size=(d_out, d_in // 4), dtype=np.uint8)


def workload(wid: int, M: int | None = None, *, d_in: int | None = None,
             d_out: int | None = None, d: int | None = None, with_dy: bool = True) -> dict:
    """Inputs of workload ``wid`` (1..4).  Shapes may be overridden to build
    small cases with the same distributions.

    Returns a dict with Wp (fp32), A, B (fp32), X (fp32 holding bf16 values
    when the workload is bf16), dY (same), and the metadata.
    """
    spec = WORKLOADS[wid]
    d_in = d_in or spec["d_in"]
    d_out = d_out or spec["d_out"]
    d = d or spec["d"]
    M = M if M is not None else spec["M"][-1]
    dt = spec["dtype"]
    out = dict(wid=wid, d_in=d_in, d_out=d_out, d=d, M=M, dtype=dt)
    if wid == 1:
        out["Wp"] = wp_uniform(d_out, d_in, rng(1, T_WP))
        out["A"], out["B"] = affine_single_layer(d, rng(1, T_A))
        out["X"] = normal((M, d_in), 1.0, rng(1, T_X), dt)
        if with_dy:
            out["dY"] = normal((M, d_out), 0.1, rng(1, T_DY), dt)
        return out
    if wid in (2, 3):
        out["Wp"] = wp_uniform(d_out, d_in, rng(wid, T_WP))
    elif wid == 4:
        out["Wp"] = wp_normal(d_out, d_in, rng(4, T_WP))
    else:
        raise ValueError("workload 5 is built by stack_layer()")
    out["A"], out["B"] = affine_diag_dominant(d, rng(wid, T_A))
    out["X"] = x_outliers(M, d_in, rng(wid, T_X), rng(wid, T_OUTLIER), dt)
    if with_dy:
        out["dY"] = normal((M, d_out), 0.1, rng(wid, T_DY), dt)
    return out


def stack_matrix(layer: int, proj: int, M: int, *, with_x: bool = True) -> dict:
    """One matrix of the 7B-shaped stack: random packed codes, its own A/B
    (diagonal-dominant recipe) and its own X (outlier recipe)."""
    name, d_in, d_out = STACK_PROJS[proj]
    sub = 1 + layer * len(STACK_PROJS) + proj
    out = dict(layer=layer, proj=name, d_in=d_in, d_out=d_out, d=8, M=M)
    out["packed"] = random_packed(d_out, d_in, rng(5, T_CODES, sub))
    out["A"], out["B"] = affine_diag_dominant(8, rng(5, T_A, sub))
    if with_x:
        out["X"] = x_outliers(M, d_in, rng(5, T_X, sub), rng(5, T_OUTLIER, sub), "bf16")
    return out


def ldlq_workload(d_out: int = 4096, d_in: int = 4096, d: int = 8, n_cal: int | None = None,
                  with_cal: bool = True) -> dict:
    """Inputs of the H-aware sequential assignment (workload id 6): code-space
    targets P ~ U[-0.5, 3.5] ``[d_out][d_in]`` (fp32), the matrix's A/B
    (diagonal-dominant recipe) and ``n_cal`` (default 2 d_in) calibration
    activation rows with the outlier recipe, fp32, from which the caller forms
    the input Hessian.  Sizes may be reduced for small cases with the same
    distributions."""
    n_cal = n_cal or 2 * d_in
    out = dict(d_in=d_in, d_out=d_out, d=d, n_cal=n_cal)
    out["P"] = wp_uniform(d_out, d_in, rng(6, T_WP))
    out["A"], out["B"] = affine_diag_dominant(d, rng(6, T_A))
    if with_cal:
        out["Xcal"] = x_outliers(n_cal, d_in, rng(6, T_X), rng(6, T_OUTLIER), "fp32")
    return out


def strict_upper_dyadic(K: int, g: np.random.Generator, step: float = 1.0 / 64,
                        limit: int = 4) -> np.ndarray:
    """A strictly upper triangular K x K fp32 matrix with entries that are
    multiples of ``step`` in [-limit step, limit step]: every product with a
    small dyadic error and every partial sum of a row is exact in fp32."""
    u = g.integers(-limit, limit + 1, size=(K, K)).astype(np.float64) * step
    return np.triu(u, 1).astype(np.float32)


def targets_dyadic(d_out: int, d_in: int, g: np.random.Generator, step: float = 1.0 / 32) -> np.ndarray:
    """Targets on a 1/32 grid in [-0.5, 3.5] (exact rounding ties included)."""
    return (g.integers(-16, 113, size=(d_out, d_in)).astype(np.float64) * step).astype(np.float32)

"""Helpers shared by the GPU tests: move synthetic inputs to the device and
compare device results with the oracle."""

import numpy as np
import torch

from oracle import lcvq_oracle as O

TOL_BF16 = 4e-3   # max |y - y_ref| / sum |x||w~| for bf16 activations
TOL_F32 = 1e-5    # same, fp32 activations


def dev():
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test run without a CUDA device")
    return torch.device("cuda:0")


def to_dev(a: np.ndarray, dtype) -> torch.Tensor:
    """Exact transfer: fp32 arrays holding bf16-representable values become
    bf16 without rounding."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(dtype).to(dev())


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def tol_for(dtype) -> float:
    return TOL_BF16 if dtype == torch.bfloat16 else TOL_F32


def assert_close(name, got, ref, D, tol):
    err = O.rel_err(got, ref, D)
    assert err <= tol, f"{name}: max rel err {err:.3e} > {tol:.1e}"
    return err


def ldlq_check(P, U, Z):
    """Validity of codes Z of the H-aware sequential assignment (computed in
    fp32): the oracle recomputes, in fp64, the target t_j that each code was
    rounded from, given the codes before it.  Every code must be
    clamp(rint(t_j), 0, 3), except where t_j lies within the fp32 error bound
    of a rounding boundary (0.5, 1.5, 2.5), where either neighbour is valid.
    The bound is (chain + 96) 2^-24 sum|terms|, chain = K/8 additions (the
    longest sum of one warp's share of the earlier blocks) plus the
    cross-warp sum and the in-block updates.  Returns (bad, near)."""
    P = np.asarray(P, dtype=np.float64)
    T, S = O.ldlq_targets(P, np.asarray(U, dtype=np.float64), Z)
    K = P.shape[1]
    tau = (K / 8 + 96) * 2.0 ** -24 * S
    ref = np.clip(np.rint(T), 0, 3)
    dist = np.abs(T - (np.floor(T) + 0.5))
    near = (dist <= tau) & (T > 0.5 - tau) & (T < 2.5 + tau)
    Zf = np.asarray(Z, dtype=np.float64)
    bad = ((Zf != ref) & ~near) | (np.abs(np.clip(T, 0, 3) - Zf) > 0.5 + tau)
    return int(bad.sum()), int(near.sum())


GUARD_BYTES = 4096     # guard on each side of a canaried output (keeps 256-byte alignment)
GUARD_FILL = 0xA5


def guarded(shape, dtype):
    """An output tensor of `shape` placed inside a larger buffer whose
    GUARD_BYTES on either side (and the output itself) are filled with the
    byte GUARD_FILL.  Returns (out, buf); guard_intact(out, buf) checks that a
    kernel writing `out` left every guard byte alone."""
    esz = torch.empty((), dtype=dtype).element_size()
    n = int(np.prod(shape))
    g = GUARD_BYTES // esz
    buf = torch.empty(n + 2 * g, dtype=dtype, device=dev())
    buf.view(torch.uint8).fill_(GUARD_FILL)
    return buf[g:g + n].view(shape), buf


def guard_intact(out, buf) -> bool:
    raw = buf.view(torch.uint8)
    nb = out.numel() * out.element_size()
    head, tail = raw[:GUARD_BYTES], raw[GUARD_BYTES + nb:]
    return bool(torch.all(head == GUARD_FILL)) and bool(torch.all(tail == GUARD_FILL))

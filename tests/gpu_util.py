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

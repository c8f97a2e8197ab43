"""The workspace-free decode-GEMV, lcvq_gemv_static, checked against lcvq_gemm.

Some callers cannot give the library a workspace: code that runs while a CUDA
graph is being captured (device allocation is not allowed there), runtimes
that reserve all device memory up front and forbid later allocations, and
extensions whose host framework owns the allocator but offers no scratch API.
lcvq_gemv_static serves them by keeping its scratch in a fixed array inside
the library.  It must give what the workspace path gives, on two calls in a
row: the second call runs on an array that still holds the first call's data.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from bit_weight_only_lcvq_b200 import lcvq, synth
from oracle import lcvq_oracle as O
from tests.gpu_util import TOL_BF16, dev

pytestmark = pytest.mark.gpu


def _case(M, d_in, d_out, d=8):
    w = synth.workload(2, M=M, d_in=d_in, d_out=d_out, d=d, with_dy=False)
    z, _ = O.assign(w["Wp"])
    t = dict(X=torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev()),
             packed=torch.from_numpy(O.pack_codes(z)).to(dev()),
             A=torch.from_numpy(w["A"]).to(dev()), B=torch.from_numpy(w["B"]).to(dev()))
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    return w, t, ref, D


def _static_call(t, M, d_out, d_in, Y, d=8):
    L = lcvq.lib()
    st = L.lcvq_gemv_static(t["X"].data_ptr(), M, t["packed"].data_ptr(), d_out, d_in, d,
                            t["A"].data_ptr(), t["B"].data_ptr(), Y.data_ptr(),
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


# (M, d_in, d_out, d): M = 32 fills the array's token rows; d = 4 changes the
# X-transform; the others span the split kernel's 16- and 32-row tiles
CASES = [(16, 4096, 4096, 8), (3, 1088, 520, 8), (32, 2048, 1032, 8), (9, 512, 264, 4)]


def test_static_scratch_matches_workspace_path_two_calls():
    """Each case is called twice in a row through the C ABI; the second call
    runs on an array that still holds the previous call's data.  Both must give
    lcvq_gemm's result (the same kernels, so the same bits) and lie within the
    forward tolerance of the oracle."""
    L = lcvq.lib()
    for M, d_in, d_out, d in CASES:
        w, t, ref, D = _case(M, d_in, d_out, d)
        Y_ref = lcvq.gemm(t["X"], t["packed"], d_in, t["A"], t["B"], d)
        for call in range(2):
            Y_static = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device=dev())
            assert _static_call(t, M, d_out, d_in, Y_static, d) == 0
            assert L.lcvq_last_launch_count() == 2
            torch.cuda.synchronize()
            err = O.rel_err(Y_static.double().cpu().numpy(), Y_ref.double().cpu().numpy(), D)
            assert err <= TOL_BF16, f"M={M} call {call}: static vs workspace path rel err {err:.3e}"
            assert torch.equal(Y_static, Y_ref), f"M={M} d={d} call {call}: bits differ"
            err = O.rel_err(Y_static.double().cpu().numpy(), ref, D)
            assert err <= TOL_BF16, f"M={M} call {call}: static vs oracle rel err {err:.3e}"


def test_static_scratch_rejects_sizes_beyond_the_array():
    w, t, _, _ = _case(4, 512, 64)
    Y = torch.zeros((40, 64), dtype=torch.bfloat16, device=dev())
    L = lcvq.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # M > 32 and d_in > 32768 are refused before anything is launched
    assert L.lcvq_gemv_static(t["X"].data_ptr(), 33, t["packed"].data_ptr(), 64, 512, 8,
                              t["A"].data_ptr(), t["B"].data_ptr(), Y.data_ptr(), s) == 4
    assert L.lcvq_gemv_static(t["X"].data_ptr(), 4, t["packed"].data_ptr(), 64, 32768 + 64, 8,
                              t["A"].data_ptr(), t["B"].data_ptr(), Y.data_ptr(), s) == 4
    # a d_out beyond lcvq_gemm's bound is an invalid argument, as there
    assert L.lcvq_gemv_static(t["X"].data_ptr(), 4, t["packed"].data_ptr(), (1 << 30) + 8, 512, 8,
                              t["A"].data_ptr(), t["B"].data_ptr(), Y.data_ptr(), s) == 1
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y) == 0

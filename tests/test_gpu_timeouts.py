"""Bounded waits, exercised on the GPU without a fault.

A workspace's header holds the wait limit of the kernels that wait on
mbarriers.  Lowered to a few dozen clock cycles, the waits give up: the call
must still return, the kernel must wind down (no hang: the test's
synchronize returns), lcvq_check_device_error must report
LCVQ_ERR_DEVICE_TIMEOUT with the site of a wait of that kernel, and the next
call on the same workspace, with the default limit, must be correct again.
Nothing here traps or touches memory out of bounds: the waits simply stop
early, as a stuck producer would make them.
"""

import numpy as np
import pytest
import torch

from bit_weight_only_lcvq_b200 import lcvq, synth
from oracle import lcvq_oracle as O
from tests.gpu_util import TOL_BF16, assert_close, dev, to_dev, to_np

pytestmark = pytest.mark.gpu

TIMEOUT = 6          # LCVQ_ERR_DEVICE_TIMEOUT
SHORT_LIMIT = 64     # clock cycles: far below one TMA round trip


def _header(ws):
    torch.cuda.synchronize()
    h = ws[:8].view(torch.int32).cpu().tolist()
    return h[0], h[1]


def _force_timeout_then_recover(run, ws, sites):
    lcvq.set_wait_limit(ws, SHORT_LIMIT)
    run()
    err, site = _header(ws)
    assert err == TIMEOUT and site in sites, (err, site)
    assert lcvq.check_device_error(ws) == TIMEOUT
    assert _header(ws) == (0, 0)  # cleared
    lcvq.set_wait_limit(ws, 0)
    out = run()
    assert lcvq.check_device_error(ws) == 0
    return out


def test_tcgen05_gemm_wait_gives_up_and_recovers():
    """Algebraic-form prefill GEMM (single-CTA tcgen05 kernel, M = 200)."""
    w = synth.workload(3, M=200, d_in=512, d_out=520, with_dy=False)
    z, _ = O.assign(w["Wp"])
    X = to_dev(w["X"], torch.bfloat16)
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, 200, 520, 512, 8))
    Y = _force_timeout_then_recover(
        lambda: lcvq.gemm(X, packed, 512, A, B, 8, form="algebraic", workspace=ws), ws,
        sites={1, 2, 3, 4, 5, 6})
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close("gemm after a timeout", to_np(Y), ref, D, TOL_BF16)


def _group(M, seed):
    shapes = [(4096, 4096)] * 10
    jobs, zs, ws_ = [], [], []
    g = np.random.Generator(np.random.PCG64(seed))
    for i, (d_in, d_out) in enumerate(shapes):
        w = synth.workload(2, M=M, d_in=d_in, d_out=d_out, with_dy=False)
        z = g.integers(0, 4, size=(d_out, d_in), dtype=np.uint8)
        jobs.append((to_dev(w["X"], torch.bfloat16), torch.from_numpy(O.pack_codes(z)).to(dev()),
                     torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev()), d_in))
        zs.append(z)
        ws_.append(w)
    return jobs, zs, ws_


@pytest.mark.parametrize("M,sites", [(4, {50, 51, 52}), (32, {60, 61, 62, 63, 64, 65, 66})])
def test_grouped_gemv_wait_gives_up_and_recovers(M, sites):
    """Grouped decode-GEMV of 10 matrices of 4096 x 4096 (320 tiles of 128
    rows): the wide-tile mma.sync kernel at M = 4, the tcgen05 kernel at
    M = 32."""
    jobs, zs, ws_ = _group(M, 2600 + M)
    ws = lcvq.new_workspace(lcvq.workspace_size_grouped(jobs, M, 8))
    outs = [torch.empty((M, 4096), dtype=torch.bfloat16, device=dev()) for _ in jobs]
    _force_timeout_then_recover(lambda: lcvq.gemm_grouped(jobs, 8, workspace=ws, outs=outs), ws,
                                sites)
    for i in (0, 9):
        ref, D = O.forward(ws_[i]["X"], zs[i], ws_[i]["A"], ws_[i]["B"])
        assert_close(f"grouped item {i} after a timeout", to_np(outs[i]), ref, D, TOL_BF16)

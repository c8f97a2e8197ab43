"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Codes, packed bytes and mask bits must match bit for bit; floating outputs
must meet max |y - y_ref| / sum|x||w~| <= 4e-3 (bf16 activations) or 1e-5
(fp32).  Shapes span several tiles and ragged tails; the full workload sizes
are covered in test_gpu_fullsize.py.
"""

import numpy as np
import pytest
import torch

from bit_weight_only_lcvq_b200 import lcvq, synth
from oracle import lcvq_oracle as O
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, dev, guard_intact, guarded, ldlq_check,
                            to_dev, to_np, tol_for)

pytestmark = pytest.mark.gpu


# --------------------------------------------------------------- assign/pack
def _adversarial_wp(n_rows, n_cols, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    w = g.uniform(-1.0, 4.0, size=(n_rows, n_cols)).astype(np.float32)
    special = np.array([0.5, 1.5, 2.5, 3.5, -0.5, -0.0, 0.0, 3.0, 3.0000002, -1e-45, 1e-45,
                        np.inf, -np.inf, np.nan, 1e30, -1e30, 0.49999997, 2.4999998,
                        np.float32(1.17549435e-38), 7.25], dtype=np.float32)
    flat = w.reshape(-1)
    idx = g.choice(flat.size, size=min(flat.size, 4 * special.size), replace=False)
    flat[idx] = np.resize(special, idx.size)
    return w


@pytest.mark.parametrize("shape", [(1, 8), (3, 40), (7, 64), (33, 520), (128, 4096), (5, 1032)])
def test_assign_pack_bit_exact(shape):
    Wp = _adversarial_wp(*shape, seed=shape[0] * 7 + shape[1])
    z, mask = O.assign(Wp)
    packed, pbuf = guarded((shape[0], shape[1] // 4), torch.uint8)
    mbits, mbuf = guarded((shape[0], shape[1] // 8), torch.uint8)
    lcvq.assign_pack(torch.from_numpy(Wp).to(dev()), d=8 if shape[1] % 8 == 0 else 4,
                     packed=packed, mask=mbits)
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(z))
    assert np.array_equal(mbits.cpu().numpy(), O.pack_mask(mask))
    assert guard_intact(packed, pbuf) and guard_intact(mbits, mbuf)


def test_assign_pack_workload_distributions():
    for wid in (2, 4):
        w = synth.workload(wid, M=1, d_in=1024, d_out=256, with_dy=False)
        z, mask = O.assign(w["Wp"])
        packed, mbits = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), d=8)
        assert np.array_equal(packed.cpu().numpy(), O.pack_codes(z))
        assert np.array_equal(mbits.cpu().numpy(), O.pack_mask(mask))


def test_assign_pack_without_mask():
    Wp = _adversarial_wp(16, 256, 3)
    z, _ = O.assign(Wp)
    packed, m = lcvq.assign_pack(torch.from_numpy(Wp).to(dev()), d=8, with_mask=False)
    assert m is None
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(z))


# --------------------------------------------------------------- decode
@pytest.mark.parametrize("d", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode(d, dtype):
    g = np.random.Generator(np.random.PCG64(100 + d))
    N, K = 40, 256
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A, B = synth.affine_diag_dominant(d, g)
    W, wbuf = guarded((N, K), dtype)
    lcvq.decode(torch.from_numpy(O.pack_codes(z)).to(dev()), K, torch.from_numpy(A).to(dev()),
                torch.from_numpy(B).to(dev()), d, out=W)
    ref = O.decode(z, A, B)
    D = O.decode_abs(z, A, B)
    tol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
    assert_close("decode", to_np(W), ref, D, tol)
    assert guard_intact(W, wbuf)


@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (37, 528), (128, 4096)])
def test_decode_d8_bf16_ragged_and_exact_zero(shape):
    """d = 8 to bf16 runs on the tensor cores: shapes whose vector count ends
    inside a warp's batch, and exact results where the pages' values are exact
    (zero codes with B = 0 give exact zeros)."""
    N, K = shape
    g = np.random.Generator(np.random.PCG64(110 + N))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    z[0, :8] = 0
    A, B = synth.affine_diag_dominant(8, g)
    B[:] = 0.0
    W, wbuf = guarded((N, K), torch.bfloat16)
    lcvq.decode(torch.from_numpy(O.pack_codes(z)).to(dev()), K, torch.from_numpy(A).to(dev()),
                torch.from_numpy(B).to(dev()), 8, out=W)
    ref = O.decode(z, A, B)
    assert_close("decode d=8", to_np(W), ref, O.decode_abs(z, A, B), 2.0 ** -8)
    assert np.all(to_np(W)[0, :8] == 0.0)
    assert guard_intact(W, wbuf)


# --------------------------------------------------------------- forward
def _fwd_case(wid, M, d_in, d_out, d=None, seed_shift=0):
    w = synth.workload(wid, M=M, d_in=d_in, d_out=d_out, d=d, with_dy=False)
    z, _ = O.assign(w["Wp"])
    return w, z


def _run_fwd(w, z, dtype, form="auto"):
    """lcvq_gemm into a canaried output: the bytes around Y stay untouched."""
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    X = to_dev(w["X"], dtype)
    A = torch.from_numpy(w["A"]).to(dev())
    B = torch.from_numpy(w["B"]).to(dev())
    Y, ybuf = guarded((X.shape[0], packed.shape[0]), dtype)
    lcvq.gemm(X, packed, w["d_in"], A, B, w["d"], form=form, out=Y)
    torch.cuda.synchronize()
    assert guard_intact(Y, ybuf), f"lcvq_gemm wrote outside Y (M={X.shape[0]}, form={form})"
    return Y


@pytest.mark.parametrize("M", [1, 2, 4, 5, 8, 13, 16, 27, 32])
def test_gemv_bf16_ragged(M):
    w, z = _fwd_case(2, M, d_in=1088, d_out=520)   # K = 17 x 64, N not a multiple of 128
    Y = _run_fwd(w, z, torch.bfloat16)
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close(f"gemv M={M}", to_np(Y), ref, D, TOL_BF16)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_gemv_bf16_decode_workload(M):
    """Decode-GEMV workload shape: d_in = d_out = 4096, d = 8."""
    w, z = _fwd_case(2, M, d_in=4096, d_out=4096)
    Y = _run_fwd(w, z, torch.bfloat16)
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close(f"gemv 4096 M={M}", to_np(Y), ref, D, TOL_BF16)


@pytest.mark.parametrize("d", [1, 2, 4])
def test_gemv_bf16_small_d(d):
    w, z = _fwd_case(2, 8, d_in=512, d_out=256, d=d)
    Y = _run_fwd(w, z, torch.bfloat16)
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close(f"gemv d={d}", to_np(Y), ref, D, TOL_BF16)


@pytest.mark.parametrize("M,d_in,d_out", [(33, 512, 264), (200, 512, 264), (300, 576, 520)])
def test_gemm_bf16_larger_m(M, d_in, d_out):
    """Tensor-core forms, including tiles ragged in M and in d_out (pairs of
    128-row halves), and an odd number of 64-wide k blocks."""
    w, z = _fwd_case(3, M, d_in=d_in, d_out=d_out)
    for form in ("auto", "decode", "algebraic"):
        Y = _run_fwd(w, z, torch.bfloat16, form)
        ref, D = O.forward(w["X"], z, w["A"], w["B"])
        assert_close(f"gemm M={M} {form}", to_np(Y), ref, D, TOL_BF16)


def test_gemm_decode_form_many_tiles_per_pair():
    """Decode form with more tiles than CTA pairs and 5 k blocks per tile, so
    some pairs run two tiles and the odd CTA's grouped "decoded" handover
    spans a tile boundary and ends on a partial group; ragged in d_out."""
    w, z = _fwd_case(3, 512, d_in=320, d_out=41 * 256 - 40)
    Y = _run_fwd(w, z, torch.bfloat16, "decode")
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close("gemm decode form, 82 tiles", to_np(Y), ref, D, TOL_BF16)


def test_gemm_f32_single_layer():
    """fp32 single-layer workload (d_in = d_out = 512, d = 4, M = 16)."""
    w, z = _fwd_case(1, 16, d_in=512, d_out=512)
    Y = _run_fwd(w, z, torch.float32)
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close("gemm f32", to_np(Y), ref, D, TOL_F32)


def test_gemm_f32_identity_is_exact():
    """A = I, B = 0, small-integer X: Y = X Z^T is exact in fp32."""
    g = np.random.Generator(np.random.PCG64(5))
    M, N, K, d = 37, 72, 256, 8
    X = g.integers(-8, 9, size=(M, K)).astype(np.float32)
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    Y = lcvq.gemm(torch.from_numpy(X).to(dev()), torch.from_numpy(O.pack_codes(z)).to(dev()), K,
                  torch.eye(d, device=dev()), torch.zeros(d, device=dev()), d)
    assert np.array_equal(Y.cpu().numpy(), (X.astype(np.int64) @ z.astype(np.int64).T).astype(np.float32))


@pytest.mark.parametrize("M,dtype", [(4, torch.bfloat16), (16, torch.float32), (64, torch.bfloat16)])
def test_gemm_pow2_scaling_bit_exact(M, dtype):
    """Y(2^k A, 2^k B) = 2^k Y(A, B) bit for bit."""
    w, z = _fwd_case(2, M, d_in=512, d_out=256)
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    X = to_dev(w["X"], dtype)
    A = torch.from_numpy(w["A"]).to(dev())
    B = torch.from_numpy(w["B"]).to(dev())
    Y1 = lcvq.gemm(X, packed, 512, A, B, 8)
    Y8 = lcvq.gemm(X, packed, 512, 8 * A, 8 * B, 8)
    assert torch.equal(Y8, 8 * Y1)


def test_gemm_linearity():
    w, z = _fwd_case(2, 16, d_in=512, d_out=256)
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    X = to_dev(w["X"], torch.float32)
    g = np.random.Generator(np.random.PCG64(9))
    A2, B2 = synth.affine_diag_dominant(8, g)
    A1 = torch.from_numpy(w["A"]).to(dev())
    B1 = torch.from_numpy(w["B"]).to(dev())
    A2t, B2t = torch.from_numpy(A2).to(dev()), torch.from_numpy(B2).to(dev())
    Y1 = lcvq.gemm(X, packed, 512, A1, B1, 8).double()
    Y2 = lcvq.gemm(X, packed, 512, A2t, B2t, 8).double()
    Y12 = lcvq.gemm(X, packed, 512, A1 + A2t, B1 + B2t, 8).double()
    _, D = O.forward(w["X"], z, np.abs(w["A"]) + np.abs(A2), np.abs(w["B"]) + np.abs(B2))
    assert O.rel_err(to_np(Y12), to_np(Y1 + Y2), D) < 1e-5


def test_gemm_empty_and_zero_k():
    A = torch.eye(8, device=dev())
    B = torch.zeros(8, device=dev())
    X = torch.zeros((0, 64), dtype=torch.bfloat16, device=dev())
    packed = torch.zeros((16, 16), dtype=torch.uint8, device=dev())
    Y = lcvq.gemm(X, packed, 64, A, B, 8)
    assert Y.shape == (0, 16)
    X = torch.ones((3, 0), dtype=torch.bfloat16, device=dev())
    packed = torch.zeros((16, 0), dtype=torch.uint8, device=dev())
    Y = torch.full((3, 16), 7.0, dtype=torch.bfloat16, device=dev())
    lcvq.gemm(X, packed, 0, A, B, 8, out=Y)
    assert torch.count_nonzero(Y) == 0


def test_gemm_deterministic():
    w, z = _fwd_case(2, 16, d_in=4096, d_out=1024)
    Y1 = _run_fwd(w, z, torch.bfloat16)
    Y2 = _run_fwd(w, z, torch.bfloat16)
    assert torch.equal(Y1, Y2)


# --------------------------------------------------------------- backward
def _bwd_case(wid, M, d_in, d_out, dtype, d=None):
    w = synth.workload(wid, M=M, d_in=d_in, d_out=d_out, d=d)
    z, mask = O.assign(w["Wp"])
    packed, mbits = O.pack_codes(z), O.pack_mask(mask)
    args = dict(X=to_dev(w["X"], dtype), dY=to_dev(w["dY"], dtype),
                packed=torch.from_numpy(packed).to(dev()), mask=torch.from_numpy(mbits).to(dev()),
                A=torch.from_numpy(w["A"]).to(dev()), B=torch.from_numpy(w["B"]).to(dev()))
    return w, z, mask, args


def _check_bwd(w, z, mask, out, tol, tag):
    ref = O.backward(w["X"], w["dY"], z, mask, w["A"], w["B"])
    assert_close(f"{tag} dX", to_np(out["dX"]), ref["dX"], ref["D_dX"], tol)
    assert_close(f"{tag} dA", to_np(out["dA"]), ref["dA"], ref["D_dA"], tol)
    assert_close(f"{tag} dB", to_np(out["dB"]), ref["dB"], ref["D_dB"], tol)
    assert_close(f"{tag} dWp", to_np(out["dWp"]), ref["dWp"], ref["D_dWp"], tol)


def test_backward_f32_single_layer():
    w, z, mask, a = _bwd_case(1, 16, 512, 512, torch.float32)
    dX, xbuf = guarded((16, 512), torch.float32)
    dWp, wbuf = guarded((512, 512), torch.float32)
    out = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 512, a["A"], a["B"], 4,
                             outs=dict(dX=dX, dWp=dWp))
    torch.cuda.synchronize()
    assert guard_intact(dX, xbuf) and guard_intact(dWp, wbuf)
    _check_bwd(w, z, mask, out, TOL_F32, "f32")


@pytest.mark.parametrize("M,d_in,d_out", [(37, 576, 264), (200, 1024, 512)])
def test_backward_bf16(M, d_in, d_out):
    """bf16 backward on ragged shapes, into canaried dX and dWp."""
    w, z, mask, a = _bwd_case(4, M, d_in, d_out, torch.bfloat16)
    dX, xbuf = guarded((M, d_in), torch.bfloat16)
    dWp, wbuf = guarded((d_out, d_in), torch.float32)
    out = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], d_in, a["A"], a["B"], 8,
                             outs=dict(dX=dX, dWp=dWp))
    torch.cuda.synchronize()
    assert guard_intact(dX, xbuf) and guard_intact(dWp, wbuf)
    _check_bwd(w, z, mask, out, TOL_BF16, f"bf16 M={M}")


@pytest.mark.parametrize("d", [1, 2, 4])
def test_backward_small_d(d):
    w, z, mask, a = _bwd_case(4, 24, 256, 128, torch.float32, d=d)
    out = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 256, a["A"], a["B"], d)
    _check_bwd(w, z, mask, out, TOL_F32, f"d={d}")


def test_backward_optional_outputs_and_determinism():
    w, z, mask, a = _bwd_case(4, 64, 512, 256, torch.bfloat16)
    o1 = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 512, a["A"], a["B"], 8,
                            want_dx=False, want_dwp=False)
    o2 = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 512, a["A"], a["B"], 8)
    o3 = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 512, a["A"], a["B"], 8)
    assert o1["dX"] is None and o1["dWp"] is None
    assert torch.equal(o1["dA"], o2["dA"]) and torch.equal(o1["dB"], o2["dB"])
    for k in ("dX", "dA", "dB", "dWp"):
        assert torch.equal(o2[k], o3[k]), k


def test_backward_empty_tokens():
    a = dict(X=torch.zeros((0, 64), dtype=torch.bfloat16, device=dev()),
             dY=torch.zeros((0, 16), dtype=torch.bfloat16, device=dev()),
             packed=torch.zeros((16, 16), dtype=torch.uint8, device=dev()),
             mask=torch.zeros((16, 8), dtype=torch.uint8, device=dev()))
    A, B = torch.eye(8, device=dev()), torch.zeros(8, device=dev())
    outs = dict(dA=torch.ones((8, 8), device=dev()), dB=torch.ones(8, device=dev()),
                dWp=torch.ones((16, 64), device=dev()))
    o = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 64, A, B, 8, outs=outs)
    assert torch.count_nonzero(o["dA"]) == 0 and torch.count_nonzero(o["dB"]) == 0
    assert torch.count_nonzero(o["dWp"]) == 0


def test_launch_count_and_error_word():
    w, z = _fwd_case(2, 4, d_in=512, d_out=256)
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, 4, 256, 512, 8))
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    lcvq.gemm(to_dev(w["X"], torch.bfloat16), packed, 512, torch.from_numpy(w["A"]).to(dev()),
              torch.from_numpy(w["B"]).to(dev()), 8, workspace=ws)
    assert lcvq.last_launch_count() >= 1
    assert lcvq.check_device_error(ws) == 0


# ------------------------------------------------ grouped decode-GEMV (M <= 32)
def _group_case(shapes, M, seed):
    jobs, zs, ws = [], [], []
    for i, (d_in, d_out) in enumerate(shapes):
        w, z = _fwd_case(2, M, d_in=d_in, d_out=d_out)
        g = np.random.Generator(np.random.PCG64(seed + i))
        z = g.integers(0, 4, size=z.shape, dtype=np.uint8)   # a different code matrix per item
        jobs.append((to_dev(w["X"], torch.bfloat16), torch.from_numpy(O.pack_codes(z)).to(dev()),
                     torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev()), d_in))
        zs.append(z)
        ws.append(w)
    return jobs, zs, ws


@pytest.mark.parametrize("M", [1, 5, 16, 32])
def test_gemm_grouped_bitwise_equals_separate_calls(M):
    """Each Y_i of lcvq_gemm_grouped equals lcvq_gemm on item i alone, bit for
    bit, for mixed shapes (square, up-, down-projection, ragged); at M = 1 both
    take the int8 path, and every item also meets the oracle there."""
    shapes = [(4096, 4096), (4096, 11008), (11008, 4096), (1088, 520), (512, 8)]
    jobs, zs, ws = _group_case(shapes, M, 300 + M)
    Ys = lcvq.gemm_grouped(jobs, 8)
    assert lcvq.last_launch_count() == 2
    for i, (job, Y) in enumerate(zip(jobs, Ys)):
        X, packed, A, B, d_in = job
        Y1 = lcvq.gemm(X, packed, d_in, A, B, 8)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y1)
        if M <= 4:
            ref, D = O.forward(ws[i]["X"], zs[i], ws[i]["A"], ws[i]["B"])
            assert_close(f"grouped int8 item {i} M={M}", to_np(Y), ref, D, TOL_BF16)
    # and the small items against the oracle
    for i in (3, 4):
        ref, D = O.forward(ws[i]["X"], zs[i], ws[i]["A"], ws[i]["B"])
        assert_close(f"grouped item {i} M={M}", to_np(Ys[i]), ref, D, TOL_BF16)


def test_gemm_grouped_many_items_and_graph_replay():
    """More items than one launch takes (two chunks), one workspace, eager and
    as CUDA-graph replays."""
    shapes = [(64 * (1 + i % 5), 8 * (1 + i % 7)) for i in range(150)]
    jobs, zs, ws = _group_case(shapes, 3, 900)
    wsb = lcvq.new_workspace(lcvq.workspace_size_grouped(jobs, 3, 8))
    outs = [torch.empty((3, p.shape[0]), dtype=torch.bfloat16, device=dev()) for _, p, _, _, _ in jobs]
    lcvq.gemm_grouped(jobs, 8, workspace=wsb, outs=outs)
    assert lcvq.last_launch_count() == 4
    torch.cuda.synchronize()
    refs = [o.clone() for o in outs]
    for i in (0, 77, 149):
        ref, D = O.forward(ws[i]["X"], zs[i], ws[i]["A"], ws[i]["B"])
        assert_close(f"grouped many item {i}", to_np(outs[i]), ref, D, TOL_BF16)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        lcvq.gemm_grouped(jobs, 8, workspace=wsb, outs=outs)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lcvq.gemm_grouped(jobs, 8, workspace=wsb, outs=outs)
    for _ in range(3):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert all(torch.equal(o, r) for o, r in zip(outs, refs))
    del g
    assert lcvq.check_device_error(wsb) == 0


@pytest.mark.parametrize("M", [1, 3, 8, 16])
def test_gemm_grouped_wide_tiles_bitwise_equal_separate_calls(M):
    """A group large enough for the wide-tile kernel (>= 296 tiles of 128 rows;
    one producer warp streams codes and X'' into a shared-memory ring) gives
    the split kernel's bits (lcvq_gemm on the item alone; the int8 path for
    M <= 4); the group includes a ragged row count and a K that ends inside a
    chunk."""
    shapes = [(4096, 4096)] * 9 + [(1088, 1000), (11008, 4096)]
    jobs, zs, ws = _group_case(shapes, M, 700 + M)
    wsb = lcvq.new_workspace(lcvq.workspace_size_grouped(jobs, M, 8))
    Ys = lcvq.gemm_grouped(jobs, 8, workspace=wsb)
    assert lcvq.last_launch_count() == 2
    assert lcvq.check_device_error(wsb) == 0
    for i, (job, Y) in enumerate(zip(jobs, Ys)):
        X, packed, A, B, d_in = job
        Y1 = lcvq.gemm(X, packed, d_in, A, B, 8)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y1), f"item {i}"
    ref, D = O.forward(ws[9]["X"], zs[9], ws[9]["A"], ws[9]["B"])
    assert_close(f"wide grouped ragged item M={M}", to_np(Ys[9]), ref, D, TOL_BF16)


# --------------------------------------------- least-squares refit of (A, B)
# Error bound of the GPU fit.  Its per-lane sums run in fp32 and are flushed
# into fp64 every 16 terms, each term carrying at most 2 roundings, so an entry
# of R (and of G when weighted; unweighted G is an exact integer count) is off
# by at most 18 * 2^-24 of the sum of its terms' absolute values.  To first
# order, theta = G^+ R moves by |G^+| (|dR| + |dG| |theta|); the result is then
# rounded to fp32 (2^-24 relative).  The oracle supplies G, R and the
# absolute-term sums, so the bound is computed, not guessed.
def _fit_bound(W0, z, d, h, A_ref, B_ref):
    G, R = O.fit_affine_normal(np.abs(W0), z, d, h)   # G's terms are >= 0: G is its own |sum|
    th = np.concatenate([A_ref, B_ref[:, None]], axis=1)   # [d][d+1]
    # per-term rounding of the GPU's sums, relative to their absolute sums: the
    # 2^-22 of the tf32 hi/lo split of W0 (d = 8), up to 14 2^-24 inside one
    # tensor-core sum of 8 products, and the fp32 additions before the fp64
    # flush every 16 terms; 24 2^-24 covers every path
    eps = 24 * 2.0 ** -24
    bnd = np.zeros_like(th)
    for i in range(d):
        dR = eps * R[i]
        dG = eps * G[i] if h is not None else 0.0 * G[i]
        Pinv = np.abs(np.linalg.pinv(G[i], rcond=O.PINV_RCOND, hermitian=True))
        bnd[i] = Pinv @ (dR + dG @ np.abs(th[i])) + 2.0 ** -24 * np.abs(th[i])
    return bnd + 1e-12 * np.max(np.abs(th))


def _fit_ok(got_A, got_B, A, B, bound) -> bool:
    got = np.concatenate([to_np(got_A), to_np(got_B)[:, None]], axis=1)
    ref = np.concatenate([np.asarray(A, np.float64), np.asarray(B, np.float64)[:, None]], axis=1)
    return bool(np.all(np.abs(got - ref) <= bound))


@pytest.mark.parametrize("d", [1, 2, 4, 8])
@pytest.mark.parametrize("weighted", [False, True])
def test_fit_affine_matches_oracle(d, weighted):
    """GPU refit against the oracle's normal equations + pseudo-inverse, on a
    ragged shape (rows and vectors not multiples of the warp's vector count)."""
    g = np.random.Generator(np.random.PCG64(1100 + 10 * d + weighted))
    N, K = 77, 16 * 13
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A0, B0 = synth.affine_diag_dominant(d, g)
    W0 = (O.decode(z, A0, B0) + 0.01 * g.standard_normal((N, K))).astype(np.float32)
    h = g.uniform(0.1, 3.0, size=K).astype(np.float32) if weighted else None
    A_ref, B_ref = O.fit_affine(W0.astype(np.float64), z, d, None if h is None else h.astype(np.float64))
    A, B = lcvq.fit_affine(torch.from_numpy(W0).to(dev()), torch.from_numpy(O.pack_codes(z)).to(dev()),
                           d, h=None if h is None else torch.from_numpy(h).to(dev()))
    hb = None if h is None else h.astype(np.float64)
    assert _fit_ok(A, B, A_ref, B_ref, _fit_bound(W0.astype(np.float64), z, d, hb, A_ref, B_ref))


def test_fit_affine_singular_and_empty_and_deterministic():
    g = np.random.Generator(np.random.PCG64(1200))
    d, N, K = 8, 64, 256
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    z[:, 5::d] = 1                                   # position 5 never varies: G singular
    W0 = g.standard_normal((N, K)).astype(np.float32)
    A_ref, B_ref = O.fit_affine(W0.astype(np.float64), z, d)
    Wt, Pt = torch.from_numpy(W0).to(dev()), torch.from_numpy(O.pack_codes(z)).to(dev())
    A1, B1 = lcvq.fit_affine(Wt, Pt, d)
    A2, B2 = lcvq.fit_affine(Wt, Pt, d)
    torch.cuda.synchronize()
    assert torch.equal(A1, A2) and torch.equal(B1, B2)
    assert _fit_ok(A1, B1, A_ref, B_ref, _fit_bound(W0.astype(np.float64), z, d, None, A_ref, B_ref))
    Ae, Be = lcvq.fit_affine(torch.zeros((0, K), device=dev()),
                             torch.zeros((0, K // 4), dtype=torch.uint8, device=dev()), d)
    assert torch.count_nonzero(Ae) == 0 and torch.count_nonzero(Be) == 0


@pytest.mark.parametrize("M", [17, 32])
def test_gemm_grouped_tcgen05_form_matches_oracle(M):
    """Large groups with 17..32 tokens run on the tcgen05 tensor cores (decoded
    weights in TMEM, tokens as the MMA's N): within the forward tolerance of the
    oracle, and of separate lcvq_gemm calls, including a ragged row count and a
    K that ends inside a code chunk."""
    shapes = [(4096, 4096)] * 9 + [(1088, 1000), (11008, 4096)]
    jobs, zs, ws = _group_case(shapes, M, 1400 + M)
    wsb = lcvq.new_workspace(lcvq.workspace_size_grouped(jobs, M, 8))
    Ys = lcvq.gemm_grouped(jobs, 8, workspace=wsb)
    assert lcvq.check_device_error(wsb) == 0
    for i in (0, 9, 10):
        Xr = to_np(jobs[i][0])
        ref, D = O.forward(Xr, zs[i], ws[i]["A"], ws[i]["B"])
        assert_close(f"tcgen05 grouped item {i} M={M}", to_np(Ys[i]), ref, D, TOL_BF16)
        Y1 = lcvq.gemm(*jobs[i][:2], jobs[i][4], jobs[i][2], jobs[i][3], 8)
        assert_close(f"tcgen05 grouped vs single item {i} M={M}", to_np(Ys[i]), to_np(Y1), D, TOL_BF16)


# ------------------------------------------------------ DGE (curve is a reading)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("k", [0.01, 4.0])
def test_dge_scale_matches_oracle(dtype, k):
    """lcvq_gemm_backward's dWp rescaled by lcvq_dge_scale equals the oracle's
    DGE gradient (STE gradient times phi_k'(Wp)) within the backward tolerance;
    k = 0.01 is near the STE limit."""
    w, z, mask, a = _bwd_case(4, 32, 256, 128, dtype)
    out = lcvq.gemm_backward(a["X"], a["dY"], a["packed"], a["mask"], 256, a["A"], a["B"], 8)
    Wp = torch.from_numpy(w["Wp"]).to(dev())
    lcvq.dge_scale(out["dWp"], Wp, k)
    ref, D = O.backward_dge_dwp(w["X"], w["dY"], z, w["Wp"], w["A"], k)
    assert_close(f"dge k={k}", to_np(out["dWp"]), ref, D, tol_for(dtype))


# --------------------------------------------------------------- H-aware sequential assignment
def _ldlq_case(N, K, d=8, n_cal=None):
    """Targets, and the code-space factor U (fp32) of a calibration Hessian
    H = Xcal^T Xcal / n + 1% damping, through the matrix's A."""
    w = synth.ldlq_workload(N, K, d, n_cal=n_cal)
    X = w["Xcal"].astype(np.float64)
    H = X.T @ X / X.shape[0]
    H += 0.01 * np.mean(np.diag(H)) * np.eye(K)
    U, _ = O.ldl_upper(O.code_space_hessian(H, w["A"].astype(np.float64)))
    return w["P"], U.astype(np.float32)


def _ldlq_gpu(P, U, d=8):
    N, K = P.shape
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_ASSIGN_LDLQ, torch.float32, 0, N, K, d))
    out = lcvq.assign_ldlq(torch.from_numpy(P).to(dev()), torch.from_numpy(U).to(dev()), d,
                           workspace=ws)
    assert lcvq.check_device_error(ws) == 0
    return out


@pytest.mark.parametrize("N,K", [(50, 256), (33, 640)])
def test_ldlq_matches_oracle_on_a_calibration_hessian(N, K):
    """Every code is the rule's choice for the target it was rounded from
    (fp64 recomputation), and the rows agree with the oracle's own run."""
    P, U = _ldlq_case(N, K)
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_ASSIGN_LDLQ, torch.float32, 0, N, K, 8))
    packed = lcvq.assign_ldlq(torch.from_numpy(P).to(dev()), torch.from_numpy(U).to(dev()), 8,
                              workspace=ws)
    assert lcvq.check_device_error(ws) == 0
    Z = O.unpack_codes(packed.cpu().numpy(), K)
    bad, near = ldlq_check(P, U, Z)
    assert bad == 0, (bad, near)
    Zo = O.ldlq_assign(P, U)
    same_rows = int(np.sum(np.all(Z == Zo, axis=1)))
    assert same_rows >= N - near, (same_rows, near)
    # the compensation is at work: the codes differ from plain rounding
    assert np.mean(Z != O.assign(P)[0]) > 0.05


def test_ldlq_exact_arithmetic_is_bit_exact():
    """Dyadic targets and factor entries make every fp32 product and sum
    exact, so the codes (exact ties to even included) match the oracle bit
    for bit."""
    g = np.random.Generator(np.random.PCG64(1500))
    N, K = 37, 512
    P = synth.targets_dyadic(N, K, g)
    U = synth.strict_upper_dyadic(K, g)
    packed = _ldlq_gpu(P, U)
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(O.ldlq_assign(P, U)))


def test_ldlq_reads_only_above_the_diagonal_and_zero_factor_is_assign_pack():
    """U = 0 above the diagonal, NaN on and below it: the codes are those of
    lcvq_assign_pack (ties, clamping and far-out values included)."""
    g = np.random.Generator(np.random.PCG64(1501))
    N, K = 40, 192
    P = _adversarial_wp(N, K, 1502)
    P[~np.isfinite(P)] = 1e30
    U = np.full((K, K), np.nan, dtype=np.float32)
    U[np.triu_indices(K, 1)] = 0.0
    packed = _ldlq_gpu(P, U)
    ref, _ = lcvq.assign_pack(torch.from_numpy(P).to(dev()), d=8, with_mask=False)
    assert torch.equal(packed, ref)
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(O.assign(P)[0]))


def test_ldlq_rows_are_independent_and_deterministic():
    P, U = _ldlq_case(50, 256)
    a = _ldlq_gpu(P, U)
    b = _ldlq_gpu(P, U)
    part = _ldlq_gpu(np.ascontiguousarray(P[16:32]), U)
    assert torch.equal(a, b)
    assert torch.equal(a[16:32], part)


@pytest.mark.parametrize("N,K", [(1, 64), (16, 64), (17, 128), (3, 1024)])
def test_ldlq_edge_shapes(N, K):
    P, U = _ldlq_case(N, K, n_cal=max(2 * K, 64))
    Z = O.unpack_codes(_ldlq_gpu(P, U).cpu().numpy(), K)
    bad, near = ldlq_check(P, U, Z)
    assert bad == 0, (bad, near)


def test_ldlq_empty_matrix_is_a_no_op():
    U = torch.zeros((64, 64), device=dev())
    out = lcvq.assign_ldlq(torch.zeros((0, 64), device=dev()), U, 8)
    assert out.shape == (0, 16)


# ------------------------------------ the algebraic form as two calls (lcvq_xform, lcvq_gemm_xformed)
def _unscramble_xpp(xpp: np.ndarray) -> np.ndarray:
    """X'' (decoder order, position c of each 16-block scaled by 4^-(c mod 3))
    back to bf16(X') in natural order, exactly (powers of two)."""
    M, K = xpp.shape
    blk = xpp.reshape(M, K // 16, 8, 2)                 # [.., pair c, (pos c, pos c + 8)]
    scale = np.array([4.0 ** (c % 3) for c in range(8)])[None, None, :]
    lo, hi = blk[..., 0] * scale, blk[..., 1] * scale
    return np.concatenate([lo, hi], axis=2).reshape(M, K)


@pytest.mark.parametrize("M,K,d", [(1, 1088, 8), (5, 4096, 8), (32, 512, 4), (3, 256, 2), (7, 128, 1)])
def test_xform_matches_its_definition(M, K, d):
    """lcvq_xform against the definition in lcvq.h, restated here in fp64:
    X'[m][g d + j] = sum_i X[m][g d + i] A[i][j] rounded to bf16 (within the
    bf16 half-ulp plus the fp32 products), stored in decoder order with the
    per-position power of two exactly; corr = s' - 3/2 sum bf16(X') -
    128 sum X'' with s' = sum_g x_g . (B + 3/2 A 1)."""
    w = synth.workload(2, M=M, d_in=K, d_out=8, d=d, with_dy=False)
    X = to_dev(w["X"], torch.bfloat16)
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    xpp, xbuf = guarded((M, K), torch.bfloat16)
    corr, cbuf = guarded((M,), torch.float32)
    lcvq.xform(X, A, B, d, xpp=xpp, corr=corr)
    torch.cuda.synchronize()
    assert guard_intact(xpp, xbuf) and guard_intact(corr, cbuf)
    x = w["X"].astype(np.float64)
    A64, B64 = w["A"].astype(np.float64), w["B"].astype(np.float64)
    xg = x.reshape(M, K // d, d)
    Xp = np.einsum("mgi,ij->mgj", xg, A64).reshape(M, K)
    DXp = np.einsum("mgi,ij->mgj", np.abs(xg), np.abs(A64)).reshape(M, K)
    xpp_np = to_np(xpp)
    xr = _unscramble_xpp(xpp_np)
    assert np.all(np.abs(xr - Xp) <= 2.0 ** -8 * DXp), "X' is not bf16(X A)"
    Bp = B64 + 1.5 * A64.sum(axis=1)
    s = np.einsum("mgi,i->m", xg, Bp)
    ref = s - 1.5 * xr.sum(1) - 128.0 * xpp_np.sum(1)
    Dc = np.einsum("mgi,i->m", np.abs(xg), np.abs(Bp)) + 1.5 * np.abs(xr).sum(1) + \
        128.0 * np.abs(xpp_np).sum(1)
    assert_close("corr", to_np(corr), ref, Dc, 1e-5)


@pytest.mark.parametrize("M,d_in,d_out", [(1, 1088, 520), (4, 4096, 1024), (13, 576, 264),
                                          (16, 1088, 520), (32, 512, 264), (33, 512, 264),
                                          (200, 576, 520)])
def test_xform_then_gemm_xformed_equals_gemm(M, d_in, d_out):
    """lcvq_gemm with the algebraic form is lcvq_xform followed by
    lcvq_gemm_xformed: for M > 4 the two calls give lcvq_gemm's bits
    (decode-GEMV and tensor-core GEMM alike); for M <= 4 lcvq_gemm takes the
    int8 path and both meet the oracle.  Neither writes outside its output."""
    w, z = _fwd_case(2, M, d_in=d_in, d_out=d_out)
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    X = to_dev(w["X"], torch.bfloat16)
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    Y1 = lcvq.gemm(X, packed, d_in, A, B, 8, form="algebraic")
    Ya = lcvq.gemm(X, packed, d_in, A, B, 8)
    xpp, corr = lcvq.xform(X, A, B, 8)
    Y2, ybuf = guarded((M, d_out), torch.bfloat16)
    lcvq.gemm_xformed(xpp, corr, packed, out=Y2)
    torch.cuda.synchronize()
    assert guard_intact(Y2, ybuf)
    assert torch.equal(Y1, Ya)
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    if M > 4:
        assert torch.equal(Ya, Y2)
    else:
        assert_close(f"gemm (int8 path) M={M}", to_np(Ya), ref, D, TOL_BF16)
    assert_close(f"gemm_xformed M={M}", to_np(Y2), ref, D, TOL_BF16)


# ------------------------------ the decode-GEMV against the split calls, over K and d_out shapes
@pytest.mark.parametrize("M,d_in,d_out,d", [
    (1, 64, 64, 8),         # one chunk of K (seven empty chunk classes), fewer tiles than CTAs
    (1, 4672, 16400, 8),    # ten chunks: classes of one and two; more tiles than the grid
    (8, 14336, 1032, 4),    # 28 chunks, ragged last tile
    (9, 4096, 264, 2),      # first count of the 32-row tile shape
    (16, 8256, 520, 1),     # 17 chunks, a 64-position tail
    (17, 1088, 4104, 8),    # first count of the four-token-tile shape
    (32, 4096, 1032, 8),
    (32, 28672, 64, 8),     # 56 chunks, seven per class
])
def test_gemm_decode_gemv_equals_split_calls(M, d_in, d_out, d):
    """lcvq_gemm for M <= 32 (X-transform, then the decode-GEMV reading codes
    before its dependency wait) meets the oracle and writes nothing outside Y;
    for M > 4 it gives the bits of lcvq_xform followed by lcvq_gemm_xformed
    (which waits first); for M <= 4 it takes the int8 path."""
    w, z = _fwd_case(2, M, d_in=d_in, d_out=d_out, d=d)
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    X = to_dev(w["X"], torch.bfloat16)
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    Y1, ybuf = guarded((M, d_out), torch.bfloat16)
    lcvq.gemm(X, packed, d_in, A, B, d, out=Y1)
    n1 = lcvq.last_launch_count()
    xpp, corr = lcvq.xform(X, A, B, d)
    Y2 = lcvq.gemm_xformed(xpp, corr, packed)
    torch.cuda.synchronize()
    assert n1 == 2
    assert guard_intact(Y1, ybuf)
    if M > 4:
        assert torch.equal(Y1, Y2)
    ref, D = O.forward(w["X"], z, w["A"], w["B"])
    assert_close(f"split calls M={M} K={d_in}", to_np(Y2), ref, D, TOL_BF16)
    assert_close(f"decode-GEMV M={M} K={d_in}", to_np(Y1), ref, D, TOL_BF16)


@pytest.mark.parametrize("M", [4, 16])
def test_gemm_decode_gemv_back_to_back_on_one_workspace(M):
    """Back-to-back lcvq_gemm calls on one workspace, with programmatic
    dependent launch (each X-transform waits for the previous call's GEMV and
    overwrites X'' and corr that GEMV read; each GEMV becomes resident before
    its X-transform has written): eagerly and replayed from a CUDA graph, every
    output equals the call run alone on a fresh workspace.  A load of X'' or
    corr through a path that can return a line an earlier call left in an
    SM's L1 fails this."""
    K, N = 4096, 4096
    cases = []
    for i in range(4):
        w, z = _fwd_case(2, M, d_in=K, d_out=N)
        X = to_dev(w["X"] * (1.0 + i), torch.bfloat16)
        cases.append((X, torch.from_numpy(O.pack_codes(z)).to(dev()),
                      torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())))
    size = lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, M, N, K, 8)
    alone = []
    for X, p, A, B in cases:
        alone.append(lcvq.gemm(X, p, K, A, B, 8, workspace=lcvq.new_workspace(size, dev())))
        torch.cuda.synchronize()
    ws = lcvq.new_workspace(size, dev())
    for _ in range(3):
        eager = [lcvq.gemm(X, p, K, A, B, 8, workspace=ws) for X, p, A, B in cases]
        torch.cuda.synchronize()
        for Y, r in zip(eager, alone):
            assert torch.equal(Y, r)
    outs = [torch.empty_like(r) for r in alone]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for (X, p, A, B), Y in zip(cases, outs):
            lcvq.gemm(X, p, K, A, B, 8, out=Y, workspace=ws)
    for _ in range(3):
        for Y in outs:
            Y.zero_()
        g.replay()
        torch.cuda.synchronize()
        for Y, r in zip(outs, alone):
            assert torch.equal(Y, r)
    del g


def _int8_positions(block: np.ndarray) -> np.ndarray:
    """Digits of 16-byte blocks back to position order (byte 4 p + i holds
    position 4 i + p)."""
    b = block.reshape(-1, 4, 4)            # [block][p][i]
    return b.transpose(0, 2, 1).reshape(-1)  # [block][i][p] -> position 4 i + p


@pytest.mark.parametrize("M,K,d", [(1, 1088, 8), (4, 4096, 8), (3, 576, 4), (2, 128, 1),
                                   (4, 640, 2), (2, 9216, 8)])
def test_int8_transform_matches_its_definition(M, K, d):
    """For M <= 4, the int8 path's X-transform writes per row and chunk class r
    (the chunks r, r + 8, ... of 512 positions) a power-of-two scale s, the
    largest with max |X'| s <= 32639 over the class, and q = rint(X' s) as two
    signed byte digits (q = 256 hi + lo, lo in [-128, 127]) per position: per
    chunk the hi plane, then the lo plane, each 16-position block in the order
    the GEMV's decoder extracts codes; and corr = s' - 3/2 sum_r (sum q_r) / s_r.
    Read back from the workspace and checked against that definition in fp64
    (X' is formed in fp32, so q may sit one step from rint of the fp64 value
    only where that value is within the fp32 error of a half-integer)."""
    w, z = _fwd_case(2, M, d_in=K, d_out=64, d=d)
    packed = torch.from_numpy(O.pack_codes(z)).to(dev())
    X = to_dev(w["X"], torch.bfloat16)
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    jobs = [(X, packed, A, B, K)]
    ws = lcvq.new_workspace(lcvq.workspace_size_grouped(jobs, M, d), dev())
    lcvq.gemm_grouped(jobs, d, workspace=ws)
    torch.cuda.synchronize()
    raw = ws.cpu().numpy()   # one item: X8 at 256, then corr [M] and inv_s [M][8]
    x8 = raw[256:256 + M * 2 * K].reshape(M, 2 * K)
    coff = (256 + M * K * 2 + 255) // 256 * 256
    corr = raw[coff:coff + 4 * M].view(np.float32)
    inv_s = raw[coff + 4 * M:coff + 36 * M].view(np.float32).reshape(M, 8)
    x = torch.from_numpy(w["X"]).to(torch.bfloat16).double().numpy()
    A64, B64 = w["A"].astype(np.float64), w["B"].astype(np.float64)
    xg = x.reshape(M, K // d, d)
    Xp = np.einsum("mgi,ij->mgj", xg, A64).reshape(M, K)
    # fp32 fused multiply-adds over d terms: within d 2^-24 of the absolute sum
    dXp = np.einsum("mgi,ij->mgj", np.abs(xg), np.abs(A64)).reshape(M, K) * (d * 2.0 ** -24 * 1.01)
    Bp = B64 + 1.5 * A64.sum(axis=1)
    sp = np.einsum("mgi,i->m", xg, Bp)
    cls = (np.arange(K) // 512) % 8
    for m in range(M):
        hi, lo = [], []
        for c0 in range(0, K, 512):
            nc = min(512, K - c0)
            seg = x8[m, 2 * c0:2 * c0 + 2 * nc].view(np.int8)
            hi.append(_int8_positions(seg[:nc]))
            lo.append(_int8_positions(seg[nc:]))
        hi, lo = np.concatenate(hi).astype(np.int64), np.concatenate(lo).astype(np.int64)
        q = 256 * hi + lo
        assert np.all((lo >= -128) & (lo <= 127)) and np.all(np.abs(q) <= 32639)
        qs = 0.0
        for r in range(8):
            s = 1.0 / float(inv_s[m, r])
            assert s == 2.0 ** np.round(np.log2(s)), "each scale is a power of two"
            sel = cls == r
            if not sel.any():
                assert s == 1.0
                continue
            mx = np.abs(Xp[m, sel]).max()
            assert mx * s <= 32639 * (1 + 1e-6) and mx * 2 * s > 32639 * (1 - 1e-6), "largest s"
            assert np.all(np.abs(q[sel] - Xp[m, sel] * s) <= 0.5 + dXp[m, sel] * s + 1e-9)
            qs += q[sel].sum() / s
        ref = sp[m] - 1.5 * qs
        scale_c = np.abs(xg[m]).sum() * np.abs(Bp).max() + 1.5 * np.abs(Xp[m]).sum()
        assert abs(float(corr[m]) - ref) <= 4e-6 * scale_c + 1e-30


def test_gemm_grouped_outputs_are_canaried():
    """Every Y_i of a grouped call (split and wide-tile kernels) stays inside
    its own buffer."""
    for shapes, M in (([(1088, 520), (512, 8), (4096, 1000)], 5),
                      ([(4096, 4096)] * 9 + [(1088, 1000)], 3)):
        jobs, zs, ws = _group_case(shapes, M, 2000 + M)
        pairs = [guarded((M, p.shape[0]), torch.bfloat16) for _, p, _, _, _ in jobs]
        lcvq.gemm_grouped(jobs, 8, outs=[o for o, _ in pairs])
        torch.cuda.synchronize()
        assert all(guard_intact(o, b) for o, b in pairs)
        ref, D = O.forward(ws[0]["X"], zs[0], ws[0]["A"], ws[0]["B"])
        assert_close("canaried grouped item 0", to_np(pairs[0][0]), ref, D, TOL_BF16)


# ------------------------------------------ least-squares refit under the full Hessian H
def _fith_bound(W0, z, d, H, A_ref, B_ref):
    """Error bound of lcvq_fit_affine_h.  The code Gram and column sums are
    exact; T~ = W0^T zt carries the bf16 hi/lo split of W0 (2^-18) and the
    fp32 sum over the rows (at most one rounding per 16-row tensor-core step,
    plus the step's own sum), so |dT~| <= eps_t sum|W0| zt; R then moves by at
    most eps_t (|H| |W0|^T zt summed as R is), and theta = L^+ R by |L^+| |dR|
    to first order.  The fp64 contraction and solve add ~1e-12 relative, the
    fp32 result 2^-24.  The oracle supplies L, R and the absolute sums."""
    N = W0.shape[0]
    L, _ = O.fit_affine_h_normal(W0, z, d, H)
    La, Ra = O.fit_affine_h_normal(np.abs(W0), z, d, np.abs(H))
    th = np.concatenate([A_ref, B_ref[:, None]], axis=1).ravel()
    eps_t = 2.0 ** -17 + (np.ceil(N / 16) + 32) * 2.0 ** -23
    Pinv = np.abs(np.linalg.pinv(L, rcond=O.PINV_RCOND, hermitian=True))
    bnd = Pinv @ ((eps_t + 1e-12) * Ra + 1e-12 * La @ np.abs(th)) + 2.0 ** -24 * np.abs(th)
    bnd = bnd + 1e-12 * np.max(np.abs(th))
    return bnd.reshape(d, d + 1)


def _fith_case(seed, N, K, d, noise=0.01, n_cal=None):
    g = np.random.Generator(np.random.PCG64(seed))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A0, B0 = synth.affine_diag_dominant(d, g)
    W0 = (O.decode(z, A0, B0) + noise * g.standard_normal((N, K))).astype(np.float32)
    n_cal = n_cal or 2 * K
    X = synth.x_outliers(n_cal, K, g, g, "fp32").astype(np.float64)
    H = X.T @ X / n_cal
    H += 0.01 * np.mean(np.diag(H)) * np.eye(K)
    return z, A0, B0, W0, H.astype(np.float32)


def _fith_gpu(W0, z, d, H):
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_FIT_AFFINE_H, torch.float32, 0,
                                                W0.shape[0], W0.shape[1], d))
    A, B = lcvq.fit_affine_h(torch.from_numpy(W0).to(dev()), torch.from_numpy(O.pack_codes(z)).to(dev()),
                             d, torch.from_numpy(H).to(dev()), workspace=ws)
    assert lcvq.check_device_error(ws) == 0
    return A, B


@pytest.mark.parametrize("d", [1, 2, 4, 8])
@pytest.mark.parametrize("N,K", [(77, 192), (300, 512)])
def test_fit_affine_h_matches_oracle(d, N, K):
    """GPU refit under a correlated calibration Hessian against the oracle's
    normal equations over every (g, g') pair, within the derived bound, on
    ragged row counts and K not a multiple of the 256-column chunk."""
    z, A0, B0, W0, H = _fith_case(2200 + 10 * d + N, N, K, d)
    H64, W64 = H.astype(np.float64), W0.astype(np.float64)
    A_ref, B_ref = O.fit_affine_h(W64, z, d, H64)
    A, B = _fith_gpu(W0, z, d, H)
    got = np.concatenate([to_np(A), to_np(B)[:, None]], axis=1)
    ref = np.concatenate([A_ref, B_ref[:, None]], axis=1)
    bnd = _fith_bound(W64, z, d, H64, A_ref, B_ref)
    assert np.all(np.abs(got - ref) <= bnd), float(np.max(np.abs(got - ref) / bnd))
    # the fit is the H-objective's minimum: the GPU answer is as good as the oracle's
    f_gpu = O.fit_objective_h(W64, z, to_np(A), to_np(B), H64)
    f_ref = O.fit_objective_h(W64, z, A_ref, B_ref, H64)
    assert f_gpu <= f_ref * (1 + 1e-6) + 1e-12


def test_fit_affine_h_with_diagonal_h_agrees_with_fit_affine():
    """H = diag(h): the full-H refit and the per-channel refit solve the same
    problem; both lie within their bounds of the oracle."""
    d, N, K = 8, 64, 256
    g = np.random.Generator(np.random.PCG64(2300))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A0, B0 = synth.affine_diag_dominant(d, g)
    W0 = (O.decode(z, A0, B0) + 0.02 * g.standard_normal((N, K))).astype(np.float32)
    h = g.uniform(0.5, 2.0, size=K).astype(np.float32)
    A_ref, B_ref = O.fit_affine(W0.astype(np.float64), z, d, h.astype(np.float64))
    A1, B1 = _fith_gpu(W0, z, d, np.diag(h).astype(np.float32))
    bnd = _fith_bound(W0.astype(np.float64), z, d, np.diag(h).astype(np.float64), A_ref, B_ref)
    got = np.concatenate([to_np(A1), to_np(B1)[:, None]], axis=1)
    ref = np.concatenate([A_ref, B_ref[:, None]], axis=1)
    assert np.all(np.abs(got - ref) <= bnd)
    A2, B2 = lcvq.fit_affine(torch.from_numpy(W0).to(dev()), torch.from_numpy(O.pack_codes(z)).to(dev()),
                             d, h=torch.from_numpy(h).to(dev()))
    assert _fit_ok(A2, B2, A_ref, B_ref, _fit_bound(W0.astype(np.float64), z, d,
                                                    h.astype(np.float64), A_ref, B_ref))


def test_fit_affine_h_singular_empty_and_deterministic():
    """A code position that never varies makes L singular: the minimum-norm
    solution (the Jacobi pseudo-inverse path); an empty matrix gives zeros; two
    runs give the same bits."""
    d, N, K = 4, 96, 128
    z, _, _, W0, H = _fith_case(2400, N, K, d, noise=0.3)
    z = z.copy()
    z[:, 1::d] = 2
    A_ref, B_ref = O.fit_affine_h(W0.astype(np.float64), z, d, H.astype(np.float64))
    A1, B1 = _fith_gpu(W0, z, d, H)
    A2, B2 = _fith_gpu(W0, z, d, H)
    assert torch.equal(A1, A2) and torch.equal(B1, B2)
    got = np.concatenate([to_np(A1).ravel(), to_np(B1)])
    ref = np.concatenate([A_ref.ravel(), B_ref])
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref)), (got, ref)
    Ae, Be = lcvq.fit_affine_h(torch.zeros((0, K), device=dev()),
                               torch.zeros((0, K // 4), dtype=torch.uint8, device=dev()), d,
                               torch.from_numpy(H).to(dev()))
    assert torch.count_nonzero(Ae) == 0 and torch.count_nonzero(Be) == 0

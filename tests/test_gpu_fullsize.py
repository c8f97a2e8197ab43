"""Parity at the full workload sizes, in the launch configuration the
benchmark times.  Every output element is compared with the fp64 oracle: codes
and mask bits bit for bit, floating outputs within the per-element tolerance.

The oracle runs on the host in fp64: the C++ oracle for the decode-GEMV
shapes (few tokens, where decoding the weights dominates), the numpy oracle
(fp64 BLAS) for the prefill and QAT shapes (where the dense products
dominate).  Both are pinned by the CPU tests."""

import numpy as np
import pytest
import torch

from bit_weight_only_lcvq_b200 import lcvq, synth
from oracle import cpp as C
from oracle import lcvq_oracle as O
from tests.gpu_util import TOL_BF16, assert_close, dev, to_np

pytestmark = pytest.mark.gpu


def _bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def test_decode_gemv_full():
    """The decode-GEMV workload the benchmark times: d_in = d_out = 4096, d = 8,
    M in {1, 4, 16} bf16; every output element against the oracle, through
    each entry point that computes it (one lcvq_gemm call; the X-transform and
    the integer-code GEMM as two calls, which the benchmark's roofline times;
    the workspace-free GEMV).  lcvq_gemm and the workspace-free GEMV give the
    same bits; the two calls give them too for M > 4 (for M <= 4 lcvq_gemm
    takes the int8 path)."""
    w = synth.workload(2, M=16, with_dy=False)
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8, with_mask=False)
    pk = packed.cpu().numpy()
    z, _ = O.assign(w["Wp"])
    assert np.array_equal(pk, O.pack_codes(z))
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    ref, Dn = C.forward_packed(w["X"], pk, 4096, w["A"], w["B"])
    for M in (1, 4, 16):
        X = torch.from_numpy(w["X"][:M].copy()).to(torch.bfloat16).to(dev())
        Y = lcvq.gemm(X, packed, 4096, A, B, 8)
        xpp, corr = lcvq.xform(X, A, B, 8)
        Y2 = lcvq.gemm_xformed(xpp, corr, packed)
        Y3 = lcvq.gemv_static(X, packed, 4096, A, B, 8)
        torch.cuda.synchronize()
        assert_close(f"decode-GEMV M={M}", _bf16_np(Y), ref[:M], Dn[:M], TOL_BF16)
        assert_close(f"split calls M={M}", _bf16_np(Y2), ref[:M], Dn[:M], TOL_BF16)
        if M > 4:
            assert torch.equal(Y, Y2), f"xform + gemm_xformed differs from lcvq_gemm at M={M}"
        assert torch.equal(Y, Y3), f"gemv_static differs from lcvq_gemm at M={M}"


@pytest.fixture(scope="module")
def prefill():
    w = synth.workload(3, with_dy=False)
    z, _ = O.assign(w["Wp"])
    ref, Dn = O.forward(w["X"], z, w["A"], w["B"])
    return w, z, ref, Dn


@pytest.mark.parametrize("form", ["algebraic", "decode"])
def test_prefill_full(form, prefill):
    """Prefill GEMM: d_in=4096, d_out=11008, d=8, M=2048 bf16, both forward
    forms, all 22.5 M outputs."""
    w, z, ref, Dn = prefill
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8, with_mask=False)
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(z))
    X = torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev())
    Y = lcvq.gemm(X, packed, 4096, torch.from_numpy(w["A"]).to(dev()),
                  torch.from_numpy(w["B"]).to(dev()), 8, form=form)
    assert_close(f"prefill {form}", _bf16_np(Y), ref, Dn, TOL_BF16)


def test_decode_full_qat_matrix():
    """Decode to bf16 at the size the benchmark times (4096 x 14336, d = 8):
    every element against the oracle."""
    w = synth.workload(4, M=1, with_dy=False)
    z, _ = O.assign(w["Wp"])
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8, with_mask=False)
    W = lcvq.decode(packed, 14336, torch.from_numpy(w["A"]).to(dev()),
                    torch.from_numpy(w["B"]).to(dev()), 8)
    got = _bf16_np(W)
    del W
    assert_close("decode full", got, O.decode(z, w["A"], w["B"]), O.decode_abs(z, w["A"], w["B"]),
                 2.0 ** -8)


@pytest.fixture(scope="module")
def qat():
    w = synth.workload(4)
    z, mask = O.assign(w["Wp"])
    return w, z, mask


def test_qat_assign_pack_full(qat):
    w, z, mask = qat
    packed, mbits = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8)
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(z))
    assert np.array_equal(mbits.cpu().numpy(), O.pack_mask(mask))
    frac = 1.0 - mask.mean()
    assert abs(frac - 0.1336) < 2e-3   # N(1.5, 1): 2 (1 - Phi(1.5)) outside [0, 3]


def test_qat_forward_and_backward_full(qat):
    """QAT step on d_in=14336, d_out=4096, M=8192: the forward Y and every
    output of the straight-through backward (dX, dA, dB, masked dWp), each in
    full against the oracle."""
    w, z, mask = qat
    M, K, N, d = 8192, 14336, 4096, 8
    Wp = torch.from_numpy(w["Wp"]).to(dev())
    packed, mbits = lcvq.assign_pack(Wp, d)
    del Wp
    A = torch.from_numpy(w["A"]).to(dev())
    B = torch.from_numpy(w["B"]).to(dev())
    X = torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev())
    dY = torch.from_numpy(w["dY"]).to(torch.bfloat16).to(dev())
    Yg = _bf16_np(lcvq.gemm(X, packed, K, A, B, d))
    out = lcvq.gemm_backward(X, dY, packed, mbits, K, A, B, d)
    got = {k: (_bf16_np(v) if v.dtype == torch.bfloat16 else v.cpu().numpy().astype(np.float64))
           for k, v in out.items()}
    del out, X, dY
    torch.cuda.empty_cache()
    ref, Dn = O.forward(w["X"], z, w["A"], w["B"])
    assert_close("qat forward", Yg, ref, Dn, TOL_BF16)
    del ref, Dn, Yg
    r = O.backward(w["X"], w["dY"], z, mask, w["A"], w["B"])
    for k in ("dX", "dA", "dB", "dWp"):
        assert_close(f"qat {k}", got[k], r[k], r["D_" + k], TOL_BF16)
    assert np.all(got["dWp"][~mask] == 0)


def test_stack_full():
    """The 7B-shaped stack (32 layers x {q,k,v,o 4096^2; gate, up 4096->11008;
    down 11008->4096}, 224 matrices, 1.62 GB of codes) at M in {1, 8, 32}, in
    the three arrangements the benchmark times: 224 lcvq_gemm calls, one
    lcvq_gemm_grouped per decoder-layer phase, and the whole stack in one
    grouped call.  Every output of every matrix against the oracle; for
    M <= 16 the three arrangements give the same bits (the int8 path at
    M = 1).  As in the benchmark,
    each projection shape has one input X, shared by the 32 layers."""
    layers, projs = 32, synth.STACK_PROJS
    mats = [synth.stack_matrix(l, p, 32, with_x=(l == 0)) for l in range(layers)
            for p in range(len(projs))]
    xs = {m["proj"]: m["X"] for m in mats if m["layer"] == 0}
    dmats = [dict(packed=torch.from_numpy(m["packed"]).to(dev()), A=torch.from_numpy(m["A"]).to(dev()),
                  B=torch.from_numpy(m["B"]).to(dev()), proj=m["proj"], d_in=m["d_in"],
                  d_out=m["d_out"]) for m in mats]
    xd = {p: torch.from_numpy(x).to(torch.bfloat16).to(dev()) for p, x in xs.items()}
    phases = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))
    got = {}   # (M, arrangement) -> list of Y on the host (bf16)
    for M in (1, 8, 32):
        seq = []
        for m in dmats:
            seq.append(lcvq.gemm(xd[m["proj"]][:M], m["packed"], m["d_in"], m["A"], m["B"], 8).cpu())
        jobs = [(xd[m["proj"]][:M], m["packed"], m["A"], m["B"], m["d_in"]) for m in dmats]
        allg = [y.cpu() for y in lcvq.gemm_grouped(jobs, 8)]
        phase = []
        nproj = len(projs)
        for l0 in range(0, len(dmats), nproj):
            named = {dmats[l0 + i]["proj"]: (l0 + i, jobs[l0 + i]) for i in range(nproj)}
            res = {}
            for ph in phases:
                ys = lcvq.gemm_grouped([named[p][1] for p in ph], 8)
                for p, y in zip(ph, ys):
                    res[named[p][0]] = y.cpu()
            phase.extend(res[i] for i in range(l0, l0 + nproj))
        torch.cuda.synchronize()
        got[(M, "sequential")] = seq
        got[(M, "grouped_all")] = allg
        got[(M, "grouped_by_phase")] = phase
        if M <= 16:
            for i in range(len(dmats)):
                assert torch.equal(seq[i], allg[i]) and torch.equal(seq[i], phase[i]), (M, i)
    del dmats, xd
    torch.cuda.empty_cache()
    worst = {}
    for i, m in enumerate(mats):
        ref, Dn = C.forward_packed(xs[m["proj"]], m["packed"], m["d_in"], m["A"], m["B"])
        for (M, arr), ys in got.items():
            e = assert_close(f"stack {m['proj']} layer {m['layer']} M={M} {arr}",
                             _bf16_np(ys[i]), ref[:M], Dn[:M], TOL_BF16)
            worst[(M, arr)] = max(worst.get((M, arr), 0.0), e)
    assert len(worst) == 9


def test_fit_affine_full_size_qat_matrix():
    """Refit on the QAT-step matrix (4096 x 14336, d = 8): W0 = A0 z + B0 plus
    noise; the GPU fit matches the oracle, and recovers (A0, B0) closely."""
    d, N, K = 8, 4096, 14336
    g = np.random.Generator(np.random.PCG64(1300))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A0, B0 = synth.affine_diag_dominant(d, g)
    W0 = O.decode(z, A0, B0)
    W0 += 0.005 * g.standard_normal((N, K))
    W0 = W0.astype(np.float32)
    h = g.uniform(0.5, 2.0, size=K).astype(np.float32)
    A_ref, B_ref = O.fit_affine(W0.astype(np.float64), z, d, h.astype(np.float64))
    A, B = lcvq.fit_affine(torch.from_numpy(W0).to(dev()), torch.from_numpy(O.pack_codes(z)).to(dev()),
                           d, h=torch.from_numpy(h).to(dev()))
    from tests.test_gpu_parity import _fit_bound, _fit_ok
    assert _fit_ok(A, B, A_ref, B_ref, _fit_bound(W0.astype(np.float64), z, d, h.astype(np.float64),
                                                  A_ref, B_ref))
    ref = np.concatenate([A_ref.ravel(), B_ref.ravel()])
    assert np.max(np.abs(ref - np.concatenate([A0.ravel(), B0.ravel()]))) < 1e-3


def test_ldlq_full_size_decode_matrix():
    """H-aware sequential assignment at 4096 x 4096 (the size the benchmark
    times) with a calibration Hessian: every row is checked against the fp64
    recomputation of every target, and sampled rows match the oracle's own run."""
    from tests.test_gpu_parity import _ldlq_case, _ldlq_gpu
    from tests.gpu_util import ldlq_check
    N = K = 4096
    P, U = _ldlq_case(N, K)
    packed = _ldlq_gpu(P, U).cpu().numpy()
    Z = O.unpack_codes(packed, K)
    bad, near = ldlq_check(P, U, Z)
    assert bad == 0, (bad, near)
    g = np.random.Generator(np.random.PCG64(1600))
    rows = np.unique(np.concatenate([[0, 15, 16, N - 1], g.choice(N, 4, replace=False)]))
    Zo = O.ldlq_assign(P[rows], U)
    assert np.sum(np.all(Z[rows] == Zo, axis=1)) >= len(rows) - near


def test_ldlq_full_size_qat_matrix():
    """4096 x 14336 (the QAT-step matrix) with a random factor: sampled rows
    checked against the fp64 recomputation."""
    from tests.gpu_util import ldlq_check
    N, K = 4096, 14336
    g = np.random.Generator(np.random.PCG64(1601))
    P = synth.wp_uniform(N, K, g)
    U = (g.standard_normal((K, K), dtype=np.float32) * np.float32(1.0 / np.sqrt(K)))
    U = np.triu(U, 1)
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_ASSIGN_LDLQ, torch.float32, 0, N, K, 8))
    out = lcvq.assign_ldlq(torch.from_numpy(P).to(dev()), torch.from_numpy(U).to(dev()), 8,
                           workspace=ws)
    assert lcvq.check_device_error(ws) == 0
    rows = np.array([0, 1, 2047, 4095] + list(g.choice(N, 4, replace=False)))
    Z = O.unpack_codes(out.cpu().numpy()[rows], K)
    bad, near = ldlq_check(P[rows], U, Z)
    assert bad == 0, (bad, near)


def test_fit_affine_h_full_size_decode_matrix():
    """Refit under the full Hessian at 4096 x 4096 (d = 8) with an 8192-row
    calibration Hessian (outlier recipe, 1% ridge): W0 = A0 z + B0 plus noise;
    the GPU fit lies within the derived bound of the oracle and reaches its
    H-objective."""
    from tests.test_gpu_parity import _fith_bound, _fith_case, _fith_gpu
    d, N, K = 8, 4096, 4096
    z, A0, B0, W0, H = _fith_case(2500, N, K, d, noise=0.005, n_cal=8192)
    H64, W64 = H.astype(np.float64), W0.astype(np.float64)
    A_ref, B_ref = O.fit_affine_h(W64, z, d, H64)
    A, B = _fith_gpu(W0, z, d, H)
    got = np.concatenate([to_np(A), to_np(B)[:, None]], axis=1)
    ref = np.concatenate([A_ref, B_ref[:, None]], axis=1)
    bnd = _fith_bound(W64, z, d, H64, A_ref, B_ref)
    assert np.all(np.abs(got - ref) <= bnd), float(np.max(np.abs(got - ref) / bnd))
    assert O.fit_objective_h(W64, z, to_np(A), to_np(B), H64) <= \
        O.fit_objective_h(W64, z, A_ref, B_ref, H64) * (1 + 1e-6)
    assert np.max(np.abs(ref - np.concatenate([A0, B0[:, None]], axis=1))) < 1e-3

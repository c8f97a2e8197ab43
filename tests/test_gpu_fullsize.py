"""Parity at the full workload sizes, in the launch configuration the
benchmark times: bit-exact codes/masks over whole matrices, floating outputs
on sampled elements the oracle computes one by one, and dB through an exact
O(M (N + K)) identity.  dA is computed in full in fp64 (chunked)."""

import numpy as np
import pytest
import torch

from bit_weight_only_lcvq_b200 import lcvq, synth
from oracle import lcvq_oracle as O
from tests.gpu_util import TOL_BF16, assert_close, dev, to_np

pytestmark = pytest.mark.gpu

N_SAMPLES = 384


def _pairs(seed, a, b, n=N_SAMPLES):
    g = np.random.Generator(np.random.PCG64(seed))
    return [(int(x), int(y)) for x, y in zip(g.integers(0, a, n), g.integers(0, b, n))]


def _check_sampled_forward(Y, Xnp, z, A, B, pairs, tag):
    y, dd = O.forward_sampled(Xnp, {n: z[n] for _, n in pairs}, A, B, pairs)
    Yc = Y.float().cpu().numpy()
    got = np.array([Yc[m, n] for m, n in pairs])
    assert_close(tag, got, y, dd, TOL_BF16)


def test_decode_gemv_full():
    """The decode-GEMV workload the benchmark times: d_in = d_out = 4096, d = 8,
    M in {1, 4, 16} bf16; every output element against the oracle."""
    w = synth.workload(2, M=16, with_dy=False)
    z, _ = O.assign(w["Wp"])
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8, with_mask=False)
    A, B = torch.from_numpy(w["A"]).to(dev()), torch.from_numpy(w["B"]).to(dev())
    for M in (1, 4, 16):
        X = torch.from_numpy(w["X"][:M].copy()).to(torch.bfloat16).to(dev())
        Y = lcvq.gemm(X, packed, 4096, A, B, 8)
        ref, Dn = O.forward(w["X"][:M], z, w["A"], w["B"])
        assert_close(f"decode-GEMV M={M}", Y.float().cpu().numpy(), ref, Dn, TOL_BF16)


@pytest.mark.parametrize("form", ["algebraic", "decode"])
def test_prefill_full(form):
    """Prefill GEMM: d_in=4096, d_out=11008, d=8, M=2048 bf16."""
    w = synth.workload(3, with_dy=False)
    z, _ = O.assign(w["Wp"])
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8, with_mask=False)
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(z))
    X = torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev())
    Y = lcvq.gemm(X, packed, 4096, torch.from_numpy(w["A"]).to(dev()),
                  torch.from_numpy(w["B"]).to(dev()), 8, form=form)
    _check_sampled_forward(Y, w["X"], z, w["A"], w["B"], _pairs(3, 2048, 11008), f"prefill {form}")


def test_decode_full_qat_matrix():
    """Decode to bf16 at the size the benchmark times (4096 x 14336, d = 8):
    sampled rows, every element, against the oracle."""
    w = synth.workload(4, M=1, with_dy=False)
    z, _ = O.assign(w["Wp"])
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev()), 8, with_mask=False)
    W = lcvq.decode(packed, 14336, torch.from_numpy(w["A"]).to(dev()),
                    torch.from_numpy(w["B"]).to(dev()), 8)
    rows = [0, 1, 2047, 4095, 1234, 3333]
    got = W[rows].float().cpu().numpy()
    ref = O.decode(z[rows], w["A"], w["B"])
    assert_close("decode full", got, ref, O.decode_abs(z[rows], w["A"], w["B"]), 2.0 ** -8)


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
    """QAT step on d_in=14336, d_out=4096, M=8192: forward, then dX, dA, dB,
    dWp of the straight-through backward."""
    w, z, mask = qat
    M, K, N, d = 8192, 14336, 4096, 8
    Wp = torch.from_numpy(w["Wp"]).to(dev())
    packed, mbits = lcvq.assign_pack(Wp, d)
    A = torch.from_numpy(w["A"]).to(dev())
    B = torch.from_numpy(w["B"]).to(dev())
    X = torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev())
    dY = torch.from_numpy(w["dY"]).to(torch.bfloat16).to(dev())
    Y = lcvq.gemm(X, packed, K, A, B, d)
    _check_sampled_forward(Y, w["X"], z, w["A"], w["B"], _pairs(4, M, N), "qat forward")
    del Y
    out = lcvq.gemm_backward(X, dY, packed, mbits, K, A, B, d)
    dX = out["dX"].float().cpu().numpy()
    pairs = _pairs(5, M, K)
    v, dd = O.backward_dx_sampled(w["dY"], lambda k: z[:, (k // d) * d:(k // d + 1) * d],
                                  w["A"], w["B"], pairs)
    assert_close("qat dX", np.array([dX[m, k] for m, k in pairs]), v, dd, TOL_BF16)
    del dX
    dWp = out["dWp"].cpu().numpy()
    pairs = _pairs(6, N, K)
    v, dd = O.backward_dwp_sampled(w["X"], w["dY"], lambda n: mask[n], w["A"], pairs)
    assert_close("qat dWp", np.array([dWp[n, k] for n, k in pairs]), v, dd, TOL_BF16)
    assert np.all(dWp[~mask] == 0)
    del dWp
    # dB through sum_m rowsum(dY)[m] * sum_g X[m, g d + i]  (exact identity)
    X64 = w["X"].astype(np.float64)
    dY64 = w["dY"].astype(np.float64)
    xs = X64.reshape(M, K // d, d).sum(1)
    ref_dB = dY64.sum(1) @ xs
    D_dB = np.abs(dY64).sum(1) @ np.abs(X64).reshape(M, K // d, d).sum(1)
    assert_close("qat dB", out["dB"].cpu().numpy(), ref_dB, D_dB, TOL_BF16)
    # dA in full: dA[i][j] = sum_m sum_g X[m, g d + i] P[m, g d + j], P = dY Z
    Z = z.astype(np.float64)
    ref_dA = np.zeros((d, d))
    D_dA = np.zeros((d, d))
    for c0 in range(0, M, 1024):
        P = dY64[c0:c0 + 1024] @ Z
        Pa = np.abs(dY64[c0:c0 + 1024]) @ Z
        Xc = X64[c0:c0 + 1024].reshape(-1, K // d, d)
        ref_dA += np.einsum("mgi,mgj->ij", Xc, P.reshape(-1, K // d, d))
        D_dA += np.einsum("mgi,mgj->ij", np.abs(Xc), Pa.reshape(-1, K // d, d))
    assert_close("qat dA", out["dA"].cpu().numpy(), ref_dA, D_dA, TOL_BF16)


@pytest.mark.parametrize("M", [1, 8, 32])
def test_stack_matrices(M):
    """One matrix of each projection shape of the 7B-shaped stack."""
    for proj in range(len(synth.STACK_PROJS)):
        m = synth.stack_matrix(proj, proj, M)
        z = O.unpack_codes(m["packed"], m["d_in"])
        X = torch.from_numpy(m["X"]).to(torch.bfloat16).to(dev())
        Y = lcvq.gemm(X, torch.from_numpy(m["packed"]).to(dev()), m["d_in"],
                      torch.from_numpy(m["A"]).to(dev()), torch.from_numpy(m["B"]).to(dev()), 8)
        pairs = _pairs(7 + proj, M, m["d_out"], 128)
        _check_sampled_forward(Y, m["X"], z, m["A"], m["B"], pairs, f"stack {m['proj']} M={M}")


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
    times) with a calibration Hessian: sampled rows are checked against the
    fp64 recomputation of every target, and match the oracle's own run."""
    from tests.test_gpu_parity import _ldlq_case, _ldlq_gpu
    from tests.gpu_util import ldlq_check
    N = K = 4096
    P, U = _ldlq_case(N, K)
    packed = _ldlq_gpu(P, U).cpu().numpy()
    g = np.random.Generator(np.random.PCG64(1600))
    rows = np.unique(np.concatenate([[0, 15, 16, N - 1], g.choice(N, 44, replace=False)]))
    Z = O.unpack_codes(packed[rows], K)
    bad, near = ldlq_check(P[rows], U, Z)
    assert bad == 0, (bad, near)
    Zo = O.ldlq_assign(P[rows[:8]], U)
    assert np.sum(np.all(Z[:8] == Zo, axis=1)) >= 8 - near


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

"""Pins for the fp64 oracle: every function is checked against something that
does not come from the oracle itself (hand-worked golden files, brute force
over all 4^d codes, closed forms, exact integer arithmetic, finite
differences, distribution statistics)."""

import itertools
import math
import os

import numpy as np
import pytest

from oracle import lcvq_oracle as O
from bit_weight_only_lcvq_b200 import synth


# ---------------------------------------------------------------- helpers
def _read(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return [ln.split("#")[0].strip() for ln in f if ln.split("#")[0].strip()]


def _f32(tok):
    return np.float32(float(tok))


# ---------------------------------------------------------------- assign
def test_round_clamp_golden(golden_dir):
    rows = [ln.split() for ln in _read(golden_dir, "round_clamp_ties.txt")]
    w = np.array([_f32(r[0]) for r in rows], dtype=np.float32)
    z, mask = O.assign(w)
    assert z.tolist() == [int(r[1]) for r in rows]
    assert mask.astype(int).tolist() == [int(r[2]) for r in rows]


@pytest.mark.parametrize("d", [1, 2, 4])
def test_assign_is_nearest_code_brute_force(d):
    """Round-and-clamp equals the exhaustive nearest-neighbour search over all
    4^d codes (the box-constrained problem is separable)."""
    g = np.random.Generator(np.random.PCG64(11 + d))
    cand = np.array(list(itertools.product(range(4), repeat=d)), dtype=np.float64)
    w = g.uniform(-1.5, 4.5, size=(400, d)).astype(np.float32)
    frac = np.abs(w - np.floor(w) - 0.5)
    w = w[np.all(frac > 1e-4, axis=1)]          # ties are pinned by the golden table
    z, _ = O.assign(w)
    dist = ((w[:, None, :].astype(np.float64) - cand[None]) ** 2).sum(-1)
    best = cand[np.argmin(dist, axis=1)].astype(np.uint8)
    assert np.array_equal(z, best)


def test_assign_brute_force_d8():
    g = np.random.Generator(np.random.PCG64(7))
    cand = np.array(list(itertools.product(range(4), repeat=8)), dtype=np.float64)
    for _ in range(3):
        w = g.uniform(-1.0, 4.0, size=8).astype(np.float32)
        if np.any(np.abs(w - np.floor(w) - 0.5) < 1e-4):
            continue
        z, _ = O.assign(w[None])
        best = cand[np.argmin(((cand - w.astype(np.float64)) ** 2).sum(-1))]
        assert np.array_equal(z[0], best.astype(np.uint8))


def test_scalar_special_case_matches_uniform_quantizer():
    """With A = s I and B = b 1 the linear-constrained codebook is a scalar
    uniform grid: nearest codeword of w0 = clamp(round((w0 - b)/s), 0, 3) and
    the decode is s z + b (decoupleQ page, eq. (3) and (4), with the integer
    range [0, 3]).  Checked by exhaustive search over the 4^d codewords."""
    d = 4
    s, b = 0.37, -0.61
    A = s * np.eye(d)
    B = b * np.ones(d)
    cand = np.array(list(itertools.product(range(4), repeat=d)), dtype=np.uint8)
    cw = O.decode(cand, A, B)                         # [256, d] codewords
    assert np.allclose(cw, s * cand + b, rtol=0, atol=1e-15)
    g = np.random.Generator(np.random.PCG64(3))
    w0 = g.uniform(b - 1.0, b + 4 * s, size=(300, d))
    q = (w0 - b) / s
    ok = np.all(np.abs(q - np.floor(q) - 0.5) > 1e-6, axis=1)
    w0, q = w0[ok], q[ok]
    nn = cand[np.argmin(((w0[:, None, :] - cw[None]) ** 2).sum(-1), axis=1)]
    z, _ = O.assign(q)
    assert np.array_equal(z, nn)


def _phi(x):
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def test_code_statistics_uniform_and_normal():
    """U[-0.5, 3.5] gives uniform codes; N(1.5, 1) gives
    Phi(-1), Phi(0)-Phi(-1), ... and a clamp fraction 2 (1 - Phi(1.5))."""
    n = 1 << 20
    g = np.random.Generator(np.random.PCG64(5))
    z, _ = O.assign(g.uniform(-0.5, 3.5, size=n).astype(np.float32))
    freq = np.bincount(z, minlength=4) / n
    assert np.allclose(freq, 0.25, atol=3e-3)
    z, mask = O.assign(g.normal(1.5, 1.0, size=n).astype(np.float32))
    freq = np.bincount(z, minlength=4) / n
    p0 = _phi(-1.0)
    p1 = _phi(0.0) - _phi(-1.0)
    assert np.allclose(freq, [p0, p1, p1, p0], atol=3e-3)
    clamp_frac = 1.0 - mask.mean()
    assert abs(clamp_frac - 2 * (1 - _phi(1.5))) < 3e-3
    assert abs(2 * (1 - _phi(1.5)) - 0.1336) < 1e-4


# ---------------------------------------------------------------- pack
def test_pack_golden(golden_dir):
    for ln in _read(golden_dir, "pack_v1.txt"):
        codes, hexes = ln.split("|")
        z = np.array([[int(t) for t in codes.split()]], dtype=np.uint8)
        want = [int(h, 16) for h in hexes.split()]
        got = O.pack_codes(z)
        assert got[0].tolist() == want
        assert np.array_equal(O.unpack_codes(got, z.shape[1]), z)


def test_mask_golden(golden_dir):
    for ln in _read(golden_dir, "mask_v1.txt"):
        bits, hexes = ln.split("|")
        m = np.array([[int(t) for t in bits.split()]], dtype=bool)
        want = [int(h, 16) for h in hexes.split()]
        got = O.pack_mask(m)
        assert got[0].tolist() == want
        assert np.array_equal(O.unpack_mask(got, m.shape[1]), m)


def test_pack_is_bijection_on_bytes():
    allb = np.arange(256, dtype=np.uint8)[None, :]
    z = O.unpack_codes(allb, 1024)
    assert np.array_equal(O.pack_codes(z), allb)
    g = np.random.Generator(np.random.PCG64(9))
    z = g.integers(0, 4, size=(37, 64), dtype=np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(z), 64), z)
    m = g.integers(0, 2, size=(5, 64)).astype(bool)
    assert np.array_equal(O.unpack_mask(O.pack_mask(m), 64), m)


def test_packed_d8_vector_is_codebook_index():
    g = np.random.Generator(np.random.PCG64(13))
    z = g.integers(0, 4, size=(4, 32), dtype=np.uint8)
    p = O.pack_codes(z)
    for r in range(4):
        for v in range(4):
            idx = sum(int(z[r, 8 * v + j]) * 4 ** j for j in range(8))
            assert int(p[r, 2 * v]) | (int(p[r, 2 * v + 1]) << 8) == idx


# ---------------------------------------------------------------- decode
def test_decode_golden(golden_dir):
    lines = _read(golden_dir, "affine_hand.txt")
    cases, cur = [], None
    for ln in lines:
        t = ln.split()
        if t[0] == "case":
            cur = dict(A=[], z=[], c=[])
            cases.append(cur)
        elif t[0] == "d":
            cur["d"] = int(t[1])
        elif t[0] == "A":
            cur["A"].append([float(v) for v in t[1:]])
        elif t[0] == "B":
            cur["B"] = [float(v) for v in t[1:]]
        elif t[0] == "z":
            k = t.index("->")
            cur["z"].append([int(v) for v in t[1:k]])
            cur["c"].append([float(v) for v in t[k + 1:]])
    assert len(cases) == 2
    for c in cases:
        z = np.array(c["z"], dtype=np.uint8)
        W = O.decode(z, np.array(c["A"]), np.array(c["B"]))
        assert np.array_equal(W, np.array(c["c"]))


def test_decode_equals_codebook_lookup():
    """Materialize the 4^d codebook and look each vector up by its packed
    index: must equal the grouped affine decode."""
    d = 4
    A, B = synth.affine_single_layer(d, np.random.Generator(np.random.PCG64(1)))
    book = {}
    for zt in itertools.product(range(4), repeat=d):
        idx = sum(v * 4 ** j for j, v in enumerate(zt))
        book[idx] = [sum(float(A[i, j]) * zt[j] for j in range(d)) + float(B[i]) for i in range(d)]
    g = np.random.Generator(np.random.PCG64(2))
    z = g.integers(0, 4, size=(6, 32), dtype=np.uint8)
    p = O.pack_codes(z)
    W = O.decode(z, A, B)
    for r in range(6):
        for v in range(32 // d):
            idx = int(p[r, v])           # d = 4: one byte per vector
            assert np.allclose(W[r, v * d:(v + 1) * d], book[idx], rtol=0, atol=1e-15)


def test_decode_scalar_case_is_cross_d_invariant():
    g = np.random.Generator(np.random.PCG64(4))
    z = g.integers(0, 4, size=(3, 64), dtype=np.uint8)
    ref = 0.25 * z.astype(np.float64) - 0.375
    for d in (1, 2, 4, 8):
        W = O.decode(z, 0.25 * np.eye(d), -0.375 * np.ones(d))
        assert np.array_equal(W, ref)


# ---------------------------------------------------------------- forward
def test_linear_layer_golden(golden_dir):
    rec = {}
    for ln in _read(golden_dir, "linear_layer_hand.txt"):
        t = ln.split()
        rec.setdefault(t[0], []).append([float(v) for v in t[1:]])
    A = np.array(rec["A"])
    B = np.array(rec["B"][0])
    Wp = np.array(rec["Wp"][0], dtype=np.float32)[None]
    z, mask = O.assign(Wp)
    assert z[0].tolist() == [int(v) for v in rec["z"][0]]
    assert mask[0].astype(int).tolist() == [int(v) for v in rec["mask"][0]]
    assert np.array_equal(O.decode(z, A, B)[0], rec["W"][0])
    X = np.array(rec["X"][0])[None]
    Y, _ = O.forward(X, z, A, B)
    assert Y[0, 0] == rec["Y"][0][0]
    assert O.forward_algebraic(X, z, A, B)[0, 0] == rec["Y"][0][0]
    dY = np.array(rec["dY"][0])[None]
    bw = O.backward(X, dY, z, mask, A, B)
    assert np.array_equal(bw["dX"][0], rec["dX"][0])
    assert np.array_equal(bw["dA"], np.array(rec["dA"]))
    assert np.array_equal(bw["dB"], rec["dB"][0])
    assert np.array_equal(bw["dWp"][0], rec["dWp"][0])


def test_forward_identity_is_integer_code_gemm():
    """A = I, B = 0: Y = X Z^T exactly (checked in int64 arithmetic)."""
    g = np.random.Generator(np.random.PCG64(21))
    for d in (4, 8):
        X = g.integers(-8, 9, size=(5, 64))
        z = g.integers(0, 4, size=(7, 64), dtype=np.uint8)
        Y, D = O.forward(X.astype(np.float64), z, np.eye(d), np.zeros(d))
        Yi = X.astype(np.int64) @ z.astype(np.int64).T
        assert np.array_equal(Y, Yi.astype(np.float64))
        assert np.array_equal(D, (np.abs(X) @ z.astype(np.int64).T).astype(np.float64))


def _rand_case(seed, M=3, N=5, K=32, d=8):
    g = np.random.Generator(np.random.PCG64(seed))
    X = g.standard_normal((M, K))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A = g.standard_normal((d, d))
    B = g.standard_normal(d)
    return X, z, A, B


def test_forward_linearity_and_pow2_scaling():
    X, z, A1, B1 = _rand_case(31)
    _, _, A2, B2 = _rand_case(32)
    Y1, D1 = O.forward(X, z, A1, B1)
    Y2, _ = O.forward(X, z, A2, B2)
    Y12, _ = O.forward(X, z, A1 + A2, B1 + B2)
    assert np.max(np.abs(Y12 - Y1 - Y2)) <= 1e-12 * np.max(D1 + 1)
    Y8, _ = O.forward(X, z, 8.0 * A1, 8.0 * B1)
    assert np.array_equal(Y8, 8.0 * Y1)


def test_forward_direct_equals_algebraic():
    X, z, A, B = _rand_case(41, M=4, N=6, K=64)
    Y, D = O.forward(X, z, A, B)
    assert O.rel_err(O.forward_algebraic(X, z, A, B), Y, D) < 1e-13


def test_forward_sampled_matches_full():
    X, z, A, B = _rand_case(43, M=4, N=6, K=64)
    Y, D = O.forward(X, z, A, B)
    pairs = [(0, 0), (3, 5), (2, 1)]
    y, dd = O.forward_sampled(X, {n: z[n] for n in range(6)}, A, B, pairs)
    for t, (m, n) in enumerate(pairs):
        assert abs(y[t] - Y[m, n]) <= 1e-13 * D[m, n] and abs(dd[t] - D[m, n]) <= 1e-13 * D[m, n]


# ---------------------------------------------------------------- backward
def _loss(X, dY, z, A, B):
    Y, _ = O.forward(X, z, A, B)
    return float(np.sum(dY * Y))


def test_backward_finite_differences_exact():
    """L = sum dY * Y is linear in X, in A and in B (codes fixed), so a
    central difference with any step is exact up to fp64 rounding."""
    X, z, A, B = _rand_case(51, M=3, N=4, K=16, d=4)
    g = np.random.Generator(np.random.PCG64(52))
    dY = g.standard_normal((3, 4))
    mask = np.ones_like(z, dtype=bool)
    bw = O.backward(X, dY, z, mask, A, B)
    h = 0.5
    for (m, k) in [(0, 0), (2, 15), (1, 7)]:
        Xp, Xm = X.copy(), X.copy()
        Xp[m, k] += h
        Xm[m, k] -= h
        fd = (_loss(Xp, dY, z, A, B) - _loss(Xm, dY, z, A, B)) / (2 * h)
        assert abs(fd - bw["dX"][m, k]) < 1e-12 * (1 + abs(fd))
    for (i, j) in [(0, 0), (3, 1), (2, 3)]:
        Ap, Am = A.copy(), A.copy()
        Ap[i, j] += h
        Am[i, j] -= h
        fd = (_loss(X, dY, z, Ap, B) - _loss(X, dY, z, Am, B)) / (2 * h)
        assert abs(fd - bw["dA"][i, j]) < 1e-11 * (1 + abs(fd))
    for i in range(4):
        Bp, Bm = B.copy(), B.copy()
        Bp[i] += h
        Bm[i] -= h
        fd = (_loss(X, dY, z, A, Bp) - _loss(X, dY, z, A, Bm)) / (2 * h)
        assert abs(fd - bw["dB"][i]) < 1e-11 * (1 + abs(fd))


def test_backward_dwp_ste_surrogate_finite_differences():
    """STE: the rounding is treated as identity, the clamp is kept.  The
    surrogate L(Wp) = sum dY * (X decode(clamp(Wp, 0, 3))^T) is piecewise
    linear; at points >= 1e-3 away from 0 and 3 a step of 1e-4 is exact up to
    rounding, and the gradient is zero wherever the clamp is active."""
    M, N, K, d = 3, 4, 16, 4
    g = np.random.Generator(np.random.PCG64(61))
    X = g.standard_normal((M, K))
    dY = g.standard_normal((M, N))
    A = g.standard_normal((d, d))
    B = g.standard_normal(d)
    Wp = g.uniform(-1.0, 4.0, size=(N, K))
    Wp[np.abs(Wp) < 1e-3] += 2e-3
    Wp[np.abs(Wp - 3) < 1e-3] += 2e-3
    z, mask = O.assign(Wp.astype(np.float32))
    bw = O.backward(X, dY, z, mask, A, B)

    def surrogate(W):
        return _loss(X, dY, np.clip(W, 0.0, 3.0), A, B)

    h = 1e-4
    for n in range(N):
        for k in range(K):
            Wa, Wb = Wp.copy(), Wp.copy()
            Wa[n, k] += h
            Wb[n, k] -= h
            fd = (surrogate(Wa) - surrogate(Wb)) / (2 * h)
            assert abs(fd - bw["dWp"][n, k]) < 1e-7 * (1 + abs(fd)), (n, k)
    assert np.all(bw["dWp"][~mask] == 0)


def test_backward_sampled_matches_full():
    M, N, K, d = 4, 6, 32, 8
    g = np.random.Generator(np.random.PCG64(71))
    X = g.standard_normal((M, K))
    dY = g.standard_normal((M, N))
    A = g.standard_normal((d, d))
    B = g.standard_normal(d)
    Wp = g.uniform(-1.0, 4.0, size=(N, K)).astype(np.float32)
    z, mask = O.assign(Wp)
    bw = O.backward(X, dY, z, mask, A, B)
    pairs = [(0, 0), (3, 31), (1, 9)]
    v, dd = O.backward_dx_sampled(dY, lambda k: z[:, (k // d) * d:(k // d + 1) * d], A, B, pairs)
    for t, (m, k) in enumerate(pairs):
        assert abs(v[t] - bw["dX"][m, k]) <= 1e-13 * bw["D_dX"][m, k]
        assert abs(dd[t] - bw["D_dX"][m, k]) <= 1e-13 * bw["D_dX"][m, k]
    pairs = [(0, 0), (5, 31), (2, 10)]
    v, dd = O.backward_dwp_sampled(X, dY, lambda n: mask[n], A, pairs)
    for t, (n, k) in enumerate(pairs):
        assert abs(v[t] - bw["dWp"][n, k]) <= 1e-13 * (bw["D_dWp"][n, k] + 1e-300)
        assert abs(dd[t] - bw["D_dWp"][n, k]) <= 1e-13 * (bw["D_dWp"][n, k] + 1e-300)


def test_db_identity_at_any_size():
    """dB[i] = sum_m rowsum(dY)[m] * sum_g X[m, g d + i]: an O(M (N + K))
    identity the tests use to check dB at full size."""
    M, N, K, d = 5, 7, 32, 8
    g = np.random.Generator(np.random.PCG64(81))
    X = g.standard_normal((M, K))
    dY = g.standard_normal((M, N))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    bw = O.backward(X, dY, z, np.ones((N, K), bool), np.eye(d), np.zeros(d))
    ident = dY.sum(1) @ X.reshape(M, K // d, d).sum(1)
    assert np.allclose(bw["dB"], ident, rtol=1e-13, atol=1e-13)


# ------------------------------------------ the normalisers of the tolerance (R15)
_NORMS = (("W", "D_W"), ("Y", "D_Y"), ("dX", "D_dX"), ("dA", "D_dA"), ("dB", "D_dB"),
          ("dWp", "D_dWp"))


def _all_outputs(X, dY, z, mask, A, B):
    out = dict(O.backward(X, dY, z, mask, A, B))
    out["Y"], out["D_Y"] = O.forward(X, z, A, B)
    out["W"], out["D_W"] = O.decode(z, A, B), O.decode_abs(z, A, B)
    return out


def test_normalisers_equal_the_outputs_when_no_term_is_negative():
    """A normaliser is the sum of its output's terms in absolute value; with
    non-negative X, dY, A and B no term is negative, so each equals its
    output (codes are non-negative too)."""
    g = np.random.Generator(np.random.PCG64(91))
    M, N, K, d = 3, 5, 32, 4
    X, dY = g.uniform(0, 2, (M, K)), g.uniform(0, 2, (M, N))
    A, B = g.uniform(0, 1, (d, d)), g.uniform(0, 1, d)
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    out = _all_outputs(X, dY, z, np.ones((N, K), bool), A, B)
    for v, dn in _NORMS:
        assert np.allclose(out[dn], out[v], rtol=1e-13, atol=0), v


def test_normalisers_ignore_the_signs_of_the_operands():
    """Flipping the sign of X, of dY, or of the decoded weights (A and B
    together: W~ -> -W~, a term of Y is x_k w~_k) changes outputs but no
    normaliser, and every normaliser bounds its output."""
    g = np.random.Generator(np.random.PCG64(92))
    M, N, K, d = 3, 5, 32, 4
    X, dY = g.standard_normal((M, K)), g.standard_normal((M, N))
    A, B = g.standard_normal((d, d)), g.standard_normal(d)
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    mask = g.random((N, K)) < 0.8
    base = _all_outputs(X, dY, z, mask, A, B)
    for v, dn in _NORMS:
        assert np.all(np.abs(base[v]) <= base[dn] * (1 + 1e-13)), v
    for flipped in (_all_outputs(-X, dY, z, mask, A, B), _all_outputs(X, -dY, z, mask, A, B),
                    _all_outputs(X, dY, z, mask, -A, -B)):
        for _, dn in _NORMS:
            assert np.allclose(flipped[dn], base[dn], rtol=1e-13, atol=0), dn


# ---------------------------------------------------------------- DGE (curve unpinned)
def test_dge_small_k_limit_is_the_ste_mask():
    """As k -> 0 the DGE factor tends to the STE's clamp mask (1 on [0, 3], 0
    outside); checked with an explicit small-k expansion bound."""
    w = np.array([-1.0, -1e-9, 0.0, 0.2, 0.5, 1.49, 1.5, 2.7, 3.0, 3.0001, 7.0])
    k = 1e-3
    g = O.dge_derivative(w, k)
    mask = ((w >= 0) & (w <= 3)).astype(np.float64)
    # k/(2 tanh(k/2)) = 1 + k^2/12 + ..., sech^2(k x) = 1 - k^2 x^2 + ...: |g - 1| <= k^2 inside
    assert np.all(np.abs(g - mask) <= k * k)


def test_dge_curve_is_a_staircase_through_the_integers():
    """phi_k equals w at the integers, is continuous at them, steps at the
    half-integers, and its derivative matches central differences of phi_k."""
    for k in (0.5, 4.0, 20.0):
        for n in (0.0, 1.0, 2.0, 3.0):
            assert O.dge_phi(n, k) == pytest.approx(n, abs=1e-12)
        for n in (1.0, 2.0):
            assert O.dge_phi(n - 1e-12, k) == pytest.approx(O.dge_phi(n + 1e-12, k), abs=1e-9)
        ws = np.linspace(0.01, 2.99, 97)
        ws = ws[np.abs(ws - np.round(ws)) > 1e-3]
        h = 1e-6
        fd = (O.dge_phi(ws + h, k) - O.dge_phi(ws - h, k)) / (2 * h)
        assert np.allclose(fd, O.dge_derivative(ws, k), rtol=1e-6, atol=1e-6)
    # large k approaches rounding away from the steps
    ws = np.array([0.2, 0.8, 1.3, 2.6])
    assert np.allclose(O.dge_phi(ws, 200.0), np.rint(ws), atol=1e-12)


def test_dge_backward_is_ste_times_the_factor():
    """dWp under DGE equals the STE dWp (all mask bits set) scaled by phi_k'."""
    g = np.random.Generator(np.random.PCG64(1500))
    M, N, K, d = 3, 5, 16, 4
    X = g.standard_normal((M, K))
    dY = g.standard_normal((M, N))
    Wp = g.uniform(-0.5, 3.5, size=(N, K))
    z, _ = O.assign(Wp)
    A = g.standard_normal((d, d))
    dWp, _ = O.backward_dge_dwp(X, dY, z, Wp, A, 3.0)
    bw = O.backward(X, dY, z, np.ones((N, K), bool), A, np.zeros(d))
    assert np.allclose(dWp, bw["dWp"] * O.dge_derivative(Wp, 3.0), rtol=1e-13, atol=1e-13)
    assert np.all(dWp[(Wp < 0) | (Wp > 3)] == 0)


# ---------------------------------------------------------------- (A, B) refit
def _fit_case(d, N, K, seed, noise=0.0):
    g = np.random.Generator(np.random.PCG64(seed))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A = g.standard_normal((d, d))
    B = g.standard_normal(d)
    W0 = O.decode(z, A, B) + noise * g.standard_normal((N, K))
    return g, z, A, B, W0


@pytest.mark.parametrize("d", [1, 2, 4, 8])
def test_fit_affine_recovers_an_exact_affine_map(d):
    """W0 generated as A z + B is fitted with zero residual: (A, B) come back."""
    _, z, A, B, W0 = _fit_case(d, 37, 16 * d, 500 + d)
    A2, B2 = O.fit_affine(W0, z, d)
    assert np.allclose(A2, A, atol=1e-10) and np.allclose(B2, B, atol=1e-10)
    assert O.fit_objective(W0, z, A2, B2) < 1e-18 * W0.size


@pytest.mark.parametrize("d", [2, 4, 8])
def test_fit_affine_equals_least_squares_on_the_stacked_design(d):
    """Row i of [A | B] solves the least-squares problem whose design matrix
    stacks [z, 1] of every vector, weighted by sqrt(h) of the vector's channel i
    (a different formulation from the oracle's normal equations)."""
    g, z, A, B, W0 = _fit_case(d, 23, 8 * d, 600 + d, noise=0.3)
    h = g.uniform(0.1, 2.0, size=8 * d)
    A2, B2 = O.fit_affine(W0, z, d, h)
    N, K = W0.shape
    for i in range(d):
        rows, rhs = [], []
        for n in range(N):
            for grp in range(K // d):
                k = grp * d + i
                s = math.sqrt(h[k])
                rows.append(s * np.append(z[n, grp * d:(grp + 1) * d].astype(np.float64), 1.0))
                rhs.append(s * W0[n, k])
        th = np.linalg.lstsq(np.array(rows), np.array(rhs), rcond=None)[0]
        assert np.allclose(A2[i], th[:d], atol=1e-10) and abs(B2[i] - th[d]) < 1e-10


def test_fit_affine_scalar_case_is_simple_linear_regression():
    """d = 1, h = 1: the per-matrix (s, zero point) of decoupleQ eq. (4) fitted by
    least squares has the textbook closed form s = cov(z, w) / var(z),
    b = mean(w) - s mean(z)."""
    _, z, _, _, W0 = _fit_case(1, 19, 40, 700, noise=0.5)
    A2, B2 = O.fit_affine(W0, z, 1)
    zz = z.astype(np.float64).ravel()
    ww = W0.ravel()
    s = np.sum((zz - zz.mean()) * (ww - ww.mean())) / np.sum((zz - zz.mean()) ** 2)
    assert A2[0, 0] == pytest.approx(s, rel=1e-12)
    assert B2[0] == pytest.approx(ww.mean() - s * zz.mean(), rel=1e-12, abs=1e-12)


def test_fit_affine_is_a_minimum():
    """Every small perturbation of (A, B) raises the weighted objective, and its
    central-difference gradient vanishes at the fit."""
    d = 4
    g, z, _, _, W0 = _fit_case(d, 11, 32, 800, noise=0.4)
    h = g.uniform(0.5, 1.5, size=32)
    A2, B2 = O.fit_affine(W0, z, d, h)
    f0 = O.fit_objective(W0, z, A2, B2, h)
    eps = 1e-4
    for t in range(d * d + d):
        dA = np.zeros((d, d))
        dB = np.zeros(d)
        if t < d * d:
            dA.flat[t] = eps
        else:
            dB[t - d * d] = eps
        fp = O.fit_objective(W0, z, A2 + dA, B2 + dB, h)
        fm = O.fit_objective(W0, z, A2 - dA, B2 - dB, h)
        assert fp > f0 and fm > f0
        assert abs(fp - fm) / (2 * eps) < 1e-6 * (1 + f0)


def test_fit_affine_singular_gram_gives_the_minimum_norm_solution():
    """A code position that never varies makes G singular (its column is a
    multiple of the ones column); the fit is then the minimum-norm
    least-squares solution, which lstsq also returns."""
    d = 4
    g, z, _, _, W0 = _fit_case(d, 17, 32, 900, noise=0.2)
    z = z.copy()
    z[:, 2::d] = 2                      # position 2 of every vector is always 2
    A2, B2 = O.fit_affine(W0, z, d)
    N, K = W0.shape
    for i in range(d):
        D = np.array([np.append(z[n, grp * d:(grp + 1) * d].astype(np.float64), 1.0)
                      for n in range(N) for grp in range(K // d)])
        y = np.array([W0[n, grp * d + i] for n in range(N) for grp in range(K // d)])
        th = np.linalg.lstsq(D, y, rcond=None)[0]
        assert np.allclose(A2[i], th[:d], atol=1e-9) and abs(B2[i] - th[d]) < 1e-9


def test_fit_affine_weights_scale_and_mask():
    """Scaling h leaves the fit unchanged; h that is zero outside a set of
    input channels fits those channels only."""
    d = 4
    g, z, _, _, W0 = _fit_case(d, 13, 64, 1000, noise=0.3)
    h = g.uniform(0.2, 1.0, size=64)
    A1, B1 = O.fit_affine(W0, z, d, h)
    A7, B7 = O.fit_affine(W0, z, d, 7.0 * h)
    assert np.allclose(A1, A7, atol=1e-12) and np.allclose(B1, B7, atol=1e-12)
    keep = np.zeros(64)
    keep[:32] = 1.0
    Am, Bm = O.fit_affine(W0, z, d, keep)
    As, Bs = O.fit_affine(W0[:, :32], z[:, :32], d)
    assert np.allclose(Am, As, atol=1e-12) and np.allclose(Bm, Bs, atol=1e-12)


def test_fit_planted_mistake_is_caught():
    """Normal equations that pair channel i's weight with coordinate j's codes
    (a transposed right-hand side) fail the exact-recovery pin."""
    d = 4
    _, z, A, B, W0 = _fit_case(d, 37, 64, 504)
    G, R = O.fit_affine_normal(W0, z, d)
    th = np.linalg.solve(G[1], R[2])  # the right-hand side of the wrong coordinate
    assert not np.allclose(th[:d], A[1], atol=1e-6)


# ---------------------------------------------------------------- refit under the full Hessian H
def _calib_hessian(g, K, n=None, ridge=0.05):
    """H = X^T X / n of correlated calibration rows (a shared component and a
    few outlier channels), plus a ridge: symmetric positive definite and far
    from diagonal."""
    n = n or 3 * K
    X = g.standard_normal((n, K)) + 0.8 * g.standard_normal((n, 1))
    X[:, g.choice(K, max(1, K // 16), replace=False)] *= 6.0
    return X.T @ X / n + ridge * np.eye(K)


@pytest.mark.parametrize("d", [1, 2, 4, 8])
def test_fit_affine_h_recovers_an_exact_affine_map(d):
    """W0 generated as A z + B is fitted with zero objective under any positive
    definite H: (A, B) come back."""
    g, z, A, B, W0 = _fit_case(d, 29, 8 * d, 1700 + d)
    H = _calib_hessian(g, 8 * d)
    A2, B2 = O.fit_affine_h(W0, z, d, H)
    assert np.allclose(A2, A, atol=1e-9) and np.allclose(B2, B, atol=1e-9)
    assert O.fit_objective_h(W0, z, A2, B2, H) < 1e-16 * np.abs(W0).sum() ** 2


@pytest.mark.parametrize("d", [2, 4, 8])
def test_fit_affine_h_equals_least_squares_with_the_hessian_root(d):
    """The objective is sum_n |H^(1/2) (Phi_n theta - w0_n)|^2 with Phi_n the
    linear map from theta = [A | B] to the decoded row n; stacking
    H^(1/2) Phi_n over the rows and solving by lstsq (a different formulation:
    a matrix square root and an orthogonal factorisation instead of the normal
    equations) gives the same (A, B)."""
    g, z, A, B, W0 = _fit_case(d, 13, 6 * d, 1800 + d, noise=0.3)
    K = 6 * d
    H = _calib_hessian(g, K)
    ev, V = np.linalg.eigh(H)
    Hr = (V * np.sqrt(ev)) @ V.T                       # H^(1/2)
    N = W0.shape[0]
    rows, rhs = [], []
    for n in range(N):
        Phi = np.zeros((K, d * (d + 1)))
        for grp in range(K // d):
            zt = np.append(z[n, grp * d:(grp + 1) * d].astype(np.float64), 1.0)
            for i in range(d):
                Phi[grp * d + i, i * (d + 1):(i + 1) * (d + 1)] = zt
        rows.append(Hr @ Phi)
        rhs.append(Hr @ W0[n])
    th = np.linalg.lstsq(np.vstack(rows), np.concatenate(rhs), rcond=None)[0].reshape(d, d + 1)
    A2, B2 = O.fit_affine_h(W0, z, d, H)
    assert np.allclose(A2, th[:, :d], atol=1e-9) and np.allclose(B2, th[:, d], atol=1e-9)


@pytest.mark.parametrize("d", [1, 4, 8])
def test_fit_affine_h_with_a_diagonal_hessian_is_the_weighted_fit(d):
    """H = diag(h) decouples the output coordinates: the result is the
    per-channel weighted fit (fit_affine with weights h)."""
    g, z, _, _, W0 = _fit_case(d, 21, 8 * d, 1900 + d, noise=0.4)
    h = g.uniform(0.2, 3.0, size=8 * d)
    A1, B1 = O.fit_affine(W0, z, d, h)
    A2, B2 = O.fit_affine_h(W0, z, d, np.diag(h))
    assert np.allclose(A1, A2, atol=1e-10) and np.allclose(B1, B2, atol=1e-10)


def test_fit_affine_h_is_a_minimum_and_scale_invariant():
    """Every small perturbation of (A, B) raises sum_n r_n^T H r_n, its
    central-difference gradient vanishes at the fit, and scaling H leaves the
    fit unchanged."""
    d = 4
    g, z, _, _, W0 = _fit_case(d, 11, 32, 2000, noise=0.4)
    H = _calib_hessian(g, 32)
    A2, B2 = O.fit_affine_h(W0, z, d, H)
    A5, B5 = O.fit_affine_h(W0, z, d, 5.0 * H)
    assert np.allclose(A2, A5, atol=1e-11) and np.allclose(B2, B5, atol=1e-11)
    f0 = O.fit_objective_h(W0, z, A2, B2, H)
    eps = 1e-4
    for t in range(d * d + d):
        dA = np.zeros((d, d))
        dB = np.zeros(d)
        if t < d * d:
            dA.flat[t] = eps
        else:
            dB[t - d * d] = eps
        fp = O.fit_objective_h(W0, z, A2 + dA, B2 + dB, H)
        fm = O.fit_objective_h(W0, z, A2 - dA, B2 - dB, H)
        assert fp > f0 and fm > f0
        assert abs(fp - fm) / (2 * eps) < 1e-6 * (1 + f0)


def test_fit_affine_h_beats_the_diagonal_fit_on_a_correlated_hessian():
    """On a correlated H the full-H fit reaches a lower H-objective than the
    fit that keeps only diag(H); dropping the off-diagonal blocks (g != g') of
    the normal equations, a plausible mistake, is caught by the stacked
    least-squares pin's answer."""
    d = 4
    g, z, _, _, W0 = _fit_case(d, 15, 32, 2100, noise=0.5)
    H = _calib_hessian(g, 32)
    Af, Bf = O.fit_affine_h(W0, z, d, H)
    Ad, Bd = O.fit_affine(W0, z, d, np.diag(H))
    assert O.fit_objective_h(W0, z, Af, Bf, H) < O.fit_objective_h(W0, z, Ad, Bd, H)
    # block-diagonal mistake: H with its off-diagonal d x d blocks removed
    Hb = np.zeros_like(H)
    for grp in range(32 // d):
        sl = slice(grp * d, (grp + 1) * d)
        Hb[sl, sl] = H[sl, sl]
    Ab, Bb = O.fit_affine_h(W0, z, d, Hb)
    assert not np.allclose(Ab, Af, atol=1e-6)


# ---------------------------------------------------------------- H-aware sequential assignment
def _spd(g, K, n=None, ridge=0.05):
    """A correlated symmetric positive definite K x K matrix: X^T X / n from
    rows with a shared component, plus a ridge."""
    n = n or 4 * K
    X = g.standard_normal((n, K)) + 0.8 * g.standard_normal((n, 1))
    return X.T @ X / n + ridge * np.eye(K)


def _eq11_direct(p, Q):
    """The pages' procedure written out for one row: fix element j by rounding
    and clipping the j-th element of the continuous minimiser of
    1/2 (z - p)^T Q (z - p) over the elements not fixed yet (a linear solve on
    the sub-block of Q), then move on to j + 1."""
    K = len(p)
    z = np.zeros(K)
    for j in range(K):
        f, x = slice(j, K), slice(0, j)
        y = p[f] - np.linalg.solve(Q[f, f], Q[f, x] @ (z[x] - p[x]))
        z[j] = np.clip(np.rint(y[0]), 0, 3)
    return z


def test_ldl_upper_reconstructs_the_matrix():
    g = np.random.Generator(np.random.PCG64(71))
    Q = _spd(g, 12)
    U, D = O.ldl_upper(Q)
    I = np.eye(12)
    assert np.array_equal(U, np.triu(U, 1))
    assert np.all(D > 0)
    assert np.allclose((I + U) @ np.diag(D) @ (I + U).T, Q, atol=1e-12)


def test_ldlq_with_a_diagonal_hessian_is_round_and_clamp(golden_dir):
    """Q diagonal: no compensation, the codes are those of the assignment step
    (ties to even, clamping, the golden tie cases included)."""
    g = np.random.Generator(np.random.PCG64(72))
    rows = [ln.split() for ln in _read(golden_dir, "round_clamp_ties.txt")]
    w = np.array([_f32(r[0]) for r in rows if np.isfinite(_f32(r[0]))], dtype=np.float64)
    K = len(w)
    P = np.stack([w, g.uniform(-0.5, 3.5, K), g.uniform(-2, 5, K)])
    U, _ = O.ldl_upper(np.diag(g.uniform(0.1, 3.0, K)))
    assert np.array_equal(U, np.zeros((K, K)))
    assert np.array_equal(O.ldlq_assign(P, U), O.assign(P.astype(np.float32))[0])


def test_ldlq_equals_the_eq11_procedure_solved_directly():
    """The factor form gives the same codes as re-solving the remaining
    elements with a linear solve at every step."""
    g = np.random.Generator(np.random.PCG64(73))
    for K in (1, 2, 5, 10):
        Q = _spd(g, K)
        U, _ = O.ldl_upper(Q)
        P = g.uniform(-0.5, 3.5, size=(40, K))
        Z = O.ldlq_assign(P, U)
        for n in range(40):
            assert np.array_equal(Z[n], _eq11_direct(P[n], Q)), (K, n)


def test_ldlq_choice_is_the_best_code_by_exhaustive_search():
    """At every step the chosen code minimises, over all four codes, the
    objective with the earlier codes fixed and the later elements at their
    continuous optimum."""
    g = np.random.Generator(np.random.PCG64(74))
    K = 7
    Q = _spd(g, K)
    U, _ = O.ldl_upper(Q)
    P = g.uniform(-1.0, 4.0, size=(25, K))
    Z = O.ldlq_assign(P, U)
    for n in range(25):
        p = P[n]
        for j in range(K):
            best, arg = np.inf, -1
            for c in range(4):
                z = np.concatenate([Z[n, :j].astype(np.float64), [c]])
                r = slice(j + 1, K)
                x = slice(0, j + 1)
                rest = p[r] - np.linalg.solve(Q[r, r], Q[r, x] @ (z - p[x])) if j + 1 < K else p[r]
                full = np.concatenate([z, rest]) - p
                val = 0.5 * full @ Q @ full
                if val < best:
                    best, arg = val, c
            assert Z[n, j] == arg, (n, j)


def test_ldlq_equals_the_inverse_cholesky_error_feedback_form():
    """The same codes from the other standard form of the update: after fixing
    element j, subtract (t_j - z_j) / L[j, j] * L[j, >j] from the later targets,
    with L^T L = Q^-1 and L upper triangular."""
    g = np.random.Generator(np.random.PCG64(75))
    K = 24
    Q = _spd(g, K)
    U, _ = O.ldl_upper(Q)
    L = np.linalg.cholesky(np.linalg.inv(Q)).T
    P = g.uniform(-0.5, 3.5, size=(30, K))
    T = P.copy()
    Zg = np.zeros((30, K))
    for j in range(K):
        Zg[:, j] = np.clip(np.rint(T[:, j]), 0, 3)
        T[:, j + 1:] -= np.outer((T[:, j] - Zg[:, j]) / L[j, j], L[j, j + 1:])
    assert np.array_equal(O.ldlq_assign(P, U), Zg)


def test_code_space_objective_is_the_weight_space_objective():
    """1/2 (z - p)^T Q (z - p) with Q = Abar^T H Abar and p = Abar^-1 (w0 - bbar)
    equals 1/2 (W~ - w0)^T H (W~ - w0) with W~ decoded from the codes."""
    g = np.random.Generator(np.random.PCG64(76))
    d, K, N = 4, 16, 6
    A = np.eye(d) * 0.3 + 0.05 * g.standard_normal((d, d))
    B = g.standard_normal(d)
    H = _spd(g, K)
    W0 = g.standard_normal((N, K))
    Z = g.integers(0, 4, size=(N, K)).astype(np.uint8)
    R = O.decode(Z, A, B) - W0
    direct = 0.5 * np.einsum("nk,kl,nl->n", R, H, R)
    got = O.ldlq_objective(O.code_targets(W0, A, B), O.code_space_hessian(H, A), Z)
    assert np.allclose(got, direct, rtol=1e-10, atol=1e-12)


def test_ldlq_targets_reproduce_the_choices():
    g = np.random.Generator(np.random.PCG64(77))
    K = 32
    U, _ = O.ldl_upper(_spd(g, K))
    P = g.uniform(-0.5, 3.5, size=(16, K))
    Z = O.ldlq_assign(P, U)
    T, S = O.ldlq_targets(P, U, Z)
    assert np.array_equal(np.clip(np.rint(T), 0, 3), Z)
    assert np.all(S >= np.abs(T) - 1e-12)


def test_ldlq_lowers_the_objective_on_a_correlated_hessian():
    """The point of the compensation: on a strongly correlated Q the mean
    objective is below that of plain rounding (fixed seed, 200 rows)."""
    g = np.random.Generator(np.random.PCG64(78))
    K = 32
    Q = _spd(g, K, ridge=0.01)
    U, _ = O.ldl_upper(Q)
    P = g.uniform(-0.5, 3.5, size=(200, K))
    seq = O.ldlq_objective(P, Q, O.ldlq_assign(P, U)).mean()
    rnd = O.ldlq_objective(P, Q, np.clip(np.rint(P), 0, 3)).mean()
    assert seq < 0.8 * rnd


def test_ldlq_planted_mistakes_are_caught():
    """Feeding back the error of the compensated target (t_i - z_i) instead of
    p_i - z_i, or factoring Q without reversing its order (the transposed
    lower factor in place of the upper one), breaks agreement with the direct
    procedure."""
    g = np.random.Generator(np.random.PCG64(79))
    K = 10
    Q = _spd(g, K)
    U, _ = O.ldl_upper(Q)
    P = g.uniform(-0.5, 3.5, size=(40, K))
    ref = np.stack([_eq11_direct(P[n], Q) for n in range(40)])
    T = P.copy()
    Zw = np.zeros_like(P)
    for j in range(K):
        Zw[:, j] = np.clip(np.rint(T[:, j]), 0, 3)
        T[:, j + 1:] += np.outer(T[:, j] - Zw[:, j], U[j, j + 1:])
    assert not np.array_equal(Zw, ref)
    C = np.linalg.cholesky(Q)  # the factor without the reversal: Q = (I + L) D (I + L)^T, L lower
    wrong = (C / np.diag(C)[None, :] - np.eye(K)).T
    assert not np.array_equal(O.ldlq_assign(P, wrong), ref)


# ---------------------------------------------------------------- metric
def test_rel_err_semantics():
    assert O.rel_err([1.0, 2.0], [1.0, 2.5], [1.0, 5.0]) == pytest.approx(0.1)
    assert O.rel_err([0.0], [0.0], [0.0]) == 0.0
    assert O.rel_err([1e-30], [0.0], [0.0]) == float("inf")
    assert O.rel_err([float("nan")], [0.0], [1.0]) == float("inf")


def test_planted_mistakes_are_caught(golden_dir):
    """A transposed A, a dropped B, or a wrong tie rule in a copy of the
    oracle's formulas each fail a pin above (checked here directly)."""
    A = np.array([[1.0, 2.0], [3.0, 4.0]])
    B = np.array([10.0, 20.0])
    z = np.array([[1, 3]], dtype=np.uint8)
    assert not np.array_equal(O.decode(z, A.T, B), [[17.0, 35.0]])
    assert not np.array_equal(O.decode(z, A, 0 * B), [[17.0, 35.0]])
    w = np.array([2.5], dtype=np.float32)
    assert np.floor(w + 0.5)[0] != O.assign(w)[0][0]   # half-up would give 3


def test_ldlq_validity_checker_is_not_vacuous():
    """The check the GPU tests apply to H-aware codes (every code must be the
    rule's choice for its own fp64 target, except within the fp32 band of a
    rounding boundary) accepts the oracle's codes and rejects plain rounding,
    a single code flipped away from any tie, and shifted codes; a tie sitting
    inside the band may go either way."""
    from tests.gpu_util import ldlq_check
    g = np.random.Generator(np.random.PCG64(80))
    K = 128
    Q = _spd(g, K, ridge=0.01)
    U, _ = O.ldl_upper(Q)
    U = U.astype(np.float32)
    P = g.uniform(-0.5, 3.5, size=(12, K)).astype(np.float32)
    Z = O.ldlq_assign(P, U)
    assert ldlq_check(P, U, Z)[0] == 0
    assert ldlq_check(P, U, np.clip(np.rint(P), 0, 3).astype(np.uint8))[0] > 0
    T, _ = O.ldlq_targets(P, U, Z)
    far = np.argwhere((np.abs(T - (np.floor(T) + 0.5)) > 0.2) & (T > 0.3) & (T < 2.7))
    n, j = far[0]
    Zf = Z.copy()
    Zf[n, j] = 3 - Zf[n, j] if Zf[n, j] in (0, 3) else Zf[n, j] + 1
    assert ldlq_check(P, U, Zf)[0] >= 1
    assert ldlq_check(P, U, np.minimum(Z + 1, 3))[0] > 0
    # an exact tie (target 1.5 with no compensation) is valid rounded up or down
    P1 = np.full((1, 64), 0.25, dtype=np.float32)
    P1[0, 7] = 1.5
    U0 = np.zeros((64, 64), dtype=np.float32)
    Zt = O.ldlq_assign(P1, U0)
    Zu = Zt.copy()
    Zu[0, 7] = 1 if Zt[0, 7] == 2 else 2
    assert ldlq_check(P1, U0, Zt)[0] == 0 and ldlq_check(P1, U0, Zu)[0] == 0

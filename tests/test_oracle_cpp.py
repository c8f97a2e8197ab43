"""Pins for the C++ fp64 oracle (oracle/lcvq_oracle.cpp).

The C++ oracle must pass the same pins as the numpy one: every pin of the
assign, pack, decode, forward, backward, DGE, H-aware assignment and (A, B)
refit functions runs here with the C++ functions put in place of the numpy ones.  It must also agree with the numpy
oracle (an independent restatement of the same definitions) on random ragged
cases, and give the same bits whatever the thread count.  CPU only.
"""

import numpy as np
import pytest

from oracle import cpp as C
from oracle import lcvq_oracle as O
from tests import test_oracle_pins as P

SUBSTITUTED = ("assign", "pack_codes", "unpack_codes", "pack_mask", "unpack_mask", "decode",
               "forward", "backward", "ldlq_assign", "fit_affine", "fit_affine_h", "dge_phi",
               "dge_derivative")


@pytest.fixture
def cpp_oracle(monkeypatch):
    for name in SUBSTITUTED:
        monkeypatch.setattr(O, name, getattr(C, name))
    return O


PINS = [
    ("round/clamp ties golden", lambda gd: P.test_round_clamp_golden(gd)),
    ("nearest code d=1", lambda gd: P.test_assign_is_nearest_code_brute_force(1)),
    ("nearest code d=2", lambda gd: P.test_assign_is_nearest_code_brute_force(2)),
    ("nearest code d=4", lambda gd: P.test_assign_is_nearest_code_brute_force(4)),
    ("nearest code d=8", lambda gd: P.test_assign_brute_force_d8()),
    ("scalar quantizer", lambda gd: P.test_scalar_special_case_matches_uniform_quantizer()),
    ("code statistics", lambda gd: P.test_code_statistics_uniform_and_normal()),
    ("pack golden", lambda gd: P.test_pack_golden(gd)),
    ("mask golden", lambda gd: P.test_mask_golden(gd)),
    ("pack bijection", lambda gd: P.test_pack_is_bijection_on_bytes()),
    ("d=8 vector is codebook index", lambda gd: P.test_packed_d8_vector_is_codebook_index()),
    ("decode golden", lambda gd: P.test_decode_golden(gd)),
    ("decode = codebook lookup", lambda gd: P.test_decode_equals_codebook_lookup()),
    ("decode scalar cross-d", lambda gd: P.test_decode_scalar_case_is_cross_d_invariant()),
    ("linear layer golden", lambda gd: P.test_linear_layer_golden(gd)),
    ("A=I, B=0 integer GEMM", lambda gd: P.test_forward_identity_is_integer_code_gemm()),
    ("linearity, 2^k scaling", lambda gd: P.test_forward_linearity_and_pow2_scaling()),
    ("direct = algebraic", lambda gd: P.test_forward_direct_equals_algebraic()),
    ("backward finite differences", lambda gd: P.test_backward_finite_differences_exact()),
    ("dWp STE surrogate", lambda gd: P.test_backward_dwp_ste_surrogate_finite_differences()),
    ("dB identity", lambda gd: P.test_db_identity_at_any_size()),
    ("normalisers = outputs without negative terms",
     lambda gd: P.test_normalisers_equal_the_outputs_when_no_term_is_negative()),
    ("normalisers ignore operand signs", lambda gd: P.test_normalisers_ignore_the_signs_of_the_operands()),
    ("H-aware: diagonal Hessian is round and clamp",
     lambda gd: P.test_ldlq_with_a_diagonal_hessian_is_round_and_clamp(gd)),
    ("H-aware: eq. (11) procedure solved directly",
     lambda gd: P.test_ldlq_equals_the_eq11_procedure_solved_directly()),
    ("H-aware: best code by exhaustive search",
     lambda gd: P.test_ldlq_choice_is_the_best_code_by_exhaustive_search()),
    ("H-aware: inverse-Cholesky feedback form",
     lambda gd: P.test_ldlq_equals_the_inverse_cholesky_error_feedback_form()),
    ("H-aware: targets reproduce the choices", lambda gd: P.test_ldlq_targets_reproduce_the_choices()),
    ("H-aware: lower objective than rounding",
     lambda gd: P.test_ldlq_lowers_the_objective_on_a_correlated_hessian()),
    ("DGE: small-k limit is the STE mask", lambda gd: P.test_dge_small_k_limit_is_the_ste_mask()),
    ("DGE: staircase through the integers",
     lambda gd: P.test_dge_curve_is_a_staircase_through_the_integers()),
    ("DGE: backward is STE times the factor", lambda gd: P.test_dge_backward_is_ste_times_the_factor()),
    ("refit: exact recovery d=1", lambda gd: P.test_fit_affine_recovers_an_exact_affine_map(1)),
    ("refit: exact recovery d=8", lambda gd: P.test_fit_affine_recovers_an_exact_affine_map(8)),
    ("refit: stacked-design least squares d=4",
     lambda gd: P.test_fit_affine_equals_least_squares_on_the_stacked_design(4)),
    ("refit: scalar case is linear regression",
     lambda gd: P.test_fit_affine_scalar_case_is_simple_linear_regression()),
    ("refit: a minimum", lambda gd: P.test_fit_affine_is_a_minimum()),
    ("refit: singular Gram, minimum norm",
     lambda gd: P.test_fit_affine_singular_gram_gives_the_minimum_norm_solution()),
    ("refit: weights scale and mask", lambda gd: P.test_fit_affine_weights_scale_and_mask()),
    ("full-H refit: exact recovery d=2", lambda gd: P.test_fit_affine_h_recovers_an_exact_affine_map(2)),
    ("full-H refit: exact recovery d=8", lambda gd: P.test_fit_affine_h_recovers_an_exact_affine_map(8)),
    ("full-H refit: least squares with H^1/2 d=4",
     lambda gd: P.test_fit_affine_h_equals_least_squares_with_the_hessian_root(4)),
    ("full-H refit: diagonal H is the weighted fit d=8",
     lambda gd: P.test_fit_affine_h_with_a_diagonal_hessian_is_the_weighted_fit(8)),
    ("full-H refit: a minimum, scale invariant",
     lambda gd: P.test_fit_affine_h_is_a_minimum_and_scale_invariant()),
    ("full-H refit: beats the diagonal fit",
     lambda gd: P.test_fit_affine_h_beats_the_diagonal_fit_on_a_correlated_hessian()),
]


@pytest.mark.parametrize("name,pin", PINS, ids=[p[0] for p in PINS])
def test_cpp_oracle_passes_the_pins(name, pin, cpp_oracle, golden_dir):
    pin(golden_dir)


def _case(seed, M, N, K, d, scale=1.0):
    g = np.random.Generator(np.random.PCG64(seed))
    X = scale * g.standard_normal((M, K))
    dY = g.standard_normal((M, N))
    Wp = g.uniform(-1.0, 4.0, size=(N, K)).astype(np.float32)
    A = g.standard_normal((d, d))
    B = g.standard_normal(d)
    return X, dY, Wp, A, B


@pytest.mark.parametrize("M,N,K,d", [(1, 8, 64, 8), (5, 24, 192, 4), (17, 40, 72, 2),
                                     (3, 16, 40, 1), (0, 8, 64, 8)])
def test_cpp_agrees_with_numpy(M, N, K, d):
    X, dY, Wp, A, B = _case(100 + M + N + K + d, M, N, K, d)
    z, mask = C.assign(Wp)
    zn, maskn = O.assign(Wp)
    assert np.array_equal(z, zn) and np.array_equal(mask, maskn)
    assert np.array_equal(C.pack_codes(z), O.pack_codes(z))
    assert np.array_equal(C.pack_mask(mask), O.pack_mask(mask))
    Y, D = C.forward(X, z, A, B)
    Yn, Dn = O.forward(X, z, A, B)
    if M:
        assert O.rel_err(Y, Yn, Dn) < 1e-13 and np.allclose(D, Dn, rtol=1e-13, atol=0)
    bw, bn = C.backward(X, dY, z, mask, A, B), O.backward(X, dY, z, mask, A, B)
    for k in ("dX", "dA", "dB", "dWp"):
        if bn[k].size:
            assert O.rel_err(bw[k], bn[k], bn["D_" + k]) < 1e-13, k
            assert np.allclose(bw["D_" + k], bn["D_" + k], rtol=1e-13, atol=0), k


def test_cpp_non_finite_and_ties():
    w = np.array([np.nan, np.inf, -np.inf, 0.5, 1.5, 2.5, 3.5, -0.5, 2.4999999, -0.0, 3.0, 3.0000002],
                 dtype=np.float32)
    z, m = C.assign(w)
    zn, mn = O.assign(w)
    assert z.tolist() == zn.tolist() == [0, 3, 0, 0, 2, 2, 3, 0, 2, 0, 3, 3]
    assert m.tolist() == mn.tolist()


def test_cpp_results_do_not_depend_on_the_thread_count():
    X, dY, Wp, A, B = _case(7, 9, 40, 128, 8)
    z, mask = C.assign(Wp)
    Y1, D1 = C.forward(X, z, A, B, threads=1)
    Y7, D7 = C.forward(X, z, A, B, threads=7)
    assert np.array_equal(Y1, Y7) and np.array_equal(D1, D7)
    b1 = C.backward(X, dY, z, mask, A, B, threads=1)
    b5 = C.backward(X, dY, z, mask, A, B, threads=5)
    for k in b1:
        assert np.array_equal(b1[k], b5[k]), k


def test_cpp_h_aware_assignment_equals_numpy_on_exact_inputs_at_any_thread_count():
    """On a 1/32 grid of targets and a 1/64 grid of factor entries every fp64
    operation of the rule is exact, so the two oracles' codes agree bit for
    bit whatever their summation orders; rounding ties are on the grid."""
    from bit_weight_only_lcvq_b200 import synth
    g = np.random.Generator(np.random.PCG64(123))
    P_ = synth.targets_dyadic(37, 192, g)
    U = synth.strict_upper_dyadic(192, g)
    Zn = O.ldlq_assign(P_, U)
    assert np.array_equal(C.ldlq_assign(P_, U, threads=1), Zn)
    assert np.array_equal(C.ldlq_assign(P_, U, threads=6), Zn)


@pytest.mark.parametrize("d", [1, 2, 4, 8])
def test_cpp_refits_agree_with_numpy(d):
    """Both refits, random codes and weights, against the numpy oracle (its own
    einsum contractions and LAPACK pseudo-inverse), to fp64 rounding."""
    g = np.random.Generator(np.random.PCG64(200 + d))
    N, K = 29, 16 * d
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    W0 = g.standard_normal((N, K))
    h = g.uniform(0.5, 2.0, K)
    Xc = g.standard_normal((2 * K, K))
    H = Xc.T @ Xc / (2 * K) + 0.01 * np.eye(K)
    for got, ref in ((C.fit_affine(W0, z, d, h), O.fit_affine(W0, z, d, h)),
                     (C.fit_affine(W0, z, d), O.fit_affine(W0, z, d)),
                     (C.fit_affine_h(W0, z, d, H), O.fit_affine_h(W0, z, d, H))):
        for a, b in zip(got, ref):
            assert np.allclose(a, b, rtol=1e-10, atol=1e-12 * np.max(np.abs(b))), d


def test_cpp_dge_agrees_with_numpy():
    w = np.concatenate([np.linspace(-1.0, 4.0, 2001), [0.0, 1.0, 2.0, 3.0, np.nan, np.inf, -np.inf]])
    for k in (1e-3, 0.5, 4.0, 30.0):
        assert np.allclose(C.dge_derivative(w, k), O.dge_derivative(w, k), rtol=1e-13, atol=0)
        fin = np.isfinite(w)
        assert np.allclose(C.dge_phi(w[fin], k), O.dge_phi(w[fin], k), rtol=1e-13, atol=1e-15)


def test_cpp_planted_transpose_is_caught(monkeypatch, golden_dir):
    """A decode with A transposed, fed through the C++ forward, fails the
    hand-worked layer: the substituted pins are not vacuous for this oracle."""
    for name in SUBSTITUTED:
        monkeypatch.setattr(O, name, getattr(C, name))
    fwd = C.forward
    monkeypatch.setattr(O, "forward", lambda X, z, A, B: fwd(X, z, np.asarray(A).T, B))
    with pytest.raises(AssertionError):
        P.test_linear_layer_golden(golden_dir)


def test_cpp_forward_from_packed_codes_equals_forward():
    X, _, Wp, A, B = _case(9, 4, 24, 256, 8)
    z, _ = C.assign(Wp)
    Y, D = C.forward(X, z, A, B)
    Yp, Dp = C.forward_packed(X, C.pack_codes(z), 256, A, B)
    assert np.array_equal(Y, Yp) and np.array_equal(D, Dp)

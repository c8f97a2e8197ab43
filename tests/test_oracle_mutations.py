"""The pins are not vacuous.

Each case plants one plausible mistake in a single oracle function on the CPU.
It then runs the pins that should notice, and at least one must fail. The
mistakes:
- a transposed or dropped operand;
- a flipped sign;
- a wrong tie or bit order;
- a lost mask;
- a normaliser built from signed terms;
- a dropped intercept or normaliser;
- missing error feedback;
- an unreversed factorisation;
- a Hessian with its cross-position coupling dropped, or left out of one side.

Nothing here touches a GPU.
"""

import numpy as np
import pytest

from oracle import lcvq_oracle as O
from tests import test_oracle_pins as P

_decode, _assign, _pack = O.decode, O.assign, O.pack_codes
_backward, _fit, _ldlq = O.backward, O.fit_affine, O.ldlq_assign
_pack_mask, _dge_d, _ldl, _hess = O.pack_mask, O.dge_derivative, O.ldl_upper, O.code_space_hessian
_fit_h, _fit_h_normal = O.fit_affine_h, O.fit_affine_h_normal
_forward = O.forward


def _fit_h_block_diagonal(W0, z, d, H):  # the (g, g') coupling of H dropped
    H = np.asarray(H, dtype=np.float64)
    Hb = np.zeros_like(H)
    for g0 in range(0, H.shape[0], d):
        Hb[g0:g0 + d, g0:g0 + d] = H[g0:g0 + d, g0:g0 + d]
    return _fit_h(W0, z, d, Hb)


def _fit_h_rhs_without_h(W0, z, d, H):  # the right-hand side formed with H = I
    G, _ = _fit_h_normal(W0, z, d, H)
    _, R = _fit_h_normal(W0, z, d, np.eye(np.asarray(H).shape[0]))
    th = (np.linalg.pinv(G, rcond=O.PINV_RCOND, hermitian=True) @ R).reshape(d, d + 1)
    return th[:, :d].copy(), th[:, d].copy()


def _assign_half_up(Wp):
    z, mask = _assign(Wp)
    w = np.asarray(Wp, dtype=np.float64)
    up = np.clip(np.floor(np.where(np.isnan(w), 0.0, w) + 0.5), 0, 3).astype(np.uint8)
    return up, mask


def _pack_msb_first(z):
    z = np.asarray(z, dtype=np.uint8)
    n, k = z.shape
    return _pack(z.reshape(n, k // 4, 4)[:, :, ::-1].reshape(n, k))


def _backward_with(change):
    def bw(*args):
        out = dict(_backward(*args))
        change(out)
        return out
    return bw


def _negate_dx(o):
    o["dX"] = -o["dX"]


def _transpose_da(o):
    o["dA"] = o["dA"].T.copy()


def _signed_dwp_normaliser(o):  # |A| forgotten in D_dWp
    o["D_dWp"] = o["D_dWp"] * 0 + o["dWp"]


def _dwp_with_a_untransposed(X, dY, z, mask, A, B):  # dWp = mask * A G instead of A^T G
    return _backward(X, dY, z, mask, np.asarray(A).T, B) | {
        k: v for k, v in _backward(X, dY, z, mask, A, B).items() if k != "dWp"}


def _forward_signed_normaliser(X, z, A, B):  # D_Y = |X W~^T| instead of |X| |W~|^T
    Y, _ = _forward(X, z, A, B)
    return Y, np.abs(Y)


def _backward_no_mask(X, dY, z, mask, A, B):
    return _backward(X, dY, z, np.ones_like(mask, dtype=bool), A, B)


def _pack_mask_msb_first(mask):
    m = np.asarray(mask, dtype=np.uint8)
    n, k = m.shape
    return _pack_mask(m.reshape(n, k // 8, 8)[:, :, ::-1].reshape(n, k))


def _dge_unnormalised(Wp, k):  # the k / (2 tanh(k / 2)) factor forgotten
    return _dge_d(Wp, k) / (k / (2.0 * np.tanh(k / 2.0)))


def _ldl_lower_factor(Q):  # the factor without the row and column reversal
    Q = np.asarray(Q, dtype=np.float64)
    C = np.linalg.cholesky(Q)
    v = np.diag(C).copy()
    return np.triu((C / v[None, :] - np.eye(Q.shape[0])).T, 1), v * v


def _hessian_untransposed(H, A):  # Abar H Abar^T instead of Abar^T H Abar
    return _hess(H, np.asarray(A).T)


MUTATIONS = [
    ("decode: A transposed", "decode", lambda z, A, B: _decode(z, np.asarray(A).T, B),
     [lambda gd: P.test_decode_golden(gd), lambda gd: P.test_linear_layer_golden(gd)]),
    ("decode: B dropped", "decode", lambda z, A, B: _decode(z, A, 0.0 * np.asarray(B)),
     [lambda gd: P.test_decode_golden(gd)]),
    ("assign: ties rounded half up", "assign", _assign_half_up,
     [lambda gd: P.test_round_clamp_golden(gd)]),
    ("pack: most significant code first", "pack_codes", _pack_msb_first,
     [lambda gd: P.test_pack_golden(gd), lambda gd: P.test_packed_d8_vector_is_codebook_index()]),
    ("backward: dX sign flipped", "backward", _backward_with(_negate_dx),
     [lambda gd: P.test_backward_finite_differences_exact()]),
    ("backward: dA transposed", "backward", _backward_with(_transpose_da),
     [lambda gd: P.test_backward_finite_differences_exact()]),
    ("backward: clamp mask lost", "backward", _backward_no_mask,
     [lambda gd: P.test_backward_dwp_ste_surrogate_finite_differences()]),
    ("backward: dWp with A where A^T belongs", "backward", _dwp_with_a_untransposed,
     [lambda gd: P.test_backward_dwp_ste_surrogate_finite_differences()]),
    ("backward: dWp's normaliser from signed terms", "backward",
     _backward_with(_signed_dwp_normaliser),
     [lambda gd: P.test_normalisers_ignore_the_signs_of_the_operands()]),
    ("forward: normaliser from the signed product", "forward", _forward_signed_normaliser,
     [lambda gd: P.test_forward_identity_is_integer_code_gemm(),
      lambda gd: P.test_normalisers_ignore_the_signs_of_the_operands()]),
    ("refit: intercept dropped", "fit_affine", lambda W0, z, d, h=None: (_fit(W0, z, d, h)[0],
                                                                         np.zeros(d)),
     [lambda gd: P.test_fit_affine_recovers_an_exact_affine_map(4)]),
    ("H-aware assignment: no error feedback", "ldlq_assign",
     lambda Pm, U: _ldlq(Pm, np.zeros_like(np.asarray(U))),
     [lambda gd: P.test_ldlq_equals_the_eq11_procedure_solved_directly()]),
    ("mask: most significant bit first", "pack_mask", _pack_mask_msb_first,
     [lambda gd: P.test_mask_golden(gd)]),
    ("DGE: derivative not normalised", "dge_derivative", _dge_unnormalised,
     [lambda gd: P.test_dge_curve_is_a_staircase_through_the_integers()]),
    ("LDL: factor of the unreversed matrix", "ldl_upper", _ldl_lower_factor,
     [lambda gd: P.test_ldl_upper_reconstructs_the_matrix()]),
    ("code-space Hessian: A on the wrong side", "code_space_hessian", _hessian_untransposed,
     [lambda gd: P.test_code_space_objective_is_the_weight_space_objective()]),
    ("full-H refit: (g, g') coupling dropped", "fit_affine_h", _fit_h_block_diagonal,
     [lambda gd: P.test_fit_affine_h_equals_least_squares_with_the_hessian_root(4)]),
    ("full-H refit: right-hand side without H", "fit_affine_h", _fit_h_rhs_without_h,
     [lambda gd: P.test_fit_affine_h_recovers_an_exact_affine_map(4)]),
]


@pytest.mark.parametrize("name,target,mutant,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(name, target, mutant, pins, monkeypatch, golden_dir):
    for pin in pins:  # the pins pass on the oracle as written
        pin(golden_dir)
    monkeypatch.setattr(O, target, mutant)
    caught = 0
    for pin in pins:
        try:
            pin(golden_dir)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin noticed: {name}"

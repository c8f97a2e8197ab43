"""fp64 reference oracle for the LC-VQ hot path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The library and its Python binding
never import it, and it imports nothing from them; the two share no code.

What it computes, and where the method is stated
------------------------------------------------
Sources (cited below by these short names):

* "LC-QAT page": the technical summary of *LC-QAT: Data-Efficient 2-Bit QAT
  for LLMs via Linear-Constrained Vector Quantization* (gist.science,
  paper 2606.10531; Chinese, Portuguese and French editions say the same).
  - Methodology 1 "linear-constrained parameterization": codewords are
    ``c = A z + B`` with ``z`` in ``{0,1,2,3}^d`` and ``A`` (d x d), ``B`` (d)
    floating-point parameters shared within one weight matrix; index search
    becomes rounding and clamping followed by a linear projection, and
    gradients flow through the linear map.
  - Methodology 3 "training pipeline": proxy weights ``W_p`` are rounded and
    clamped to integers ``W_z`` and decoded as ``A W_z + B``; the forward is
    recast onto INT2 x FP16 matmul operators; the backward uses a gradient
    estimator through the rounding (DGE in the paper, STE in its ablation).
* "decoupleQ page": *decoupleQ: 2-bit post-training uniform quantization by
  decoupling parameters into integer and floating-point parts* (lryc.cn
  translation).  Eq. (1) fixes the linear-layer convention ``Y = X W~`` with
  ``W~`` of shape ``d_in x d_out``; eq. (3)/(4) are the scalar
  round/clip/affine special case used as a pin; eq. (5) and section 3.3 (the
  float part solved in closed form with the integer part fixed) define the
  least-squares refit of (A, B); eq. (6)-(11) (the integer part solved one
  element at a time, the rest re-solved without the integer constraint) define
  the H-aware sequential code assignment.

Readings where the pages are silent:

* rounding is round-half-to-even (numpy ``rint``); clamp to ``[0, 3]``;
  NaN -> 0, +Inf -> 3, -Inf -> 0;
* the STE clamp mask is ``0 <= W_p <= 3`` on the proxy weight itself;
* vectors are ``d`` consecutive elements along ``d_in``; ``A`` acts on column
  vectors (``c_i = sum_j A[i, j] z_j``);
* weights are stored ``[d_out][d_in]`` (the transpose of the decoupleQ
  ``W~``), so ``Y[m, n] = sum_k X[m, k] W~[n, k]``;
* packed format V1: 4 codes per byte, LSB first along ``d_in``; the clamp
  mask is 8 bits per byte, LSB first.

All arithmetic is fp64 after exact widening of the fp32/bf16 inputs.  Every
floating result comes with the per-element normaliser ``D`` = the sum of the
absolute values of the terms that make that element; the parity metric is
``|got - ref| / D``.

Parity status: every function here is pinned by a CPU test against values
that do not come from this module (brute force, closed forms, hand-worked
golden files, finite differences, distribution statistics).  No function is
"parity unpinned".
"""

from __future__ import annotations

import numpy as np

CODE_MAX = 3  # z in {0, 1, 2, 3}: 2 bits per weight


# --------------------------------------------------------------------------
# code assignment (LC-QAT page, Methodology 1 and 3: "rounding and clamping")
# --------------------------------------------------------------------------
def assign(Wp: np.ndarray):
    """Round the proxy weights to the nearest integer (ties to even) and clamp
    to ``[0, 3]``.  Returns ``(z uint8, mask bool)`` with ``mask`` the STE
    pass-through region ``0 <= W_p <= 3`` (false for NaN)."""
    w = np.asarray(Wp, dtype=np.float64)
    r = np.rint(w)
    r = np.where(np.isnan(w), 0.0, r)
    z = np.clip(r, 0.0, float(CODE_MAX)).astype(np.uint8)
    with np.errstate(invalid="ignore"):
        mask = (w >= 0.0) & (w <= float(CODE_MAX))
    return z, mask


# --------------------------------------------------------------------------
# 2-bit storage (format V1; the pages fix only "2 bits per weight")
# --------------------------------------------------------------------------
def pack_codes(z: np.ndarray) -> np.ndarray:
    """``[d_out][d_in]`` codes -> ``[d_out][d_in/4]`` bytes; element ``k`` of a
    row sits in byte ``k // 4`` at bits ``2 (k % 4)`` and ``2 (k % 4) + 1``."""
    z = np.asarray(z, dtype=np.uint8)
    n, k = z.shape
    assert k % 4 == 0
    out = np.zeros((n, k // 4), dtype=np.uint8)
    for pos in range(4):
        out |= (z[:, pos::4] & 3) << (2 * pos)
    return out


def unpack_codes(packed: np.ndarray, d_in: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    z = np.zeros((n, d_in), dtype=np.uint8)
    for pos in range(4):
        z[:, pos::4] = (packed >> (2 * pos)) & 3
    return z


def pack_mask(mask: np.ndarray) -> np.ndarray:
    """``[d_out][d_in]`` bools -> ``[d_out][d_in/8]`` bytes, bit ``k % 8`` of
    byte ``k // 8``."""
    m = np.asarray(mask, dtype=np.uint8)
    n, k = m.shape
    assert k % 8 == 0
    out = np.zeros((n, k // 8), dtype=np.uint8)
    for pos in range(8):
        out |= (m[:, pos::8] & 1) << pos
    return out


def unpack_mask(bits: np.ndarray, d_in: int) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint8)
    m = np.zeros((bits.shape[0], d_in), dtype=bool)
    for pos in range(8):
        m[:, pos::8] = (bits >> pos) & 1
    return m


# --------------------------------------------------------------------------
# decode (LC-QAT page, Methodology 1: c = A z + B; Methodology 3: A W_z + B)
# --------------------------------------------------------------------------
def decode(z: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """``W~[n, g d + i] = sum_j A[i, j] z[n, g d + j] + B[i]`` in fp64."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    d = A.shape[0]
    n, k = z.shape
    zg = np.asarray(z, dtype=np.float64).reshape(n, k // d, d)
    w = np.einsum("ij,ngj->ngi", A, zg) + B
    return w.reshape(n, k)


def decode_abs(z: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Normaliser of :func:`decode`: ``sum_j |A[i, j]| z_j + |B[i]|``."""
    return decode(z, np.abs(np.asarray(A, np.float64)), np.abs(np.asarray(B, np.float64)))


# --------------------------------------------------------------------------
# forward  Y = X W~  (decoupleQ page eq. (1) convention; LC-QAT Methodology 3)
# --------------------------------------------------------------------------
def forward(X: np.ndarray, z: np.ndarray, A: np.ndarray, B: np.ndarray):
    """Returns ``(Y, D_Y)`` with ``Y[m, n] = sum_k X[m, k] W~[n, k]`` and
    ``D_Y[m, n] = sum_k |X[m, k]| |W~[n, k]|``."""
    X = np.asarray(X, dtype=np.float64)
    W = decode(z, A, B)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def forward_sampled(X, z_rows: dict, A, B, pairs):
    """Y and D_Y at the listed ``(m, n)`` pairs only.  ``z_rows`` maps ``n`` to
    that row's codes (so a caller can unpack only the rows it samples)."""
    X = np.asarray(X, dtype=np.float64)
    y = np.empty(len(pairs))
    dd = np.empty(len(pairs))
    cache = {}
    for t, (m, n) in enumerate(pairs):
        if n not in cache:
            cache[n] = decode(np.asarray(z_rows[n]).reshape(1, -1), A, B)[0]
        w = cache[n]
        y[t] = float(np.dot(X[m], w))
        dd[t] = float(np.dot(np.abs(X[m]), np.abs(w)))
    return y, dd


def forward_algebraic(X, z, A, B):
    """The same product regrouped as ``X' Z^T + s 1^T`` with
    ``X'[m, g d + j] = sum_i X[m, g d + i] A[i, j]`` and
    ``s[m] = sum_g sum_i X[m, g d + i] B[i]``: exact algebra on
    ``sum_k x_k w~_k = sum_g x_g^T (A z_g + B)``.  Used only as an fp64
    cross-check of :func:`forward`."""
    X = np.asarray(X, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    d = A.shape[0]
    m, k = X.shape
    Xg = X.reshape(m, k // d, d)
    Xp = np.einsum("mgi,ij->mgj", Xg, A).reshape(m, k)
    s = np.einsum("mgi,i->m", Xg, B)
    return Xp @ np.asarray(z, np.float64).T + s[:, None]


# --------------------------------------------------------------------------
# straight-through backward (LC-QAT page, Methodology 1 "gradients flow
# through the linear map"; Methodology 3 and the gradient-estimation
# ablation: STE).  Loss gradient dY = dL/dY is an input.
# --------------------------------------------------------------------------
def backward(X, dY, z, mask, A, B):
    """Returns a dict with dX, dA, dB, dWp and their normalisers.

    * ``dX = dY W~``                                        (input gradient)
    * ``G[n, k] = sum_m dY[m, n] X[m, k]``                  (dL/dW~)
    * ``dA[i, j] = sum_{n, g} G[n, g d + i] z[n, g d + j]`` (chain rule on
      ``c = A z + B``)
    * ``dB[i] = sum_{n, g} G[n, g d + i]``
    * ``dWp[n, g d + j] = mask * sum_i A[i, j] G[n, g d + i]`` (STE: identity
      through the rounding, zero where the clamp is active)
    """
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    d = A.shape[0]
    n, k = z.shape
    W = decode(z, A, B)
    Wabs = np.abs(W)
    out = {}
    out["dX"] = dY @ W
    out["D_dX"] = np.abs(dY) @ Wabs
    G = dY.T @ X
    DG = np.abs(dY).T @ np.abs(X)
    Gg = G.reshape(n, k // d, d)
    DGg = DG.reshape(n, k // d, d)
    zg = np.asarray(z, np.float64).reshape(n, k // d, d)
    out["dA"] = np.einsum("ngi,ngj->ij", Gg, zg)
    out["D_dA"] = np.einsum("ngi,ngj->ij", DGg, zg)
    out["dB"] = Gg.sum(axis=(0, 1))
    out["D_dB"] = DGg.sum(axis=(0, 1))
    mg = np.asarray(mask, np.float64).reshape(n, k // d, d)
    out["dWp"] = (mg * np.einsum("ij,ngi->ngj", A, Gg)).reshape(n, k)
    out["D_dWp"] = (mg * np.einsum("ij,ngi->ngj", np.abs(A), DGg)).reshape(n, k)
    return out


def backward_dx_sampled(dY, z_cols_fn, A, B, pairs):
    """dX and D_dX at ``(m, k)`` pairs; ``z_cols_fn(k)`` returns the codes of
    column group ``k // d`` for all rows, shape ``[d_out, d]``."""
    dY = np.asarray(dY, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    d = A.shape[0]
    v = np.empty(len(pairs))
    dd = np.empty(len(pairs))
    for t, (m, kk) in enumerate(pairs):
        zc = np.asarray(z_cols_fn(kk), dtype=np.float64)  # [d_out, d]
        i = kk % d
        wcol = zc @ A[i] + B[i]                          # W~[:, kk]
        v[t] = float(np.dot(dY[m], wcol))
        dd[t] = float(np.dot(np.abs(dY[m]), np.abs(wcol)))
    return v, dd


def backward_dwp_sampled(X, dY, mask_rows_fn, A, pairs):
    """dWp and D_dWp at ``(n, k)`` pairs; ``mask_rows_fn(n)`` returns the clamp
    mask of row ``n``."""
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    d = A.shape[0]
    v = np.empty(len(pairs))
    dd = np.empty(len(pairs))
    for t, (n, kk) in enumerate(pairs):
        g0 = (kk // d) * d
        j = kk % d
        Gv = dY[:, n] @ X[:, g0:g0 + d]                  # G[n, g d + i], i < d
        DGv = np.abs(dY[:, n]) @ np.abs(X[:, g0:g0 + d])
        mk = float(mask_rows_fn(n)[kk])
        v[t] = mk * float(np.dot(A[:, j], Gv))
        dd[t] = mk * float(np.dot(np.abs(A[:, j]), DGv))
    return v, dd


# --------------------------------------------------------------------------
# DGE: a differentiable gradient estimator through the rounding (LC-QAT page,
# Methodology 3: the backward approximates the discretization by a smooth,
# differentiable curve instead of the straight-through estimator).  The pages
# give no formula; this is the reading taken here (parity of the curve itself
# is unpinned, only its limits are):
#   phi_k(w) = floor(w) + 1/2 + tanh(k (frac(w) - 1/2)) / (2 tanh(k/2))  on [0, 3]
# a staircase whose steps sit at the rounding points (frac = 1/2), equal to w
# at the integers, tending to rint(w) as k -> inf and to w (the STE) as k -> 0.
# Its derivative on [0, 3] is
#   phi_k'(w) = k / (2 tanh(k/2)) * sech^2(k (frac(w) - 1/2)),
# and 0 outside [0, 3] (the clamp), so that k -> 0 gives the STE mask exactly.
# --------------------------------------------------------------------------
def dge_phi(w, k):
    """The smooth rounding curve phi_k on [0, 3] (clamped outside)."""
    w = np.clip(np.asarray(w, dtype=np.float64), 0.0, 3.0)
    fl = np.minimum(np.floor(w), 2.0)        # w = 3 belongs to the last step
    f = w - fl
    return fl + 0.5 + np.tanh(k * (f - 0.5)) / (2.0 * np.tanh(k / 2.0))


def dge_derivative(Wp, k):
    """phi_k'(Wp): the factor DGE puts where the STE puts the clamp mask."""
    w = np.asarray(Wp, dtype=np.float64)
    inside = (w >= 0.0) & (w <= 3.0)
    fl = np.minimum(np.floor(np.where(inside, w, 0.0)), 2.0)
    f = np.where(inside, w, 0.0) - fl
    g = (k / (2.0 * np.tanh(k / 2.0))) / np.cosh(k * (f - 0.5)) ** 2
    return np.where(inside, g, 0.0)


def backward_dge_dwp(X, dY, z, Wp, A, k):
    """dWp under DGE: the STE gradient A^T G per vector, times phi_k'(Wp) instead
    of the clamp mask.  Returns (dWp, D) with D the normaliser of the STE dWp
    scaled by |phi_k'|."""
    ones = np.ones(z.shape, dtype=bool)
    bw = backward(X, dY, z, ones, A, np.zeros(A.shape[0]))
    s = dge_derivative(Wp, k)
    return bw["dWp"] * s, bw["D_dWp"] * np.abs(s)


# --------------------------------------------------------------------------
# least-squares refit of the float part given the codes (decoupleQ page,
# eq. (5): the layer objective tr{(W~ - W0)^T H (W~ - W0)}; section 3.3: with
# the integer part fixed the float part is an unconstrained quadratic, solved
# by setting the derivative to zero).  LC-VQ's float part is (A, B); H is
# taken as its diagonal h (one weight per input channel; h = 1 is the plain
# least-squares fit).
# --------------------------------------------------------------------------
PINV_RCOND = 1e-12  # eigenvalues below this fraction of the largest count as zero


def fit_affine_normal(W0: np.ndarray, z: np.ndarray, d: int, h=None):
    """The normal equations of the refit.  Output coordinate i of every vector
    (row n, group g) has input channel k = g d + i; with zt = [z_0 .. z_{d-1}, 1]
    (the vector's codes and a one for B):
        G[i] = sum_{n,g} h_k zt zt^T        ((d+1) x (d+1))
        R[i] = sum_{n,g} h_k W0[n, k] zt    (d+1)
    Returns (G [d][d+1][d+1], R [d][d+1])."""
    N, K = W0.shape
    ng = K // d
    zt = np.concatenate([z.reshape(N, ng, d).astype(np.float64), np.ones((N, ng, 1))], axis=2)
    w = np.asarray(W0, dtype=np.float64).reshape(N, ng, d)
    hv = (np.ones(K) if h is None else np.asarray(h, dtype=np.float64)).reshape(ng, d)
    G = np.einsum("gi,ngj,ngk->ijk", hv, zt, zt)
    R = np.einsum("gi,ngi,ngj->ij", hv, w, zt)
    return G, R


def fit_affine(W0: np.ndarray, z: np.ndarray, d: int, h=None):
    """(A, B) minimizing sum_n sum_k h_k (W0[n, k] - W~[n, k])^2 over W~ = A z + B
    per vector.  The objective splits over the output coordinate i, and row i
    of [A | B] is theta_i = G[i]^+ R[i]: the solution of the normal equations,
    the minimum-norm one when G[i] is singular (a code position that never
    varies, or weights h that vanish)."""
    G, R = fit_affine_normal(W0, z, d, h)
    A = np.zeros((d, d))
    B = np.zeros(d)
    for i in range(d):
        th = np.linalg.pinv(G[i], rcond=PINV_RCOND, hermitian=True) @ R[i]
        A[i] = th[:d]
        B[i] = th[d]
    return A, B


def fit_affine_h_normal(W0: np.ndarray, z: np.ndarray, d: int, H: np.ndarray):
    """The normal equations of the refit under the full input Hessian H
    (decoupleQ page, eq. (5): the objective tr{(W~ - W0)^T H (W~ - W0)} with
    W~ = d_in x d_out; in this storage order it is sum_n r_n^T H r_n over the
    rows r_n = W~[n] - W0[n]).  With zt = [z_0 .. z_{d-1}, 1] per vector, the
    decoded element is W~[n, g d + i] = sum_a theta[i, a] zt[n, g, a] with
    theta = [A | B], so the objective is a quadratic in theta whose normal
    equations couple every pair of vector positions (g, g'):
        G[(i, a), (j, b)] = sum_n sum_{g, g'} H[g d + i, g' d + j] zt[n, g, a] zt[n, g', b]
        R[(i, a)]         = sum_n sum_g sum_k H[g d + i, k] W0[n, k] zt[n, g, a]
    Returns (G [d (d+1)][d (d+1)], R [d (d+1)]), index (i, a) -> i (d+1) + a."""
    W0 = np.asarray(W0, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    N, K = W0.shape
    ng = K // d
    zt = np.concatenate([np.asarray(z, np.float64).reshape(N, ng, d), np.ones((N, ng, 1))], axis=2)
    # (optimize=True lets numpy contract these sums through BLAS)
    S = np.einsum("nga,nhb->gahb", zt, zt, optimize=True)   # code Gram of every (g, g') pair
    Hg = H.reshape(ng, d, ng, d)                            # H[g d + i, h d + j] -> [g, i, h, j]
    G = np.einsum("gihj,gahb->iajb", Hg, S, optimize=True).reshape(d * (d + 1), d * (d + 1))
    T = np.einsum("nk,nga->kga", W0, zt, optimize=True)     # W0^T zt per position
    R = np.einsum("gik,kga->ia", H.reshape(ng, d, K), T, optimize=True).reshape(d * (d + 1))
    return G, R


def fit_affine_h(W0: np.ndarray, z: np.ndarray, d: int, H: np.ndarray):
    """(A, B) minimizing sum_n (W~[n] - W0[n])^T H (W~[n] - W0[n]) over W~ = A z + B
    per vector (decoupleQ page, eq. (5) with the codes fixed, solved in closed
    form as in its section 3.3): theta = G^+ R from fit_affine_h_normal, the
    minimum-norm solution when G is singular."""
    G, R = fit_affine_h_normal(W0, z, d, H)
    th = np.linalg.pinv(G, rcond=PINV_RCOND, hermitian=True) @ R
    th = th.reshape(d, d + 1)
    return th[:, :d].copy(), th[:, d].copy()


def fit_objective_h(W0, z, A, B, H) -> float:
    """sum_n (W~[n] - W0[n])^T H (W~[n] - W0[n]), the quantity fit_affine_h minimizes."""
    r = decode(z, A, B) - np.asarray(W0, dtype=np.float64)
    return float(np.einsum("nk,kl,nl->", r, np.asarray(H, dtype=np.float64), r))


def fit_objective(W0, z, A, B, h=None) -> float:
    """sum_n sum_k h_k (W0[n, k] - (A z + B)[n, k])^2, the quantity fit_affine minimizes."""
    r = np.asarray(W0, dtype=np.float64) - decode(z, A, B)
    hh = np.ones(r.shape[1]) if h is None else np.asarray(h, dtype=np.float64)
    return float(np.sum(hh[None, :] * r * r))


# --------------------------------------------------------------------------
# H-aware sequential code assignment: the PTQ initialisation of the codes
# (LC-QAT page, Methodology 2: the initial integer weights come from LDLQ,
# which quantizes column by column and compensates the reconstruction error
# of the columns already fixed; decoupleQ page, section 3.3, eq. (8)-(11):
# round and clip one element, then re-solve the remaining elements of the
# quadratic objective (7) with the integer constraint and the box dropped,
# the second approximation, eq. (11)).
#
# In LC-VQ terms the integer part of one weight row is its code vector z and
# the decoded row is Abar z + bbar (Abar = blockdiag(A, .., A), bbar = B
# repeated per vector), so objective (7) of a row with target w0 is
#     g(z) = 1/2 (Abar z + bbar - w0)^T H (Abar z + bbar - w0)
#          = 1/2 (z - p)^T Q (z - p),   Q = Abar^T H Abar,  p = Abar^-1 (w0 - bbar),
# p being the row's continuous code-space target (what the proxy weight W_p
# holds).  With Q factored as (I + U) diag(D) (I + U)^T, U strictly upper
# triangular,
#     g(z) = 1/2 sum_k D_k ((z_k - p_k) + sum_{i<k} U[i, k] (z_i - p_i))^2,
# so once z_0 .. z_{j-1} are fixed the minimiser of eq. (11) over the rest
# zeroes every bracket k >= j, and its j-th element is
#     t_j = p_j + sum_{i<j} U[i, j] (p_i - z_i).
# Element j then takes z_j = clamp(rint(t_j), 0, 3), the rounding and clamping
# of the assignment step (with Q diagonal, U = 0 and this is that step).
# --------------------------------------------------------------------------
def code_space_hessian(H: np.ndarray, A: np.ndarray) -> np.ndarray:
    """Q = Abar^T H Abar for a K x K input Hessian H and the d x d matrix A:
    Q[g d + a, h d + b] = sum_{i,j} A[i, a] H[g d + i, h d + j] A[j, b]."""
    H = np.asarray(H, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    K = H.shape[0]
    d = A.shape[0]
    Abar = np.kron(np.eye(K // d), A)
    return Abar.T @ H @ Abar


def code_targets(W0: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """p = Abar^-1 (w0 - bbar) per row: each length-d vector solved against A."""
    W0 = np.asarray(W0, dtype=np.float64)
    N, K = W0.shape
    d = A.shape[0]
    r = (W0.reshape(N, K // d, d) - np.asarray(B, dtype=np.float64)[None, None, :])
    sol = np.linalg.solve(np.asarray(A, dtype=np.float64), r.reshape(-1, d).T).T
    return sol.reshape(N, K)


def ldl_upper(Q: np.ndarray):
    """Q = (I + U) diag(D) (I + U)^T with U strictly upper triangular.  This is
    the Cholesky factorisation of Q with rows and columns reversed: if
    J Q J = C C^T (C lower), then V = J C J is upper triangular with
    Q = V V^T, and U = V diag(1 / diag V) - I, D = diag(V)^2.
    Returns (U, D)."""
    Q = np.asarray(Q, dtype=np.float64)
    C = np.linalg.cholesky(Q[::-1, ::-1])
    V = C[::-1, ::-1]
    v = np.diag(V).copy()
    U = V / v[None, :] - np.eye(Q.shape[0])
    return np.triu(U, 1), v * v


def ldlq_assign(P: np.ndarray, U: np.ndarray) -> np.ndarray:
    """Codes Z (u8, N x K) of the sequential rule above, every row of the
    targets P (N x K) on its own, elements in increasing k.  Only the strictly
    upper triangle of U (K x K) is used."""
    P = np.asarray(P, dtype=np.float64)
    Ut = np.triu(np.asarray(U, dtype=np.float64), 1)
    N, K = P.shape
    Z = np.zeros((N, K), dtype=np.uint8)
    E = np.zeros((N, K))  # p_i - z_i of the elements already fixed
    for j in range(K):
        t = P[:, j] + E[:, :j] @ Ut[:j, j]
        z = np.clip(np.rint(t), 0, CODE_MAX)
        Z[:, j] = z.astype(np.uint8)
        E[:, j] = P[:, j] - z
    return Z


def ldlq_targets(P: np.ndarray, U: np.ndarray, Z: np.ndarray):
    """The targets t_j that the rule rounds, given the codes Z that were chosen
    (each t_j depends only on the codes before it), and the per-element sum of
    the absolute values of its terms, |p_j| + sum_{i<j} |U[i, j] (p_i - z_i)|.
    A code z_j is the rule's choice when it equals clamp(rint(t_j), 0, 3).
    Returns (T, S)."""
    P = np.asarray(P, dtype=np.float64)
    Ut = np.triu(np.asarray(U, dtype=np.float64), 1)
    E = P - np.asarray(Z, dtype=np.float64)
    return P + E @ Ut, np.abs(P) + np.abs(E) @ np.abs(Ut)


def ldlq_objective(P: np.ndarray, Q: np.ndarray, Z: np.ndarray) -> np.ndarray:
    """g(z) = 1/2 (z - p)^T Q (z - p) for every row; returns a length-N array."""
    R = np.asarray(Z, dtype=np.float64) - np.asarray(P, dtype=np.float64)
    return 0.5 * np.einsum("nk,kl,nl->n", R, np.asarray(Q, dtype=np.float64), R)


# --------------------------------------------------------------------------
# parity metric
# --------------------------------------------------------------------------
def rel_err(got, ref, D) -> float:
    """max over elements of ``|got - ref| / D``; where ``D == 0`` the element
    must be exactly equal (returns inf otherwise)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    diff = np.abs(got - ref)
    if not np.all(np.isfinite(got)):
        return float("inf")
    zero = D == 0
    if np.any(diff[zero] != 0):
        return float("inf")
    if np.all(zero):
        return 0.0
    return float(np.max(diff[~zero] / D[~zero]))

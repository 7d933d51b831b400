"""Pins for oracle.soap and oracle.qr: the one-SVD identity, exact
eigenbases, AdamW as the identity-basis special case, power-iteration
convergence and textbook QR properties."""
import numpy as np
import pytest

from oracle import qr as oqr
from oracle import soap


def _eig_desc(S):
    w, Q = np.linalg.eigh(S)
    return Q[:, ::-1]


# ---------------------------------------------------------------- QR

def _gram_schmidt(Y):
    # brute-force classical Gram-Schmidt in pure Python loops (tiny inputs)
    m, n = len(Y), len(Y[0])
    Q = [[0.0] * n for _ in range(m)]
    R = [[0.0] * n for _ in range(n)]
    for j in range(n):
        v = [Y[i][j] for i in range(m)]
        for k in range(j):
            R[k][j] = sum(Q[i][k] * Y[i][j] for i in range(m))
            v = [v[i] - R[k][j] * Q[i][k] for i in range(m)]
        R[j][j] = sum(x * x for x in v) ** 0.5
        for i in range(m):
            Q[i][j] = v[i] / R[j][j]
    return np.array(Q), np.array(R)


@pytest.mark.parametrize("shape", [(5, 5), (7, 4), (6, 6)])
def test_qr_positive_matches_gram_schmidt(shape):
    rng = np.random.default_rng(21)
    Y = rng.standard_normal(shape)
    Q, R = oqr.qr_positive(Y)
    Qg, Rg = _gram_schmidt(Y.tolist())
    np.testing.assert_allclose(Q, Qg, atol=1e-12)
    np.testing.assert_allclose(R, Rg, atol=1e-12)


def test_qr_properties():
    rng = np.random.default_rng(22)
    Y = rng.standard_normal((64, 64)) @ np.diag(np.geomspace(1, 1e-3, 64))
    Q, R = oqr.qr_positive(Y)
    u = np.finfo(np.float64).eps
    assert np.abs(Q.T @ Q - np.eye(64)).max() <= 50 * 64 * u
    assert np.allclose(np.tril(R, -1), 0) and (np.diag(R) > 0).all()
    assert np.linalg.norm(Q @ R - Y) / np.linalg.norm(Y) <= 1e-12


# ---------------------------------------------------------------- exact basis

@pytest.mark.parametrize("shape", [(8, 8), (6, 11), (11, 6)])
def test_one_svd_identity(shape):
    """Exact eigenbases, EMAs off, no bias correction, eps tiny: the SOAP
    step is -lr U V^T ('Reading notes on SOAP, Muon, and Beyond', section 2)."""
    m, n = shape
    k = min(m, n)
    rng = np.random.default_rng(23)
    # well separated singular values, so eigh's basis is accurate to ~1e-15
    Uo, _ = np.linalg.qr(rng.standard_normal((m, k)))
    Vo, _ = np.linalg.qr(rng.standard_normal((n, k)))
    G = (Uo * np.geomspace(2.0, 0.5, k)) @ Vo.T
    QL, QR = _eig_desc(G @ G.T), _eig_desc(G.T @ G)
    U, _, Vt = np.linalg.svd(G, full_matrices=False)
    out = soap.soap_step(np.zeros((m, n)), G, np.zeros((m, n)), np.zeros((m, n)),
                         None, QL, None, QR, t=1, lr=0.5, beta1=0.0, beta2=0.0,
                         eps=1e-8, bias_correction=False, refresh=False)
    # off-diagonal round-off (~1e-15) / eps and eps / sigma_min both <~ 1e-7
    np.testing.assert_allclose(out["dW"], -0.5 * (U @ Vt), atol=1e-6)


@pytest.mark.parametrize("shape", [(9, 9), (5, 12)])
def test_exact_eigenbasis_diagonalises(shape):
    m, n = shape
    rng = np.random.default_rng(24)
    G = rng.standard_normal((m, n))
    QL, QR = _eig_desc(G @ G.T), _eig_desc(G.T @ G)
    out = soap.soap_step(np.zeros((m, n)), G, np.zeros((m, n)), np.zeros((m, n)),
                         None, QL, None, QR, refresh=False)
    Gr = np.abs(out["Gr"])
    # one entry per row survives (the singular value), the rest are round-off
    big = Gr > 1e-10 * np.linalg.norm(G)
    assert big.sum() == min(m, n)
    assert (big.sum(axis=1) <= 1).all() and (big.sum(axis=0) <= 1).all()
    np.testing.assert_allclose(np.sort(Gr[big]), np.sort(np.linalg.svd(G, compute_uv=False)), rtol=1e-10)


def test_rotation_preserves_frobenius_norm():
    rng = np.random.default_rng(25)
    G = rng.standard_normal((10, 14))
    QL, _ = np.linalg.qr(rng.standard_normal((10, 10)))
    QR, _ = np.linalg.qr(rng.standard_normal((14, 14)))
    out = soap.soap_step(np.zeros_like(G), G, np.zeros_like(G), np.zeros_like(G),
                         None, QL, None, QR, refresh=False)
    assert np.linalg.norm(out["Gr"]) == pytest.approx(np.linalg.norm(G), rel=1e-13)


# ---------------------------------------------------------------- AdamW case

def test_identity_bases_is_adamw():
    """With both bases identity the step is AdamW (LLM Optimizers guide,
    sections 5-6 recurrences, written out here per coordinate)."""
    rng = np.random.default_rng(26)
    m, n = 5, 7
    b1, b2, eps, lr, wd = 0.9, 0.99, 1e-8, 1e-2, 0.1
    W = rng.standard_normal((m, n))
    Wr = W.tolist()
    mom = [[0.0] * n for _ in range(m)]
    sec = [[0.0] * n for _ in range(m)]
    M = np.zeros((m, n))
    V = np.zeros((m, n))
    for t in range(1, 5):
        G = rng.standard_normal((m, n))
        out = soap.soap_step(W, G, M, V, t=t, lr=lr, beta1=b1, beta2=b2, eps=eps,
                             weight_decay=wd)
        W, M, V = out["W"], out["M"], out["V"]
        for i in range(m):
            for j in range(n):
                g = G[i, j]
                mom[i][j] = b1 * mom[i][j] + (1 - b1) * g
                sec[i][j] = b2 * sec[i][j] + (1 - b2) * g * g
                mh = mom[i][j] / (1 - b1 ** t)
                vh = sec[i][j] / (1 - b2 ** t)
                Wr[i][j] = (1 - lr * wd) * Wr[i][j] - lr * mh / (vh ** 0.5 + eps)
        np.testing.assert_allclose(W, np.array(Wr), atol=1e-13)


def test_constant_gradient_adam_step():
    g = np.array([[2.0, -3.0, 1e-9]])
    W = np.zeros_like(g)
    M = np.zeros_like(g)
    V = np.zeros_like(g)
    for t in range(1, 4):
        out = soap.soap_step(W, g, M, V, t=t, lr=1.0, beta1=0.95, beta2=0.95, eps=1e-8)
        np.testing.assert_allclose(out["Dbar"], g / (np.abs(g) + 1e-8), rtol=1e-12)
        W, M, V = out["W"], out["M"], out["V"]


# ---------------------------------------------------------------- refresh

def test_first_step_from_zero_state():
    """L_1 = (1-b) G G^T includes the current gradient; Q = qr(L_1 I)."""
    rng = np.random.default_rng(27)
    m, n = 6, 9
    G = rng.standard_normal((m, n))
    out = soap.soap_step(np.zeros((m, n)), G, np.zeros((m, n)), np.zeros((m, n)),
                         np.zeros((m, m)), np.eye(m), np.zeros((n, n)), np.eye(n),
                         beta2=0.9)
    np.testing.assert_allclose(out["L"], 0.1 * G @ G.T, atol=1e-14)
    np.testing.assert_allclose(out["R"], 0.1 * G.T @ G, atol=1e-14)
    # Q_L's columns are the Gram-Schmidt orthonormalisation of L_1's columns
    # (L_1 Q_0 = L_1), in a Python loop
    Qg, _ = _gram_schmidt(out["L"].tolist())
    np.testing.assert_allclose(out["QL"], Qg, atol=1e-9)
    np.testing.assert_allclose(out["QL"].T @ out["QL"], np.eye(m), atol=1e-12)
    # the damped option: the Gram-Schmidt basis of L_1 + d I, d = 1e-5 trace(L_1)
    out1 = soap.soap_step(np.zeros((m, n)), G, np.zeros((m, n)), np.zeros((m, n)),
                          np.zeros((m, m)), np.eye(m), None, None, beta2=0.9, damping=1e-5)
    L1 = out1["L"].tolist()
    d = 1e-5 * sum(L1[i][i] for i in range(m))
    Qg1, _ = _gram_schmidt([[L1[i][j] + (d if i == j else 0.0) for j in range(m)] for i in range(m)])
    np.testing.assert_allclose(out1["QL"], Qg1, atol=1e-9)


def test_power_step_worked_example():
    """2 x 2 by hand: L = diag(3, 1), old basis the rotation with cos 0.6 and
    sin 0.8.  L Q_old has columns (3 * 0.6, 1 * 0.8) = (1.8, 0.8) and
    (3 * -0.8, 1 * 0.6) = (-2.4, 0.6); the new basis is the first column
    normalised, (1.8, 0.8) / sqrt(3.88), and the orthogonal unit vector
    (-0.8, 1.8) / sqrt(3.88), whose product with the second column,
    (1.92 + 1.08) / sqrt(3.88), is positive (diag(R) > 0).  The state is
    chosen so that the EMA leaves L = diag(3, 1): beta2 = 0.5, G = 0,
    L_prev = diag(6, 2)."""
    L_prev = np.diag([6.0, 2.0])
    Q_old = np.array([[0.6, -0.8], [0.8, 0.6]])
    Z = np.zeros((2, 2))
    out = soap.soap_step(Z, Z, Z, Z, L_prev, Q_old, t=1, beta2=0.5)
    np.testing.assert_allclose(out["L"], np.diag([3.0, 1.0]), atol=0)
    r = 3.88 ** 0.5
    expect = np.array([[1.8, -0.8], [0.8, 1.8]]) / r
    np.testing.assert_allclose(out["QL"], expect, rtol=0, atol=1e-14)
    # the damped option (trace 4, d = 4e-5): (L + d I) Q_old has first column
    # (3.00004 * 0.6, 1.00004 * 0.8) = (1.800024, 0.800032)
    out1 = soap.soap_step(Z, Z, Z, Z, L_prev, Q_old, t=1, beta2=0.5, damping=1e-5)
    r1 = (1.800024 ** 2 + 0.800032 ** 2) ** 0.5
    q1 = np.array([1.800024, 0.800032]) / r1
    np.testing.assert_allclose(out1["QL"], np.array([[q1[0], -q1[1]], [q1[1], q1[0]]]), rtol=0, atol=1e-13)
    # the two differ at the 1e-5 level, far above the tolerances
    assert abs(out1["QL"][0, 0] - out["QL"][0, 0]) > 1e-7


def test_power_step_keeps_an_exact_eigenbasis_and_resets_a_zero_factor():
    rng = np.random.default_rng(31)
    m = 7
    U, _ = np.linalg.qr(rng.standard_normal((m, m)))
    lam = np.array([9.0, 5.0, 3.0, 2.0, 1.0, 0.5, 0.1])
    L = (U * lam) @ U.T
    Z = np.zeros((m, 3))
    # shampoo_beta = 1: the factor is L itself; L U = U diag(lam) with lam > 0,
    # so the positive-diagonal QR returns U exactly (R = diag(lam))
    out = soap.soap_step(Z, Z, Z, Z, L, U, None, None, shampoo_beta=1.0)
    np.testing.assert_allclose(out["QL"], U, atol=1e-12)
    # a factor that has seen only zero gradients: L Q = 0, whose Householder
    # QR has only trivial reflectors, Q = I (R = 0, no column sign to fix)
    out = soap.soap_step(Z, Z, Z, Z, np.zeros((m, m)), U, None, None)
    np.testing.assert_array_equal(out["QL"], np.eye(m))
    # the damped option keeps the basis there instead: d = 1, qr(U) = U
    out = soap.soap_step(Z, Z, Z, Z, np.zeros((m, m)), U, None, None, damping=1e-5)
    np.testing.assert_allclose(out["QL"], U, atol=1e-12)


def test_power_iteration_converges_to_eigenbasis():
    """Repeated steps with one fixed gradient: L -> G G^T and Q_L^T L Q_L
    becomes diagonal (textbook subspace iteration)."""
    rng = np.random.default_rng(28)
    m, n = 6, 10
    U, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, m)))
    G = (U * np.array([4.0, 2.5, 1.6, 1.0, 0.6, 0.3])) @ V.T
    state = dict(W=np.zeros((m, n)), M=np.zeros((m, n)), V=np.zeros((m, n)),
                 L=np.zeros((m, m)), QL=np.eye(m))
    for t in range(1, 80):
        out = soap.soap_step(state["W"], G, state["M"], state["V"], state["L"], state["QL"],
                             t=t, beta2=0.5)
        state.update(W=out["W"], M=out["M"], V=out["V"], L=out["L"], QL=out["QL"])
    D = state["QL"].T @ state["L"] @ state["QL"]
    off = D - np.diag(np.diag(D))
    assert np.abs(off).max() < 1e-8 * np.abs(D).max()
    np.testing.assert_allclose(np.diag(D), np.array([4.0, 2.5, 1.6, 1.0, 0.6, 0.3]) ** 2, rtol=1e-8)


def test_diagonal_gradient_stays_elementwise():
    # G diagonal with distinct entries: bases stay the identity and the step
    # is Adam on the diagonal entries
    g = np.array([3.0, -1.0, 0.5])
    G = np.diag(g)
    out = soap.soap_step(np.zeros((3, 3)), G, np.zeros((3, 3)), np.zeros((3, 3)),
                         np.zeros((3, 3)), np.eye(3), np.zeros((3, 3)), np.eye(3),
                         t=1, lr=1.0, eps=1e-8)
    np.testing.assert_allclose(np.abs(out["QL"]), np.eye(3), atol=1e-14)
    np.testing.assert_allclose(out["D"], np.diag(g / (np.abs(g) + 1e-8)), atol=1e-14)


def test_bf16_mode_without_rounding_is_fp64(monkeypatch):
    rng = np.random.default_rng(29)
    m, n = 6, 9
    args = (rng.standard_normal((m, n)), rng.standard_normal((m, n)),
            rng.standard_normal((m, n)), np.abs(rng.standard_normal((m, n))))
    L = np.eye(m) * 0.3
    Rf = np.eye(n) * 0.2
    QL, _ = np.linalg.qr(rng.standard_normal((m, m)))
    QR, _ = np.linalg.qr(rng.standard_normal((n, n)))
    monkeypatch.setattr(soap, "rnd", lambda x: np.asarray(x, dtype=np.float64))
    for sides in ((L, QL, Rf, QR), (L, QL, None, None), (None, None, Rf, QR)):
        a = soap.soap_step(*args, *sides, t=3, precision="fp64")
        b = soap.soap_step(*args, *sides, t=3, precision="bf16")
        np.testing.assert_allclose(a["W"], b["W"], atol=1e-12)


def test_stale_basis_keeps_q_and_updates_factors():
    """Between refreshes the factors keep accumulating and the basis stays."""
    rng = np.random.default_rng(30)
    m, n = 5, 8
    G = rng.standard_normal((m, n))
    QL, _ = np.linalg.qr(rng.standard_normal((m, m)))
    L0 = np.eye(m)
    out = soap.soap_step(np.zeros((m, n)), G, np.zeros((m, n)), np.zeros((m, n)), L0, QL,
                         beta2=0.9, basis_refresh=False)
    np.testing.assert_array_equal(out["QL"], QL)
    np.testing.assert_allclose(out["L"], 0.9 * L0 + 0.1 * G @ G.T, atol=1e-14)
    np.testing.assert_allclose(out["Gr"], QL.T @ G, atol=1e-14)

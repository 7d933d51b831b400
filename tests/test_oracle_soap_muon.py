"""Pins for oracle.soap_muon: closed forms on Hadamard and known-SVD
gradients (the Newton-Schulz output of a matrix with one repeated singular
value is the scalar map applied to it), the previous-basis rule, the basis
refresh for the next step, and the bf16 mode without rounding."""
import numpy as np

from oracle import ns as ons
from oracle import soap_muon as osm


def _hadamard(n):
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


LR, WD = 0.02, 0.01


def test_identity_bases_sign_gradient_closed_form():
    """mu = 0, b2 = 0, identity bases, G = H_16 (entries +-1): P = G / (1 + eps),
    whose singular values are all 4 = sqrt(16); NS normalises by ||P||_F = 16,
    so every singular value enters the map at 1/4 and O = (H/4) phi^5(1/4)."""
    n = 16
    H = _hadamard(n)
    Z = np.zeros((n, n))
    W0 = np.full((n, n), 0.5)
    out = osm.soap_muon_step(W0, H, Z, Z, t=1, momentum=0.0, beta2=0.0, lr=LR, weight_decay=WD)
    np.testing.assert_allclose(out["P"], H / (1 + 1e-8), rtol=1e-15)
    # the map's argument with both epsilons: sigma(P) / (||P||_F + 1e-7)
    sv = 4 / (1 + 1e-8)
    t0 = sv / (4 * sv + 1e-7)
    phi = float(ons.scalar_map(np.array([t0]))[0])
    np.testing.assert_allclose(out["O"], H / 4 * phi, rtol=0, atol=1e-13)
    s = 0.2 * np.sqrt(16)
    np.testing.assert_allclose(out["W"], (1 - LR * WD) * W0 - LR * s * H / 4 * phi, atol=1e-13)


def test_previous_basis_is_used_and_refreshed_for_next_step():
    """Q_L = U (orthogonal), G = U H: with mu = 0, b2 = 0 the rotated
    momentum is H, its Adam normalisation sign(H) = H, so P = U H and
    O = U (H/4) phi^5(1/4) (NS commutes with an orthogonal left factor).
    A refreshed basis would rotate G differently.  The returned basis is
    the power step of the updated factor, qr(L U): Q^T L U is upper
    triangular with a positive diagonal."""
    n = 16
    rng = np.random.default_rng(41)
    U, _ = np.linalg.qr(rng.standard_normal((n, n)))
    H = _hadamard(n)
    G = U @ H
    Z = np.zeros((n, n))
    L0 = np.diag(np.linspace(1.0, 2.0, n))
    out = osm.soap_muon_step(Z, G, Z, Z, L0, U, t=1, momentum=0.0, beta2=0.0, lr=1.0, weight_decay=0.0)
    phi = float(ons.scalar_map(np.array([0.25]))[0])
    np.testing.assert_allclose(out["P"], U @ H, atol=1e-12)
    np.testing.assert_allclose(out["O"], U @ H / 4 * phi, atol=1e-9)
    np.testing.assert_allclose(out["L"], 0.9 * L0 + 0.1 * G @ G.T, atol=1e-12)
    Q = out["QL"]
    np.testing.assert_allclose(Q.T @ Q, np.eye(n), atol=1e-12)
    T = Q.T @ out["L"] @ U
    assert np.abs(np.tril(T, -1)).max() <= 1e-12 * np.abs(T).max()
    assert (np.diag(T) > 0).all()
    assert np.abs(Q - U).max() > 1e-2            # the basis did move


def test_exact_eigenbasis_gives_the_polar_factor():
    """G = U diag(s) V^T (square, full rank) with Q_L = U, Q_R = V: the rotated
    gradient and momentum are diag(s), Adam maps it to the identity, P = U V^T
    (the polar factor), and O = phi^5(1/sqrt(n)) U V^T."""
    n = 12
    rng = np.random.default_rng(42)
    U, _ = np.linalg.qr(rng.standard_normal((n, n)))
    Vb, _ = np.linalg.qr(rng.standard_normal((n, n)))
    s = np.linspace(3.0, 0.5, n)
    G = (U * s) @ Vb.T
    Z = np.zeros((n, n))
    out = osm.soap_muon_step(Z, G, Z, Z, Z, U, Z, Vb, t=1, momentum=0.0, beta2=0.0,
                             lr=1.0, weight_decay=0.0)
    # off the diagonal the rotated gradient is fp64 round-off (~1e-16), which
    # Adam divides by itself + eps = 1e-8: entries of P off by ~1e-8 each
    # (the one-SVD identity holds only while round-off << eps)
    np.testing.assert_allclose(out["P"], U @ Vb.T, atol=1e-6)
    phi = float(ons.scalar_map(np.array([1 / np.sqrt(n)]))[0])
    np.testing.assert_allclose(out["O"], phi * U @ Vb.T, atol=1e-6)


def test_momentum_and_second_moment_recurrences():
    """Identity bases: B and V follow their recurrences elementwise; with
    Nesterov off the preconditioned matrix is B / (sqrt(V / bc2) + eps)."""
    rng = np.random.default_rng(43)
    m, n = 5, 7
    G = rng.standard_normal((m, n))
    B0 = rng.standard_normal((m, n))
    V0 = rng.random((m, n))
    out = osm.soap_muon_step(np.zeros((m, n)), G, B0, V0, t=3, momentum=0.9, nesterov=False,
                             beta2=0.95)
    np.testing.assert_allclose(out["B"], 0.9 * B0 + G, rtol=1e-15)
    np.testing.assert_allclose(out["V"], 0.95 * V0 + 0.05 * G * G, rtol=1e-15)
    bc2 = 1 - 0.95 ** 3
    np.testing.assert_allclose(out["P"], out["B"] / (np.sqrt(out["V"] / bc2) + 1e-8), rtol=1e-14)
    nest = osm.soap_muon_step(np.zeros((m, n)), G, B0, V0, t=3, momentum=0.9, beta2=0.95)
    np.testing.assert_allclose(nest["N"], G + 0.9 * (0.9 * B0 + G), rtol=1e-15)


def test_bf16_mode_without_rounding_is_fp64(monkeypatch):
    rng = np.random.default_rng(44)
    m, n = 6, 10
    G = rng.standard_normal((m, n))
    B0 = rng.standard_normal((m, n))
    V0 = rng.random((m, n))
    QL, _ = np.linalg.qr(rng.standard_normal((m, m)))
    QR, _ = np.linalg.qr(rng.standard_normal((n, n)))
    ident = lambda x: np.asarray(x, dtype=np.float64)
    monkeypatch.setattr(osm, "rnd", ident)
    monkeypatch.setattr(osm, "rnd32", ident)
    monkeypatch.setattr(osm, "newton_schulz_bf16", osm.newton_schulz)
    args = (np.zeros((m, n)), G, B0, V0, np.eye(m), QL, np.eye(n), QR)
    a = osm.soap_muon_step(*args, t=2, precision="fp64")
    b = osm.soap_muon_step(*args, t=2, precision="bf16")
    for k in ("W", "QL", "QR", "P"):
        np.testing.assert_allclose(a[k], b[k], atol=1e-12)

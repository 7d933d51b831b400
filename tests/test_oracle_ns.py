"""Pins for oracle.ns: the pages' printed values, Lemma 3's closed form and
special cases with known polar factors."""
import numpy as np
import pytest

import workloads as wl
from oracle import ns


def _sv(X):
    return np.sort(np.linalg.svd(X, compute_uv=False))[::-1]


def _closed_form(U, s, V, coeffs=ns.QUINTIC, steps=5, eps=1e-7):
    # Lemma 3: the iteration maps each singular value of the normalised input
    # through phi; singular vectors are unchanged.
    t = np.asarray(s, dtype=np.float64) / (np.linalg.norm(s) + eps)
    return (U * ns.scalar_map(t, coeffs, steps)[None, :]) @ V.T


# ---------------------------------------------------------------- worked 2x2

def test_worked_example_setup(golden):
    g = golden("worked_example_2x2.json")
    G = np.array(g["G"])
    U, s, Vt = np.linalg.svd(G)
    np.testing.assert_allclose(np.round(s, 4), g["singular_values_4dp"])
    np.testing.assert_allclose(np.sqrt(5) * (U @ Vt), g["sqrt5_times_polar"], atol=1e-12)
    np.testing.assert_allclose(np.round(s / np.linalg.norm(G), 3), g["normalised_singular_values_3dp"])


def test_worked_example_quintic_trajectory(golden):
    g = golden("worked_example_2x2.json")
    G = np.array(g["G"])
    for k, pair in enumerate(g["quintic_trajectory_3dp"], start=1):
        X = ns.newton_schulz(G, ns.QUINTIC, k, eps=0.0)
        np.testing.assert_allclose(np.round(_sv(X), 3), sorted(pair, reverse=True), atol=1e-12)
    X5 = ns.newton_schulz(G, ns.QUINTIC, 5, eps=0.0)
    np.testing.assert_allclose(np.round(_sv(X5), 3), g["quintic_5_steps_printed_sv_3dp"])


def test_worked_example_cubic(golden):
    g = golden("worked_example_2x2.json")
    G = np.array(g["G"])
    U, _, Vt = np.linalg.svd(G)
    polar = U @ Vt
    X1 = ns.newton_schulz(G, ns.CUBIC, 1, eps=0.0)
    np.testing.assert_allclose(np.round(_sv(X1), 3), sorted(g["cubic_first_step_3dp"], reverse=True))
    for k, pair in enumerate(g["cubic_later_steps_3dp"], start=2):
        Xk = ns.newton_schulz(G, ns.CUBIC, k, eps=0.0)
        np.testing.assert_allclose(np.round(_sv(Xk), 3), sorted(pair, reverse=True))
    e6 = np.abs(ns.newton_schulz(G, ns.CUBIC, 6, eps=0.0) - polar).max()
    e7 = np.abs(ns.newton_schulz(G, ns.CUBIC, 7, eps=0.0) - polar).max()
    assert 0.2 * g["cubic_max_error_after_6"] < e6 < 2 * g["cubic_max_error_after_6"]
    assert e7 < 2 * g["cubic_max_error_after_7"]


def test_worked_example_polar_maximises_inner_product(golden):
    """The lesson's duality check: among unit-spectral-norm directions the
    polar factor maximises <G, O>, reaching the nuclear norm; G / sigma_max
    and sign(G) / ||sign(G)||_2 fall short by the printed amounts.  The
    polar factor is the oracle's cubic iteration run to convergence."""
    g = golden("worked_example_2x2.json")
    G = np.array(g["G"])
    ip = g["inner_products_4dp"]
    polar = ns.newton_schulz(G, ns.CUBIC, 40, eps=0.0)
    nuclear = np.linalg.svd(G, compute_uv=False).sum()
    S = np.sign(G)
    got = {"polar": np.sum(G * polar),
           "G_over_sigma_max": np.sum(G * G) / np.linalg.norm(G, 2),
           "sign_G_over_spectral_norm": np.sum(G * S) / np.linalg.norm(S, 2)}
    for k, v in got.items():
        assert round(float(v), 4) == ip[k], (k, v)
    assert round(float(nuclear), 4) == g["nuclear_norm_4dp"]
    assert got["polar"] > max(got["G_over_sigma_max"], got["sign_G_over_spectral_norm"])


def _sym_power(S, p):
    """S^p for a symmetric positive definite S, from its eigendecomposition."""
    w, Q = np.linalg.eigh(S)
    return (Q * w ** p) @ Q.T


@pytest.mark.parametrize("k", [1, 4])
def test_shampoo_without_accumulation_is_the_scaled_polar_factor(golden, k):
    """The lesson's Shampoo check: with k identical gradients and no
    accumulation beyond them, L = k G G^T and R = k G^T G, and the Shampoo
    direction L^{-1/4} G R^{-1/4} is the polar factor scaled by the printed
    factor (1 for k = 1, 1/2 for k = 4).  The polar factor comes from the
    oracle's cubic iteration run to convergence, the fractional powers from
    numpy's eigh: the two constructions share nothing."""
    g = golden("worked_example_2x2.json")
    G = np.array(g["G"])
    scale = g["shampoo_k_identical_gradients"][str(k)]
    shampoo = _sym_power(k * G @ G.T, -0.25) @ G @ _sym_power(k * G.T @ G, -0.25)
    polar = ns.newton_schulz(G, ns.CUBIC, 40, eps=0.0)
    np.testing.assert_allclose(shampoo, scale * polar, rtol=0, atol=1e-12)


def test_worked_example_singular_vectors_kept():
    # the quintic output is U diag(.) V^T with G's own singular vectors
    G = np.array([[3.0, 0.0], [4.0, 5.0]])
    U, s, Vt = np.linalg.svd(G)
    X = ns.newton_schulz(G, ns.QUINTIC, 5, eps=0.0)
    D = U.T @ X @ Vt.T
    assert abs(D[0, 1]) < 1e-12 and abs(D[1, 0]) < 1e-12
    np.testing.assert_allclose(np.diag(D), [0.753, 1.134], atol=5e-4)


# ---------------------------------------------------------------- scalar map

def test_scalar_map_printed(golden):
    g = golden("quintic_scalar_map.json")
    c = tuple(g["coefficients"])
    assert c == ns.QUINTIC
    traj = [ns.scalar_map(0.01, c, k) for k in range(1, 6)]
    np.testing.assert_allclose(np.round(traj, 3), g["start_0_01_trajectory_3dp"])
    assert round(float(ns.scalar_map(1.0, c, 1)), 3) == g["p_of_1_3dp"]
    assert round(float(ns.scalar_map(0.99995, c, 5)), 3) == g["start_0_99995_after_5_3dp"]
    assert round(float(ns.scalar_map(0.0100, c, 5)), 3) == g["start_0_0100_after_5_3dp"]
    band = ns.scalar_map(np.geomspace(0.01, 1.0, 20001), c, 5)
    lo, hi = g["band_after_5_for_start_in_0_01_to_1_2dp"]
    assert lo - 0.01 <= band.min() and band.max() <= hi + 0.01


def test_scalar_map_is_the_odd_polynomial():
    a, b, c = ns.QUINTIC
    for s in (0.3, -0.7, 1.2):
        assert ns.scalar_map(s, steps=1) == pytest.approx(a * s + b * s ** 3 + c * s ** 5, rel=1e-15)
    assert ns.scalar_map(-0.4, steps=5) == pytest.approx(-ns.scalar_map(0.4, steps=5), rel=1e-15)


def test_spectrum_64x256(golden):
    g = golden("spectrum_64x256.json")
    rng = np.random.default_rng(5)
    U, _ = np.linalg.qr(rng.standard_normal((64, 64)))
    V, _ = np.linalg.qr(rng.standard_normal((256, 64)))
    G = U @ np.diag(np.geomspace(1.0, 0.01, 64)) @ V.T
    O = ns.newton_schulz(G, ns.QUINTIC, g["steps"], eps=0.0)
    sv = _sv(O)
    assert round(sv.min(), 2) == g["sv_min_2dp"]
    assert round(sv.max(), 2) == g["sv_max_2dp"]
    update = 0.2 * np.sqrt(256) * O
    assert round(float(np.sqrt(np.mean(update ** 2))), 3) == g["update_rms_3dp_with_0_2_sqrt_max"]


# ---------------------------------------------------------------- Lemma 3

@pytest.mark.parametrize("shape", [(48, 80), (80, 48), (37, 37), (1, 9), (9, 1)])
@pytest.mark.parametrize("coeffs,steps", [(ns.QUINTIC, 5), (ns.CUBIC, 9), ((2.0, -1.5, 0.5), 12)])
def test_lemma3_closed_form(shape, coeffs, steps):
    m, n = shape
    k = min(m, n)
    rng = np.random.default_rng(m * 100 + n)
    U, _ = np.linalg.qr(rng.standard_normal((m, k)))
    V, _ = np.linalg.qr(rng.standard_normal((n, k)))
    s = np.geomspace(3.0, 0.02, k)
    G = (U * s[None, :]) @ V.T
    X = ns.newton_schulz(G, coeffs, steps, eps=1e-7)
    np.testing.assert_allclose(X, _closed_form(U, s, V, coeffs, steps, 1e-7), rtol=0, atol=1e-12)


def test_orientation_transposes_only_tall():
    rng = np.random.default_rng(3)
    G = rng.standard_normal((30, 20))
    np.testing.assert_allclose(ns.newton_schulz(G), ns.newton_schulz(G.T).T, atol=1e-13)


def test_special_cases_exact_polar():
    # diag(5, -2) -> diag(1, -1); rank one -> G / ||G||_F
    X = ns.newton_schulz(np.diag([5.0, -2.0]), ns.CUBIC, 40, eps=0.0)
    np.testing.assert_allclose(X, np.diag([1.0, -1.0]), atol=1e-14)
    rng = np.random.default_rng(4)
    d, a = rng.standard_normal(7), rng.standard_normal(11)
    G = np.outer(d, a)
    X = ns.newton_schulz(G, ns.CUBIC, 40, eps=0.0)
    np.testing.assert_allclose(X, G / np.linalg.norm(G), atol=1e-14)


def test_dyadic_workload_closed_form():
    # workloads.dyadic has a known SVD; the NS output keeps its structure
    rng = np.random.default_rng(6)
    n = 64
    d = wl.dyadic_spectrum(rng, n, 1e4)
    G = wl.dyadic_from_diag(d)
    X = ns.newton_schulz(G, ns.QUINTIC, 5, eps=1e-7)
    t = np.abs(d) / (np.linalg.norm(d) + 1e-7)
    expect = wl.dyadic_from_diag(np.sign(d) * ns.scalar_map(t, ns.QUINTIC, 5))
    np.testing.assert_allclose(X, expect, atol=1e-12)
    np.testing.assert_allclose(np.sort(np.linalg.svd(G, compute_uv=False)), np.sort(np.abs(d)), rtol=1e-10)


# ---------------------------------------------------------------- bf16 emulation

def test_bf16_emulation_without_rounding_is_the_iteration(monkeypatch):
    rng = np.random.default_rng(7)
    N = rng.standard_normal((24, 40)) * 1e-3
    monkeypatch.setattr(ns, "rnd", lambda x: np.asarray(x, dtype=np.float64))
    np.testing.assert_allclose(ns.newton_schulz_bf16(N), ns.newton_schulz(N), atol=1e-12)
    np.testing.assert_allclose(ns.newton_schulz_bf16(N.T), ns.newton_schulz(N.T), atol=1e-12)


def test_bf16_emulation_outputs_bf16_and_is_close():
    from oracle.bf16 import rnd
    rng = np.random.default_rng(8)
    N = rng.standard_normal((64, 160))
    X = ns.newton_schulz_bf16(N)
    np.testing.assert_array_equal(rnd(X), X)
    ref = ns.newton_schulz(N)
    assert np.linalg.norm(X - ref) / np.linalg.norm(ref) < 0.03

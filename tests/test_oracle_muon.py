"""Pins for oracle.muon: hand-derived two-step sequences with rank-one
gradients, closed forms from Lemma 3 and the pages' update-RMS numbers."""
import numpy as np
import pytest

from oracle import muon, ns


def _unit(rng, k):
    v = rng.standard_normal(k)
    return v / np.linalg.norm(v)


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (8, 8)])
@pytest.mark.parametrize("nesterov", [True, False])
@pytest.mark.parametrize("ema", [False, True])
def test_two_steps_rank_one(shape, nesterov, ema):
    m, n = shape
    rng = np.random.default_rng(11)
    u, v = _unit(rng, m), _unit(rng, n)
    uv = np.outer(u, v)
    g1, g2 = 0.7, -2.9          # gradient scalars along the fixed u v^T
    beta, lr, wd = 0.95, 0.02, 0.01
    W0 = rng.standard_normal((m, n))
    B = np.zeros((m, n))
    # hand recurrences for the scalar b_t along u v^T
    f = (1 - beta) if ema else 1.0
    b1 = f * g1
    nn1 = g1 + beta * b1 if nesterov else b1
    b2 = beta * b1 + f * g2
    nn2 = g2 + beta * b2 if nesterov else b2
    W = W0
    for g, b_exp, n_exp in ((g1, b1, nn1), (g2, b2, nn2)):
        out = muon.muon_step(W, g * uv, B, lr=lr, weight_decay=wd, momentum=beta,
                             nesterov=nesterov, momentum_ema=ema)
        np.testing.assert_allclose(out["B"], b_exp * uv, atol=1e-14)
        # rank one: normalised singular value |n|/(|n| + eps), sign kept
        sv = abs(n_exp) / (abs(n_exp) + 1e-7)
        O_exp = np.sign(n_exp) * ns.scalar_map(sv, ns.QUINTIC, 5) * uv
        np.testing.assert_allclose(out["O"], O_exp, atol=1e-13)
        s = 0.2 * np.sqrt(max(m, n))
        np.testing.assert_allclose(out["W"], (1 - lr * wd) * W - lr * s * O_exp, atol=1e-13)
        np.testing.assert_allclose(out["dW"], -lr * s * O_exp, atol=1e-13)
        W, B = out["W"], out["B"]


def test_full_rank_closed_form_and_original_scale():
    m, n = 12, 20
    rng = np.random.default_rng(12)
    U, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, m)))
    s = np.geomspace(1.0, 1e-3, m)
    G = (U * s) @ V.T
    W = rng.standard_normal((m, n))
    beta = 0.9
    for mode, scale in (("match_rms_adamw", 0.2 * np.sqrt(n)), ("original", 1.0)):
        out = muon.muon_step(W, G, np.zeros((m, n)), momentum=beta, lr=0.1,
                             weight_decay=0.5, adjust_lr=mode)
        t = (1 + beta) * s / ((1 + beta) * np.linalg.norm(s) + 1e-7)
        O = (U * ns.scalar_map(t)) @ V.T
        np.testing.assert_allclose(out["O"], O, atol=1e-12)
        np.testing.assert_allclose(out["W"], (1 - 0.05) * W - 0.1 * scale * O, atol=1e-12)
    # tall: the original factor is sqrt(m / n)
    assert muon.shape_scale(30, 10, "original") == pytest.approx(np.sqrt(3.0))
    assert muon.shape_scale(10, 30, "original") == 1.0
    with pytest.raises(ValueError):
        muon.shape_scale(3, 4, "spectral_unclamped")


def test_ema_and_sum_momentum_give_the_same_update():
    rng = np.random.default_rng(13)
    G = rng.standard_normal((16, 24))
    W = rng.standard_normal((16, 24))
    a = muon.muon_step(W, G, np.zeros_like(G), momentum_ema=False)
    b = muon.muon_step(W, G, np.zeros_like(G), momentum_ema=True)
    np.testing.assert_allclose(b["B"], 0.05 * a["B"], atol=1e-15)
    np.testing.assert_allclose(a["O"], b["O"], atol=1e-6)


def test_update_rms_numbers(golden):
    g = golden("update_rms.json")
    m, n = g["mlp_weight"]["rows"], g["mlp_weight"]["cols"]
    polar_rms = np.sqrt(min(m, n) / (m * n))            # ||UV^T||_F^2 = min(m, n)
    assert round(polar_rms, 3) == g["mlp_weight"]["polar_rms_3dp"]
    assert muon.shape_scale(m, n, "original") == g["mlp_weight"]["original_factor"]
    assert round(muon.shape_scale(m, n, "original") * polar_rms, 3) == g["mlp_weight"]["original_rms_3dp"]
    assert round(muon.shape_scale(m, n), 1) == g["mlp_weight"]["match_factor_1dp"]
    assert round(muon.shape_scale(m, n) * polar_rms, 1) == g["mlp_weight"]["match_rms_1dp"]
    q = g["quick_check"]
    r = muon.shape_scale(q["rows"], q["cols"]) * np.sqrt(min(q["rows"], q["cols"]) / (q["rows"] * q["cols"]))
    assert r == pytest.approx(q["update_rms_over_lr"])


def test_bf16_precision_mode_is_close_and_bf16():
    from oracle.bf16 import rnd
    rng = np.random.default_rng(14)
    G = rng.standard_normal((32, 48)).astype(np.float32)
    W = rng.standard_normal((32, 48)).astype(np.float32)
    a = muon.muon_step(W, G, np.zeros_like(G))
    b = muon.muon_step(W, G, np.zeros_like(G), precision="bf16")
    np.testing.assert_array_equal(rnd(b["O"]), b["O"])
    assert np.linalg.norm(a["O"] - b["O"]) / np.linalg.norm(a["O"]) < 0.03
    with pytest.raises(ValueError):
        muon.muon_step(W, G, np.zeros_like(G), precision="fp16")

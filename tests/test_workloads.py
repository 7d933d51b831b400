"""The seeded input recipes: determinism, shapes and the stated scalings."""
import numpy as np

import workloads as wl


def test_cfg1_recipe():
    W, G, B = wl.cfg1()
    assert W.shape == G.shape == (256, 512) and W.dtype == np.float32
    assert abs(np.linalg.norm(G.astype(np.float64)) - 1) < 1e-6
    # rank 64 up to the float32 rounding of the entries
    sv = np.linalg.svd(G.astype(np.float64), compute_uv=False)
    assert sv[63] > 1e3 * sv[64]
    assert abs(W.std() - 0.02) < 1e-3 and not B.any()
    W2, G2, _ = wl.cfg1()
    np.testing.assert_array_equal(G, G2)


def test_gauss_spike_ratio_and_rank():
    rng = wl.rng_of("t", 1)
    P, Q = wl.spike_factors(rng, 64, 96, 4)
    G = wl.gauss_spike(rng, 64, 96, 4, 1e-3, 10.0, (P, Q)).astype(np.float64)
    s = np.linalg.svd(G, compute_uv=False)
    # the spike carries ~100/101 of the energy in 4 directions
    assert (s[:4] ** 2).sum() / (s ** 2).sum() > 0.95
    assert s[4] < 0.2 * s[3]


def test_expert_scale_shared():
    Ws, Gs, scale = wl.cfg3_expert(0, 3, wl.CFG3_MINI)
    assert [g.shape for g in Gs] == [(96, 256), (96, 256), (256, 96)]
    for g in Gs:
        assert abs(g.std() / (scale * 1e-3) - 1) < 0.05


def test_dyadic_known_svd():
    G, d = wl.cfg5_square(64)
    assert abs(np.linalg.norm(G.astype(np.float64)) - 64) < 1e-3
    s = np.sort(np.linalg.svd(G.astype(np.float64), compute_uv=False))
    np.testing.assert_allclose(s, np.sort(np.abs(d)), rtol=1e-5, atol=1e-6)
    assert s[-1] / s[0] > 0.9e4


def test_haar_heads():
    mats, factors = wl.cfg5_heads(3, 16)
    U, s, V = factors[1]
    np.testing.assert_allclose(U.T @ U, np.eye(16), atol=1e-12)
    np.testing.assert_allclose(mats[1], (U * s) @ V.T, atol=1e-5)


def test_config_lists():
    assert len(wl.cfg2_list()) == 224
    assert len(wl.cfg3_list()) == 1536
    assert len(wl.cfg4_list()) == 8
    params = sum(m * n for _, _, m, n in wl.cfg2_list())
    assert abs(params / 1e9 - 6.98) < 0.01


def test_spike_stream_fixed_spike():
    s = wl.SpikeStream("t", "sq", 0, 32, 48, wl.CFG4_MINI)
    g1, g2 = s.next(), s.next()
    assert not np.array_equal(g1, g2)
    P, Q = s.factors
    # both steps share the spike directions
    Pq, _ = np.linalg.qr(P)
    for g in (g1, g2):
        proj = np.linalg.norm(Pq.T @ g) / np.linalg.norm(g)
        assert proj > 0.9

"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times: every matrix of each workload goes through one call; the checks use
sampled outputs that the fp64 oracle (or a closed form) can compute one by
one, and properties that hold at any size."""
import numpy as np
import pytest

import workloads as wl
from gates import basis_gate, ns_gate, rel
from gpu_env import context
from oracle import muon as omuon
from oracle import ns as ons
from oracle import soap as osoap

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    return context()


def _np(t):
    return t.detach().cpu().numpy().astype(np.float64)


def _hadamard_cols(n, idx):
    """Columns idx of the Sylvester-Hadamard matrix H_n (entries +-1)."""
    r = np.arange(n)[:, None] & np.asarray(idx)[None, :]
    bits = np.zeros(r.shape, dtype=np.int64)
    while r.any():
        bits += r & 1
        r = r >> 1
    return 1.0 - 2.0 * (bits & 1)


@pytest.mark.parametrize("n", [2048, 8192, 16384])
def test_ns_sweep_full_size(ctx, n):
    """Known-SVD input G = H diag(d) H / n: project the GPU output on a
    sample of 48 of its own resolved singular pairs (the exact result is
    diag(phi^5(|d| / ||d||)) there) and check sampled rows elementwise."""
    import torch
    G, d = wl.cfg5_square(n)
    O = ctx.ns_orthogonalize([torch.from_numpy(G).cuda()])[0]
    torch.cuda.synchronize()
    t = np.abs(d) / (np.linalg.norm(d) + 1e-7)
    phi = ons.scalar_map(t)
    rng = np.random.default_rng(n)
    resolved = np.nonzero(t >= 1e-2)[0]
    S = rng.choice(resolved, size=48, replace=False)
    H = _hadamard_cols(n, S) / np.sqrt(n)            # u_k = H e_k / sqrt(n)
    V = H * np.sign(d[S])[None, :]                   # v_k = sign(d_k) u_k
    Ot = O.cpu().numpy()                               # float32, n x n
    P = H.T @ (Ot @ V.astype(np.float32)).astype(np.float64)
    assert rel(P, np.diag(phi[S])) <= 2e-2
    sv = np.linalg.svd(P, compute_uv=False)
    assert 0.6 <= sv.min() and sv.max() <= 1.3
    # sampled rows against the closed form O[i, j] = o[i xor j]
    o = wl.fwht(np.sign(d) * phi) / n
    rows = rng.choice(n, size=8, replace=False)
    cols = np.arange(n)
    exact = o[rows[:, None] ^ cols[None, :]]
    assert rel(Ot[rows].astype(np.float64), exact) <= 0.1   # noise floor of the full matrix (cond 1e4)


def _gpt_on_gpu(dev, keep, layers=32, hidden=4096, kv=1024, ffn=14336, rank=16):
    """The benchmark's dense-GPT workload (bench.gpt_workload recipe),
    keeping the spike factors of the (layer, name) pairs in ``keep``."""
    import torch
    Ws, Gs, Bs, shapes, spikes = [], [], [], [], {}
    for layer in range(layers):
        for name, m, n in wl.gpt_shapes(hidden, kv, ffn):
            g = torch.Generator(device=dev)
            g.manual_seed(wl.seed_of("bench-cfg2", layer, name))
            W = torch.randn(m, n, generator=g, device=dev) * 0.02
            G = torch.randn(m, n, generator=g, device=dev) * 1e-3
            P = torch.randn(m, rank, generator=g, device=dev)
            Q = torch.randn(n, rank, generator=g, device=dev)
            S = P @ Q.T
            S *= 10.0 * G.norm() / S.norm()
            G += S
            del S
            if (layer, name) in keep:
                spikes[(layer, name)] = (P.cpu().numpy().astype(np.float64), Q.cpu().numpy().astype(np.float64),
                                         len(Ws))
            Ws.append(W)
            Gs.append(G)
            Bs.append(torch.zeros_like(W))
            shapes.append((m, n))
    return Ws, Gs, Bs, shapes, spikes


def _leading_svd(N, seed, k):
    """Leading k singular triplets of N by subspace iteration started from
    the columns of ``seed`` (the spike's left factor), then a Rayleigh-Ritz
    step; the gap after the spike's singular values is a factor of about 50,
    so a few iterations reach fp64 accuracy."""
    rng = np.random.default_rng(0)
    U = np.linalg.qr(np.hstack([seed, rng.standard_normal((N.shape[0], k - seed.shape[1]))]))[0]
    for _ in range(8):
        V = np.linalg.qr(N.T @ U)[0]
        U = np.linalg.qr(N @ V)[0]
    u, s, vt = np.linalg.svd(U.T @ N @ V)
    return U @ u, s, (V @ vt.T).T


def test_muon_dense_gpt_full_step(ctx):
    """All 224 matrices (6.98 G parameters) in one call.  Five of them are
    recomputed by the fp64 oracle and its bf16 emulation and gated like every
    Newton-Schulz parity test: wk, wv, wq, and one matrix of each orientation
    of the 4096 x 14336 bucket that dominates the step (gate, stored tall,
    and down, stored wide)."""
    import torch
    dev = torch.device("cuda", 0)
    keep = {(3, "wk"), (17, "wv"), (5, "wq"), (9, "gate"), (30, "down")}
    Ws, Gs, Bs, shapes, spikes = _gpt_on_gpu(dev, keep)
    W0 = {k: _np(Ws[v[2]]) for k, v in spikes.items()}
    G0 = {k: _np(Gs[v[2]]) for k, v in spikes.items()}
    flags = torch.full((len(Ws),), -1, dtype=torch.int32, device=dev)
    ctx.muon_step(Ws, Gs, Bs, lr=0.02, weight_decay=0.01, momentum=0.95, nonfinite=flags)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    assert (flags.cpu().numpy() == 0).all()
    decay = np.float64(np.float32(1 - 0.02 * 0.01))
    for key, (P, Q, i) in spikes.items():
        m, n = shapes[i]
        Wg, Bg = _np(Ws[i]), _np(Bs[i])
        np.testing.assert_array_equal(Bg, G0[key])          # B = 0.95 * 0 + G exactly
        O = (decay * W0[key] - Wg) / (0.02 * 0.2 * np.sqrt(max(m, n)))
        hp = dict(lr=0.02, weight_decay=0.01, momentum=0.95)
        ref = omuon.muon_step(W0[key], G0[key], np.zeros((m, n)), **hp)
        emu = omuon.muon_step(W0[key], G0[key], np.zeros((m, n)), precision="bf16", **hp)
        if m * n <= 1024 * 4096:
            svd = np.linalg.svd(ref["N"], full_matrices=False)
            fro = None
        else:
            # the resolved subspace (sigma >= 1e-2 ||N||_F) is the spike's: 20
            # leading triplets hold it with room to spare
            svd = _leading_svd(ref["N"], P, 20)
            fro = np.linalg.norm(ref["N"])
        g = ns_gate(ref["N"], O, ref["O"], emu["O"], svd=svd, fro=fro)
        assert g["k"] >= 16, (key, g)
        # any size: on the rank-16 spike subspace the update is near-orthogonal
        Pq, _ = np.linalg.qr(P)
        Qq, _ = np.linalg.qr(Q)
        sv = np.linalg.svd(Pq.T @ O @ Qq, compute_uv=False)
        assert 0.6 <= sv.min() and sv.max() <= 1.3, (key, sv.min(), sv.max())
        rms = np.sqrt(np.mean(O ** 2)) * np.sqrt(max(m, n))
        assert 0.2 <= rms <= 1.3, (key, rms)                 # singular values in the band, most resolved
    del Ws, Gs, Bs
    ctx.workspace = None
    torch.cuda.empty_cache()


def test_muon_moe_full_step(ctx):
    """All 1536 expert matrices (4 layers x 128 experts x 3) in one call;
    sampled experts against the oracle in both precision modes."""
    import torch
    import bench
    dev = torch.device("cuda", 0)
    cfg = wl.CFG3
    # the benchmark's expert batch (generated on the device), with three
    # experts replaced by the NumPy recipe so the oracle sees the same inputs
    Ws, Gs, _, _ = bench.moe_workload(dev)
    W0 = {}
    for layer, e in ((0, 5), (2, 77), (3, 127)):
        w, g, _ = wl.cfg3_expert(layer, e, cfg)
        for k in range(3):
            i = (layer * cfg["experts"] + e) * 3 + k
            Ws[i] = torch.from_numpy(w[k]).cuda()
            Gs[i] = torch.from_numpy(g[k]).cuda()
            W0[(layer, e, k)] = (i, w[k], g[k])
    Bs = [torch.zeros_like(w) for w in Ws]
    ctx.muon_step(Ws, Gs, Bs, lr=0.02, weight_decay=0.01, momentum=0.95)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    decay = np.float64(np.float32(1 - 0.02 * 0.01))
    for key, (i, w, g) in W0.items():
        m, n = w.shape
        ref = omuon.muon_step(w, g, np.zeros((m, n)), lr=0.02, weight_decay=0.01, momentum=0.95)
        emu = omuon.muon_step(w, g, np.zeros((m, n)), lr=0.02, weight_decay=0.01, momentum=0.95, precision="bf16")
        O = (decay * w.astype(np.float64) - _np(Ws[i])) / (0.02 * 0.2 * np.sqrt(max(m, n)))
        ns_gate(ref["N"], O, ref["O"], emu["O"])
    del Ws, Gs, Bs
    ctx.workspace = None
    torch.cuda.empty_cache()


def test_soap_full_size_sampled(ctx):
    """The SOAP workload at full size (4 x 4096^2 two-sided, 4 x 4096x14336
    left-sided), warmed up by 10 steps of the GPU path; step 11 of one
    two-sided and one one-sided matrix is recomputed by the fp64 oracle from
    the same state."""
    import torch
    import bench
    dev = torch.device("cuda", 0)
    mats, fill = bench.soap_workload(dev)
    hp = dict(lr=3e-3, beta1=0.95, beta2=0.95, eps=1e-8, weight_decay=0.0)
    for t in range(1, 11):
        fill()
        ctx.soap_step(mats, t, **hp)
    fill()
    torch.cuda.synchronize()
    keys = ("W", "G", "M", "V", "L", "QL", "R", "QR")
    state = {i: {k: (_np(mats[i][k]) if k in mats[i] else None) for k in keys} for i in (0, 4)}
    flags = torch.full((len(mats),), -1, dtype=torch.int32, device=dev)
    ctx.soap_step(mats, 11, nonfinite=flags, **hp)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    assert (flags.cpu().numpy() == 0).all()
    from oracle.bf16 import rnd
    from oracle.qr import qr_positive
    for i, S in state.items():
        ref = osoap.soap_step(S["W"], S["G"], S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"], t=11, **hp)
        out = {k: _np(mats[i][k]) for k in keys if k in mats[i] and k != "G"}
        assert rel(out["M"], ref["M"]) <= 1e-6
        # the refresh with the emulation's bf16 factor-EMA operands
        Gb = rnd(S["G"])
        L_emu = 0.95 * S["L"] + 0.05 * (Gb @ Gb.T)
        Y = L_emu @ S["QL"]
        Q_emu, R_emu = qr_positive(Y)
        assert rel(out["L"], L_emu) <= 1e-4
        Q = out["QL"]
        idx = np.random.default_rng(i).choice(Q.shape[0], 256, replace=False)
        assert np.abs(Q[:, idx].T @ Q[:, idx] - np.eye(256)).max() <= 1e-4
        # warm factor: every column of qr(L Q_old) resolved (r_j >= 1e-3) and
        # within the fp32-level bound of gates.basis_gate, and the whole basis
        # within 5e-3
        sel, _ = basis_gate(Q, L_emu, S["QL"])
        assert sel.all()
        assert rel(Q, Q_emu) <= 5e-3
        assert rel(out["W"] - S["W"], ref["dW"]) <= 2e-2
    del mats
    ctx.workspace = None
    torch.cuda.empty_cache()

"""Seeded synthetic inputs for the Muon / SOAP optimizer-step workloads.

This module is shared by the oracle-side tests and by the GPU-side tests and
benchmark.  It holds input recipes only - random draws, shapes and scalings -
and none of the optimizer arithmetic.  Every array is float32 (what the GPU
path receives); the oracle upcasts it exactly.

Recipes (seeded NumPy PCG64 streams; float64 draws rounded to float32):

* ``lowrank_sum``  - G = sum_i delta_i x_i^T of ``k`` rank-one terms with
  N(0,1) factors, scaled to Frobenius norm 1 (single-matrix Muon workload).
* ``gauss_spike``  - G = E + S: E iid N(0, noise_std^2) and S = P Q^T with
  P (m x k), Q (n x k) iid N(0,1), rescaled so ||S||_F = ratio * ||E||_F
  (gradient-shaped matrices of the dense-GPT and SOAP workloads).
* ``expert_grads`` - G_e = exp(z_e) E with z_e ~ N(0,1) shared by one
  expert's matrices and E iid N(0, noise_std^2) (heavy-tailed per-expert
  scale of the MoE workload).
* ``dyadic``       - an n x n matrix (n a power of two) with a KNOWN SVD:
  G = H diag(d) H / n with H the Sylvester-Hadamard matrix and d a random
  sign-and-permutation of a geometric spectrum 1 -> 1/cond.  Then
  G[i, j] = g[i xor j] with g = H d / n, so it is built in O(n^2) and any
  function of its singular values has the same structure (left singular
  vectors H/sqrt(n), right singular vectors H diag(sign d)/sqrt(n)).
  Scaled to entry RMS 1 (||G||_F = n).
* ``haar_spectrum`` - U diag(s) V^T with Haar-random U, V (QR of a Gaussian
  with the sign fix) and the same geometric spectrum; used for the batched
  per-head matrices.
* weights W ~ N(0, 0.02^2); momentum and moment buffers start at zero.
"""

import zlib

import numpy as np

# ----------------------------------------------------------------------------
# basic seeded streams


def seed_of(*parts):
    """Stable 32-bit seed from a tuple of names/numbers."""
    return zlib.crc32("/".join(str(p) for p in parts).encode())


def rng_of(*parts):
    return np.random.default_rng(seed_of(*parts))


def f32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))


def gaussian(rng, shape, std=1.0):
    return f32(rng.standard_normal(shape) * std)


def weights(rng, m, n, std=0.02):
    return gaussian(rng, (m, n), std)


# ----------------------------------------------------------------------------
# gradient recipes


def lowrank_sum(rng, m, n, k=64):
    delta = rng.standard_normal((m, k))
    x = rng.standard_normal((n, k))
    G = delta @ x.T
    return f32(G / np.linalg.norm(G))


def spike_factors(rng, m, n, k):
    return rng.standard_normal((m, k)), rng.standard_normal((n, k))


def gauss_spike(rng, m, n, k=16, noise_std=1e-3, ratio=10.0, factors=None):
    """E + S with ||S||_F = ratio ||E||_F; ``factors`` fixes (P, Q)."""
    E = rng.standard_normal((m, n)) * noise_std
    P, Q = factors if factors is not None else spike_factors(rng, m, n, k)
    S = P @ Q.T
    S *= ratio * np.linalg.norm(E) / np.linalg.norm(S)
    return f32(E + S)


def expert_grads(rng, shapes, noise_std=1e-3):
    """One expert's gradients: a log-normal scale shared by its matrices."""
    scale = np.exp(rng.standard_normal())
    return [f32(scale * rng.standard_normal(s) * noise_std) for s in shapes], scale


def geometric_spectrum(n, cond=1e4):
    return 10.0 ** (-np.log10(cond) * np.arange(n) / max(n - 1, 1))


def fwht(x):
    """Unnormalised fast Walsh-Hadamard transform along the last axis."""
    x = np.array(x, dtype=np.float64, copy=True)
    n = x.shape[-1]
    h = 1
    while h < n:
        y = x.reshape(x.shape[:-1] + (n // (2 * h), 2, h))
        a = y[..., 0, :].copy()
        b = y[..., 1, :]
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        h *= 2
    return x


def dyadic_spectrum(rng, n, cond=1e4):
    """Signed, permuted singular values d (length n, a power of two)."""
    if n & (n - 1):
        raise ValueError("dyadic matrices need a power-of-two size")
    s = geometric_spectrum(n, cond)
    d = s[rng.permutation(n)] * rng.choice([-1.0, 1.0], size=n)
    return d * (n / np.linalg.norm(d))     # entry RMS 1: ||G||_F = ||d|| = n


def dyadic_from_diag(d):
    """G[i, j] = g[i xor j] with g = H d / n (float64)."""
    n = d.shape[0]
    g = fwht(d) / n
    idx = np.arange(n)
    return g[idx[:, None] ^ idx[None, :]]


def dyadic(rng, n, cond=1e4):
    d = dyadic_spectrum(rng, n, cond)
    return f32(dyadic_from_diag(d)), d


def haar(rng, n):
    Z = rng.standard_normal((n, n))
    Q, R = np.linalg.qr(Z)
    return Q * np.sign(np.diag(R))[None, :]


def haar_spectrum(rng, n, cond=1e4):
    s = geometric_spectrum(n, cond)
    s = s * (n / np.linalg.norm(s))
    U, V = haar(rng, n), haar(rng, n)
    return f32((U * s[None, :]) @ V.T), (U, s, V)


# ----------------------------------------------------------------------------
# the workloads (full sizes and reduced "mini" variants with the same structure

# single Muon step on one 256 x 512 weight
CFG1 = dict(rows=256, cols=512, rank=64, lr=0.02, weight_decay=0.01,
            momentum=0.95, seed=0)


def cfg1():
    rng = np.random.default_rng(CFG1["seed"])
    m, n = CFG1["rows"], CFG1["cols"]
    W = weights(rng, m, n)
    G = lowrank_sum(rng, m, n, CFG1["rank"])
    return W, G, np.zeros_like(W)


# dense GPT, 32 layers, hidden 4096, 32 q heads / 8 kv heads of dim 128, FFN 14336
def gpt_shapes(hidden=4096, kv=1024, ffn=14336):
    return [("wq", hidden, hidden), ("wk", kv, hidden), ("wv", kv, hidden),
            ("wo", hidden, hidden), ("gate", ffn, hidden), ("up", ffn, hidden),
            ("down", hidden, ffn)]


CFG2 = dict(layers=32, hidden=4096, kv=1024, ffn=14336, rank=16,
            noise_std=1e-3, ratio=10.0, lr=0.02, weight_decay=0.01,
            momentum=0.95)
CFG2_MINI = dict(CFG2, layers=2, hidden=512, kv=128, ffn=1792)


def cfg2_list(cfg=CFG2):
    out = []
    for layer in range(cfg["layers"]):
        for name, m, n in gpt_shapes(cfg["hidden"], cfg["kv"], cfg["ffn"]):
            out.append((layer, name, m, n))
    return out


def cfg2_matrix(layer, name, m, n, cfg=CFG2, tag="cfg2"):
    rng = rng_of(tag, layer, name)
    W = weights(rng, m, n)
    G = gauss_spike(rng, m, n, cfg["rank"], cfg["noise_std"], cfg["ratio"])
    return W, G


# MoE experts: 4 layers x 128 experts, hidden 2048, expert FFN 768
CFG3 = dict(layers=4, experts=128, hidden=2048, ffn=768, noise_std=1e-3,
            lr=0.02, weight_decay=0.01, momentum=0.95)
CFG3_MINI = dict(CFG3, layers=1, experts=24, hidden=256, ffn=96)


def cfg3_list(cfg=CFG3):
    out = []
    for layer in range(cfg["layers"]):
        for e in range(cfg["experts"]):
            for name, m, n in (("gate", cfg["ffn"], cfg["hidden"]),
                               ("up", cfg["ffn"], cfg["hidden"]),
                               ("down", cfg["hidden"], cfg["ffn"])):
                out.append((layer, e, name, m, n))
    return out


def cfg3_expert(layer, e, cfg=CFG3, tag="cfg3"):
    rng = rng_of(tag, layer, e)
    shapes = [(cfg["ffn"], cfg["hidden"]), (cfg["ffn"], cfg["hidden"]),
              (cfg["hidden"], cfg["ffn"])]
    Gs, scale = expert_grads(rng, shapes, cfg["noise_std"])
    Ws = [weights(rng, *s) for s in shapes]
    return Ws, Gs, scale


# SOAP: 4 x 4096^2 + 4 x 4096 x 14336, factors kept only for sides <= 8192
CFG4 = dict(square=4096, wide=14336, n_square=4, n_wide=4, rank=32,
            noise_std=1e-3, ratio=10.0, warm_steps=10, lr=3e-3, beta1=0.95,
            beta2=0.95, eps=1e-8, weight_decay=0.0, max_factor=8192)
CFG4_MINI = dict(CFG4, square=256, wide=896, n_square=2, n_wide=2,
                 max_factor=512, rank=8)


def cfg4_list(cfg=CFG4):
    out = [("sq", i, cfg["square"], cfg["square"]) for i in range(cfg["n_square"])]
    out += [("wide", i, cfg["square"], cfg["wide"]) for i in range(cfg["n_wide"])]
    return out


class SpikeStream:
    """Gradients of one SOAP matrix over steps: fixed spike, fresh noise."""

    def __init__(self, tag, kind, i, m, n, cfg=CFG4):
        self.rng = rng_of(tag, kind, i)
        self.m, self.n, self.cfg = m, n, cfg
        self.factors = spike_factors(self.rng, m, n, cfg["rank"])
        self.W = weights(self.rng, m, n)

    def next(self):
        c = self.cfg
        return gauss_spike(self.rng, self.m, self.n, c["rank"], c["noise_std"],
                           c["ratio"], self.factors)


# Newton-Schulz sweep: square sizes and a batch of per-head 128 x 128 matrices
CFG5 = dict(sizes=(512, 1024, 2048, 4096, 8192, 16384), heads=4096,
            head_dim=128, cond=1e4)


def cfg5_square(n, cfg=CFG5, tag="cfg5"):
    return dyadic(rng_of(tag, n), n, cfg["cond"])


def cfg5_heads(count, dim=128, cfg=CFG5, tag="cfg5-heads"):
    rng = rng_of(tag, count, dim)
    mats, factors = [], []
    for _ in range(count):
        G, f = haar_spectrum(rng, dim, cfg["cond"])
        mats.append(G)
        factors.append(f)
    return mats, factors

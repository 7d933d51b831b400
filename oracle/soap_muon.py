"""SOAP-Muon for one matrix, in float64 (test infrastructure: only tests,
the smoke check and the benchmark's CPU baseline call the oracle).

SOAP preconditions the Muon momentum, Newton-Schulz orthogonalises the
result and Muon's scaled, decoupled-decay update applies it ("初探优化器（一）：
从SGD到SOAP-Muon", section 7.1: precondition the momentum with SOAP, then
orthogonalise with Muon; section 7.2, the implementation notes of the
Track-3 records: the basis is refreshed every step by one power step + QR,
the Gram factors are moving averages of the raw gradient with coefficient
0.9, the momentum is preconditioned with the basis built at the previous
step, and the preconditioned matrix is rescaled by a matrix norm before
Newton-Schulz).  The section's own formula did not survive extraction; the
steps below are the plainest reading of those notes:

    1. B = mu B + G ;  N = G + mu B (Nesterov) or N = B     (Muon's momentum)
    2. N' = Q_L^T N Q_R ;  G' = Q_L^T G Q_R                 (previous basis)
    3. V = b2 V + (1 - b2) G' * G'
    4. P = Q_L [ N' / (sqrt(V / (1 - b2^t)) + eps) ] Q_R^T
    5. O = NS(P)            (the rescaling is Newton-Schulz's own Frobenius
                             normalisation; the pages leave the norm open)
    6. W = (1 - lr wd) W - lr s O,   s = 0.2 sqrt(max(m, n)) or sqrt(max(1, m/n))
    7. L = bs L + (1 - bs) G G^T ;  R likewise ;  Q = qr(L Q)
       (the power step + QR of ``oracle.soap``; used from the next step on;
        ``damping > 0`` is the same optional departure as there)

A side whose factor is ``None`` uses the identity basis, as in SOAP.

``precision="bf16"`` reproduces the GPU path's rounding points: the
rotations take two-plane bf16 operands (``oracle.soap``), P is stored in
fp32, Newton-Schulz runs in its bf16 emulation, the factor EMAs take
bf16(G), and the refresh is exact.
"""

import numpy as np

from .bf16 import rnd, rnd32
from .muon import shape_scale
from .ns import QUINTIC, newton_schulz, newton_schulz_bf16
from .soap import damping_of
from .qr import qr_positive


def soap_muon_step(W, G, B, V, L=None, QL=None, R=None, QR=None, *, t=1,
                   lr=0.02, weight_decay=0.01, momentum=0.95, nesterov=True,
                   beta2=0.95, shampoo_beta=0.9, eps=1e-8, bias_correction=True,
                   ns_steps=5, coeffs=QUINTIC, ns_eps=1e-7,
                   adjust_lr="match_rms_adamw", damping=0.0, precision="fp64"):
    """One SOAP-Muon step.  Inputs are not modified; returns the new state
    and the intermediates P (preconditioned momentum) and O."""
    if precision not in ("fp64", "bf16"):
        raise ValueError(f"unknown precision {precision!r}")
    emu = precision == "bf16"

    def split2(x):
        h = rnd(x)
        return h, rnd(x - h)

    def prod(A, Bm):
        if not emu:
            return A @ Bm
        Ah, Al = split2(A)
        Bh, Bl = split2(Bm)
        return Ah @ Bh + Ah @ Bl + Al @ Bh

    def keep(x):
        if not emu:
            return x
        h, l = split2(x)
        return h + l

    f64 = lambda x: None if x is None else np.asarray(x, dtype=np.float64)
    W, G, B, V = f64(W), f64(G), f64(B), f64(V)
    L, QL, R, QR = f64(L), f64(QL), f64(R), f64(QR)
    left, right = QL is not None, QR is not None
    m, n = G.shape

    # 1. Muon momentum
    B = momentum * B + G
    N = G + momentum * B if nesterov else B

    # 2-4. precondition with the previous bases
    def rotate_in(X):
        if left and right:
            return prod(keep(prod(QL.T, X)), QR)
        if left:
            return prod(QL.T, X)
        if right:
            return prod(X, QR)
        return X

    Nr = rotate_in(N)
    Gr = rotate_in(G)
    V = beta2 * V + (1.0 - beta2) * Gr * Gr
    bc2 = 1.0 - beta2 ** t if bias_correction else 1.0
    Dbar = Nr / (np.sqrt(V / bc2) + eps)
    if left and right:
        P = prod(keep(prod(QL, Dbar)), QR.T)
    elif left:
        P = prod(QL, Dbar)
    elif right:
        P = prod(Dbar, QR.T)
    else:
        P = Dbar

    # 5-6. orthogonalise and apply
    if emu:
        O = newton_schulz_bf16(rnd32(P), coeffs, ns_steps, ns_eps)
    else:
        O = newton_schulz(P, coeffs, ns_steps, ns_eps)
    s = shape_scale(m, n, adjust_lr)
    decayed = (1.0 - lr * weight_decay) * W
    W_new = decayed - lr * s * O

    # 7. factor EMAs with the raw gradient and the basis refresh for the next step
    Gb = rnd(G) if emu else G
    QL_new, QR_new = QL, QR
    def power_step(F, Q):
        d = damping_of(F, damping)
        return qr_positive(F @ Q if d == 0.0 else (F + d * np.eye(F.shape[0])) @ Q)[0]

    if left:
        L = shampoo_beta * L + (1.0 - shampoo_beta) * (Gb @ Gb.T)
        QL_new = power_step(L, QL)
    if right:
        R = shampoo_beta * R + (1.0 - shampoo_beta) * (Gb.T @ Gb)
        QR_new = power_step(R, QR)
    return {"W": W_new, "B": B, "V": V, "L": L, "QL": QL_new, "R": R, "QR": QR_new,
            "N": N, "P": P, "O": O, "dW": W_new - decayed}

"""The SOAP step for one matrix, in float64, with a per-step basis refresh.

Steps, in the order used by the per-step-refresh variant ("Reading notes on
SOAP, Muon, and Beyond", section 4: the basis is re-orthogonalised every step
with the current gradient folded in; "初探优化器（一）", section 6.2 steps 1-5;
"LLM Optimizers: From SGD and AdamW to SOAP, Muon, and Scalable Training",
section 11.1 equations):

    1. L = bs L + (1 - bs) G G^T ;   R = bs R + (1 - bs) G^T G
    2. Q_L = qr(L Q_L) ;             Q_R = qr(R Q_R)            (one power step)
    3. M = b1 M + (1 - b1) G                            (original space)
    4. M' = Q_L^T M Q_R ;            G' = Q_L^T G Q_R
    5. V = b2 V + (1 - b2) G' * G'                      (rotated space)
       Dbar = (M' / (1 - b1^t)) / (sqrt(V / (1 - b2^t)) + eps)
    6. D = Q_L Dbar Q_R^T
    7. W = (1 - lr wd) W - lr D

Step 2 is the pages' refresh as written: one power-iteration step on the
factor, followed by a QR, with the current gradient already folded into the
factor (the reading notes, section 4; "初探优化器（一）", section 6.2 step 2;
the SOAP workload: "one power iteration Q <- qr(L Q)").  QR is LAPACK's
Householder factorisation with the positive-diagonal convention
(``oracle.qr``).  Where L Q is singular the QR is not unique; Householder
then completes Q with trivial reflectors, so a zero factor (only zero
gradients seen) gives Q = I.

``damping > 0`` is an option that departs from the pages: the power step
then runs on L + d I with d = damping * trace(L) (d = 1 when the trace is
zero), the damping the Shampoo family applies to its factors ("Matrix
optimizers: K-FAC, Shampoo and Muon", Shampoo, L0 = eps I; K-FAC's
A + gamma I).  It keeps L's eigenvectors but changes how far the basis moves
inside the low-eigenvalue subspace, and so changes the update; the default
is 0.  The stored factor L is never damped.

A side whose factor is ``None`` uses the identity basis (one-sided SOAP for
very large axes, section 11.2 of the LLM Optimizers guide); with both sides
identity the step is AdamW.  Keeping M in the original space and rotating it
with the current basis is the same as the section 11.1 change-of-basis rule
for the stored first moment.  V is never re-rotated.

``precision="bf16"`` reproduces the GPU path's declared rounding points.
The factor EMAs take bf16 operands; the basis refresh (power step and QR)
is fp32-accurate on the GPU and exact here; the rotations take each operand
as two bf16 planes, x ~ h + l with h = bf16(x), l = bf16(x - h), and form
the product from the three plane products h h' + h l' + l h' with wide
accumulation (stored intermediates are kept as h + l).  With both sides
present the two-sided products are taken left factor first:

    s1: Gb = bf16(G);  L = bs L + (1 - bs) Gb Gb^T   (L itself is not rounded)
    s2: Y = L Q_L (not rounded);  Q_L = qr(Y)
    s4: M' = p(s(p(Q_L^T, M)), Q_R);   G' = p(s(p(Q_L^T, G)), Q_R)
    s6: D  = p(s(p(Q_L, Dbar)), Q_R^T)
  where p(A, B) is the three-plane product and s(x) = h + l;
  one-sided: M' = p(Q_L^T, M), D = p(Q_L, Dbar) (left) or
             M' = p(M, Q_R),   D = p(Dbar, Q_R^T) (right);
  no side:   M' = M, G' = G, D = Dbar (plain AdamW).
"""

import numpy as np

from .bf16 import rnd
from .qr import qr_positive


def damping_of(F, damping):
    """The power step's damping d for factor F: 0 without damping (the
    pages' step); else damping * trace(F), or 1 when the trace is zero."""
    if damping == 0.0:
        return 0.0
    tr = float(np.trace(F))
    return damping * tr if tr != 0.0 else 1.0


def soap_step(W, G, M, V, L=None, QL=None, R=None, QR=None, *, t=1,
              lr=3e-3, beta1=0.95, beta2=0.95, shampoo_beta=None, eps=1e-8,
              weight_decay=0.0, bias_correction=True, precision="fp64",
              refresh=True, basis_refresh=True, damping=0.0):
    """One SOAP step.  Inputs are not modified; returns the new state.

    ``shampoo_beta`` defaults to ``beta2`` (one beta for both second-order
    statistics).  ``refresh=False`` skips steps 1-2 and uses the given bases
    as they are (for checks against an exact eigenbasis).
    ``basis_refresh=False`` still updates the factors (step 1) but keeps the
    bases (skips step 2): the steps between two refreshes of SOAP with a
    refresh interval f ("LLM Optimizers" guide, section 11.1: the bases are
    refreshed every f steps; "Matrix optimizers: K-FAC, Shampoo and Muon",
    SOAP step 3).
    ``damping`` is the optional relative damping of the power step (see
    above; 0, the default, is the pages' undamped step).
    """
    if precision not in ("fp64", "bf16"):
        raise ValueError(f"unknown precision {precision!r}")
    emu = precision == "bf16"
    r = rnd if emu else (lambda x: x)

    def split2(x):
        h = rnd(x)
        return h, rnd(x - h)

    def prod(A, B):
        # the three-plane product of the emulated rotations (exact in fp64)
        if not emu:
            return A @ B
        Ah, Al = split2(A)
        Bh, Bl = split2(B)
        return Ah @ Bh + Ah @ Bl + Al @ Bh

    def keep(x):
        if not emu:
            return x
        h, l = split2(x)
        return h + l
    f64 = lambda x: None if x is None else np.asarray(x, dtype=np.float64)
    W, G, M, V = f64(W), f64(G), f64(M), f64(V)
    L, QL, R, QR = f64(L), f64(QL), f64(R), f64(QR)
    left = QL is not None
    right = QR is not None
    bs = beta2 if shampoo_beta is None else shampoo_beta

    Gb = r(G)

    def power_step(F, Q):
        d = damping_of(F, damping)
        Y = F @ Q if d == 0.0 else (F + d * np.eye(F.shape[0])) @ Q
        return qr_positive(Y)[0]

    # 1-2. factor EMAs with the current gradient, then one power step + QR
    if refresh:
        if left:
            L = bs * L + (1.0 - bs) * (Gb @ Gb.T)
            if basis_refresh:
                QL = power_step(L, QL)
        if right:
            R = bs * R + (1.0 - bs) * (Gb.T @ Gb)
            if basis_refresh:
                QR = power_step(R, QR)
    # 3. first moment, original space
    M = beta1 * M + (1.0 - beta1) * G

    # 4. rotate into the basis
    def rotate_in(X):
        if left and right:
            return prod(keep(prod(QL.T, X)), QR)
        if left:
            return prod(QL.T, X)
        if right:
            return prod(X, QR)
        return X

    Mr = rotate_in(M)
    Gr = rotate_in(G)
    # 5. Adam in the basis
    V = beta2 * V + (1.0 - beta2) * Gr * Gr
    bc1 = 1.0 - beta1 ** t if bias_correction else 1.0
    bc2 = 1.0 - beta2 ** t if bias_correction else 1.0
    Dbar = (Mr / bc1) / (np.sqrt(V / bc2) + eps)
    # 6. rotate back
    if left and right:
        D = prod(keep(prod(QL, Dbar)), QR.T)
    elif left:
        D = prod(QL, Dbar)
    elif right:
        D = prod(Dbar, QR.T)
    else:
        D = Dbar
    # 7. decoupled weight decay and apply
    decayed = (1.0 - lr * weight_decay) * W
    W_new = decayed - lr * D
    return {"W": W_new, "M": M, "V": V, "L": L, "QL": QL, "R": R, "QR": QR,
            "Dbar": Dbar, "D": D, "dW": W_new - decayed, "Mr": Mr, "Gr": Gr}

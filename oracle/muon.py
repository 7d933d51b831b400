"""The Muon step for one matrix, in float64.

Steps, in the order of "Matrix optimizers: K-FAC, Shampoo and Muon", section
"Muon" (steps 1-4), with the momentum and Nesterov forms of "LLM Optimizers:
From SGD and AdamW to SOAP, Muon, and Scalable Training", section 11.3, and the
shape factors of its section 11.5:

    1. B_t   = beta B_{t-1} + G_t                (B_0 = 0)
       (option ``momentum_ema``: B_t = beta B_{t-1} + (1 - beta) G_t, the
        moving-average form of "Reading notes on SOAP, Muon, and Beyond",
        section 1; it only rescales B, which the normalisation removes)
    2. N_t   = G_t + beta B_t   (Nesterov)   or   N_t = B_t
    3. O_t   = NS_5(N_t)                     (see ``oracle.ns``)
    4. W_t   = (1 - lr wd) W_{t-1} - lr s O_t
       s = 0.2 sqrt(max(m, n))    ("match_rms_adamw", the default here)
       s = sqrt(max(1, m / n))    ("original")

``precision="bf16"`` runs step 3 with the GPU path's declared bf16 rounding
points (``oracle.ns.newton_schulz_bf16``); steps 1, 2 and 4 stay float64.
"""

import numpy as np

from .ns import QUINTIC, newton_schulz, newton_schulz_bf16


def shape_scale(m, n, adjust_lr="match_rms_adamw"):
    """Update scale s(m, n), section 11.5 of the LLM Optimizers guide."""
    if adjust_lr == "match_rms_adamw":
        return 0.2 * np.sqrt(max(m, n))
    if adjust_lr == "original":
        return np.sqrt(max(1.0, m / n))
    raise ValueError(f"unknown adjust_lr mode {adjust_lr!r}")


def muon_step(W, G, B, *, lr=0.02, weight_decay=0.01, momentum=0.95,
              nesterov=True, momentum_ema=False, ns_steps=5, coeffs=QUINTIC,
              eps=1e-7, adjust_lr="match_rms_adamw", precision="fp64"):
    """One Muon step.  Inputs are not modified.

    Returns a dict with the new weight ``W``, the new momentum ``B``, the
    orthogonalised update ``O`` and ``dW = W_new - (1 - lr wd) W_old``
    (the part of the change that the update, not the decay, causes).
    """
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    m, n = G.shape
    beta = momentum

    # 1. momentum
    if momentum_ema:
        B_new = beta * B + (1.0 - beta) * G
    else:
        B_new = beta * B + G
    # 2. Nesterov look-ahead
    N = G + beta * B_new if nesterov else B_new
    # 3. orthogonalise
    if precision == "fp64":
        O = newton_schulz(N, coeffs, ns_steps, eps)
    elif precision == "bf16":
        O = newton_schulz_bf16(N, coeffs, ns_steps, eps)
    else:
        raise ValueError(f"unknown precision {precision!r}")
    # 4. scaled update with decoupled weight decay
    s = shape_scale(m, n, adjust_lr)
    decayed = (1.0 - lr * weight_decay) * W
    W_new = decayed - lr * s * O
    return {"W": W_new, "B": B_new, "O": O, "N": N, "dW": W_new - decayed}

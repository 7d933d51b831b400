"""Newton-Schulz orthogonalisation toward the polar factor U V^T.

Definition followed ("LLM Optimizers: From SGD and AdamW to SOAP, Muon, and
Scalable Training", section 11.4, the displayed iteration; "Matrix optimizers:
K-FAC, Shampoo and Muon", Lemma 3 and the algorithm below it):

    X_0     = N / (||N||_F + eps)          (tall inputs are transposed first,
    A_k     = X_k X_k^T                     so that X X^T is the smaller Gram)
    X_{k+1} = a X_k + (b A_k + c A_k^2) X_k

with the quintic coefficients (a, b, c) = (3.4445, -4.7750, 2.0315) and five
iterations.  "Tall" means rows > cols; a square input is not transposed.

Two modes:

* ``newton_schulz`` - the iteration in float64, nothing rounded.
* ``newton_schulz_bf16`` - the same iteration with bfloat16 rounding at the
  points of a bf16-operand product chain (operands bf16, products
  accumulated wide, every stored matrix rounded to bf16 with ties-to-even):

      Nb  = bf16(N)                      (the cast happens before scaling, as
      s   = ||N||_F,  inv = 1/(s + eps)   in the pages' reference code; the
                                          scale is applied exactly in the
                                          first iteration instead of being
                                          rounded into a bf16 X_0)
      iteration 0:  A = bf16(inv^2 * Nb Nb^T)
                    P = bf16(b A + c A A)
                    X = bf16(a inv Nb + inv (P Nb))
      iteration k>0: A = bf16(X X^T);  P = bf16(b A + c A A);
                     X = bf16(a X + P X)

  In exact arithmetic both modes compute the same X_k (X_0 = inv * Nb when
  Nb = N); the emulation gives the noise floor that a bf16 path's result is
  held to.  (A path may round at other points with the same iteration, e.g.
  store bf16(a I + b A + c A A) and form X = bf16(P X); its error is then
  held to this same floor.)
"""

import numpy as np

from .bf16 import rnd

QUINTIC = (3.4445, -4.7750, 2.0315)   # section 11.4 equation; Lemma 3 text
CUBIC = (1.5, -0.5, 0.0)              # classical cubic iteration, Lemma 3 text


def _orient(N):
    tall = N.shape[0] > N.shape[1]
    return (N.T if tall else N), tall


def newton_schulz(N, coeffs=QUINTIC, steps=5, eps=1e-7):
    """Float64 Newton-Schulz: returns X_steps with the input's shape."""
    a, b, c = coeffs
    X, tall = _orient(np.asarray(N, dtype=np.float64))
    X = X / (np.linalg.norm(X) + eps)          # Frobenius norm
    for _ in range(steps):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.T if tall else X


def newton_schulz_bf16(N, coeffs=QUINTIC, steps=5, eps=1e-7):
    """Newton-Schulz with the GPU path's declared bf16 rounding points.

    ``N`` holds the float32 values the GPU receives (upcast exactly).  The
    result holds bfloat16 values (as float64) with the input's shape.
    """
    a, b, c = coeffs
    Xin, tall = _orient(np.asarray(N, dtype=np.float64))
    s = np.linalg.norm(Xin)
    inv = 1.0 / (s + eps)
    Nb = rnd(Xin)
    X = None
    for k in range(steps):
        if k == 0:
            A = rnd(inv * inv * (Nb @ Nb.T))
            P = rnd(b * A + c * (A @ A))
            X = rnd(a * inv * Nb + inv * (P @ Nb))
        else:
            A = rnd(X @ X.T)
            P = rnd(b * A + c * (A @ A))
            X = rnd(a * X + P @ X)
    if steps == 0:
        X = rnd(inv * Nb)
    return X.T if tall else X


def scalar_map(sigma, coeffs=QUINTIC, steps=5):
    """The odd polynomial phi(s) = a s + b s^3 + c s^5 applied ``steps`` times.

    By Lemma 3 this is what the iteration does to each singular value of the
    normalised input.
    """
    a, b, c = coeffs
    s = np.asarray(sigma, dtype=np.float64)
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s

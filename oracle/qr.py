"""QR factorisation with the positive-diagonal convention.

The SOAP basis refresh takes ``Q <- qr(L Q)`` (one power-iteration step
followed by QR: "Reading notes on SOAP, Muon, and Beyond", section 4;
"初探优化器（一）", section 6.2 step 2).  The pages do not fix a sign
convention; we use the one that makes the thin QR of a full-rank matrix
unique: every diagonal entry of R is non-negative, so Q's columns are the
Gram-Schmidt orthonormalisation of Y's columns taken in order.

The factorisation itself is LAPACK's Householder QR (``numpy.linalg.qr``), a
library primitive used as one step; only the sign fix is ours.
"""

import numpy as np


def qr_positive(Y):
    """Return (Q, R) with Y = Q R, Q^T Q = I and diag(R) >= 0."""
    Y = np.asarray(Y, dtype=np.float64)
    Q, R = np.linalg.qr(Y, mode="reduced")
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    Q = Q * d[None, :]
    R = R * d[:, None]
    return Q, R

"""Exact round-to-nearest-even rounding of float64 values to bfloat16.

bfloat16 keeps float32's 8-bit exponent and 8 significant bits (7 stored + the
implicit one).  The emulation modes of the oracle call ``rnd`` at exactly the
points where the GPU path declares a bf16 rounding; everything between two
rounding points is carried in float64.  The rounding is done in one step from
float64 (no detour through float32, which would round twice).

Pinned in ``tests/test_oracle_bf16.py`` against hand-derived bit patterns and
against the IEEE definition (ties to even, subnormals, overflow to inf).
"""

import numpy as np

# bfloat16 constants from the format's definition (IEEE-754 binary32 exponent
# range, 8-bit significand).
_P = 8                      # significand bits, implicit one included
_EMIN = -126                # smallest normal exponent
_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127   # largest finite bfloat16


def rnd(x):
    """Round every element of ``x`` to the nearest bfloat16 (ties to even).

    Returns a float64 array holding bfloat16-representable values.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    finite = np.isfinite(x)
    out[~finite] = x[~finite]
    xf = x[finite]
    ax = np.abs(xf)
    # exponent e with 2**e <= |x| < 2**(e+1); zero handled separately
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    # guard against log2 rounding at exact powers of two
    e = np.where(2.0 ** e > ax, e - 1, e)
    e = np.where(2.0 ** (e + 1) <= ax, e + 1, e)
    e = np.maximum(e, _EMIN)            # below the normal range: fixed quantum
    quantum = 2.0 ** (e - (_P - 1))     # spacing of bfloat16 values near x
    q = np.rint(xf / quantum) * quantum  # np.rint rounds half to even
    q = np.where(ax == 0, xf, q)        # keep signed zeros
    q = np.where(np.abs(q) > _MAX, np.copysign(np.inf, q), q)
    out[finite] = q
    return out


def rnd32(x):
    """Round float64 values to float32 (ties to even) and return float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)

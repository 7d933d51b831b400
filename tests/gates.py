"""Comparison gates shared by the parity tests (test-side helpers only)."""
import numpy as np


def rel(a, b):
    """Relative Frobenius error ||a - b|| / ||b||."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def ns_gate(N, O_gpu, O_ref, O_emu, *, tau=1e-2, sub_tol=2e-2, band=(0.6, 1.3), floor=1.25,
            floor_abs=2e-3, svd=None, fro=None):
    """Newton-Schulz parity on the resolved subspace plus a noise-floor gate.

    The iteration multiplies near-null singular directions by up to a^5, so
    bf16 rounding noise there is amplified whatever the kernel; the check is
    (1) on the singular subspace with sigma / ||N||_F >= tau: relative error
        of U_k^T O V_k against the fp64 oracle <= sub_tol (or, where the
        oracle's bf16 emulation is itself further off, <= floor times the
        emulation's error) and its singular values inside ``band``;
    (2) on the full matrix: the GPU's error against fp64 is no worse than
        ``floor`` times the oracle's own bf16-emulation error (+ floor_abs).
    ``svd`` may hold only the leading singular triplets of N (every
    resolved one among them); ``fro`` is then N's Frobenius norm, against
    which tau is taken (default: the norm of the given singular values).
    Returns a dict of the measured numbers (asserts inside).
    """
    N = np.asarray(N, dtype=np.float64)
    tall = N.shape[0] > N.shape[1]
    if svd is None:
        U, s, Vt = np.linalg.svd(N, full_matrices=False)
    else:
        U, s, Vt = svd
    k = int(np.sum(s / (np.linalg.norm(s) if fro is None else fro) >= tau))
    assert k < len(s) or svd is None or fro is None, "the given triplets may not hold every resolved one"
    Uk, Vk = U[:, :k], Vt[:k].T
    P = lambda O: Uk.T @ np.asarray(O, dtype=np.float64) @ Vk
    sub = rel(P(O_gpu), P(O_ref))
    sv = np.linalg.svd(P(O_gpu), compute_uv=False)
    full_gpu = rel(O_gpu, O_ref)
    full_emu = rel(O_emu, O_ref)
    sub_emu = rel(P(O_emu), P(O_ref))
    out = dict(k=k, sub=sub, sub_emu=sub_emu, sv_min=float(sv.min()), sv_max=float(sv.max()), full_gpu=full_gpu,
               full_emu=full_emu, tall=tall)
    # the bf16 noise floor applies on the subspace too: on tiny matrices the
    # emulation of the declared rounding itself can sit at the tolerance
    assert sub <= max(sub_tol, floor * sub_emu), out
    if band is not None:
        assert band[0] <= sv.min() and sv.max() <= band[1], out
    assert full_gpu <= floor * full_emu + floor_abs, out
    return out


def basis_gate(Q, F, Q_old, *, tau=1e-3, c_kappa=5e-7, c_r=2e-5, c0=1e-5, orth=1e-4):
    """A refreshed basis Q (GPU) against the positive-diagonal QR of the power
    product Y = F Q_old (fp64 oracle).

    Two things limit how well fp32-level arithmetic determines column j:
      - the power product: y_j = F q_j is computed with an error of about u
        ||F|| ||q_j||, i.e. a relative error u kappa_j with kappa_j =
        ||F||_2 / ||y_j|| (columns in F's small-eigenvalue directions cancel
        against the large ones);
      - the QR: column j of Q depends on y_j's part outside the span of the
        columns before it, r_j = R_jj / ||y_j||, to about u / r_j.
    Columns with r_j >= tau are "resolved" and must agree within
    c_kappa kappa_j + c_r / r_j + c0; for the others (a singular or nearly
    singular factor: a cold start, a rank-deficient gradient) any
    orthonormal completion is a valid QR, so only orthonormality is checked.
    Returns (resolved mask, per-column errors)."""
    from scipy.linalg import eigh
    from oracle.qr import qr_positive
    Q = np.asarray(Q, dtype=np.float64)
    F = np.asarray(F, dtype=np.float64)
    Y = F @ np.asarray(Q_old, dtype=np.float64)
    dev = float(np.abs(Q.T @ Q - np.eye(Q.shape[1])).max())
    assert dev <= orth, dict(orthonormality=dev)
    Qr, R = qr_positive(Y)
    k = F.shape[0]
    norm_f = float(np.abs(eigh((F + F.T) / 2, eigvals_only=True, subset_by_index=[k - 1, k - 1])[0]))
    with np.errstate(divide="ignore", invalid="ignore"):
        ny = np.linalg.norm(Y, axis=0)
        r = np.abs(np.diag(R)) / ny
        kappa = norm_f / ny
    sel = r >= tau
    err = np.linalg.norm(Q - Qr, axis=0)
    bound = c_kappa * np.where(sel, kappa, 0.0) + c_r / np.where(sel, r, 1.0) + c0
    bad = np.nonzero(sel & (err > bound))[0]
    assert bad.size == 0, dict(columns=bad[:8].tolist(), err=err[bad[:8]].tolist(), r=r[bad[:8]].tolist(),
                               kappa=kappa[bad[:8]].tolist())
    return sel, err

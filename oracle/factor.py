"""Oracle: damping and the upper Cholesky factor of the inverse Hessian (test infrastructure only).

Sources
  * hncyxsy.com/news/243429 §3.1 step 1 and §3.3: a damping term λ on the diagonal keeps H
    invertible; damp_percent is a ratio on the Hessian diagonal, default 0.01 (raise to 0.1
    when calibration is unstable).
  * gtnt.cn/news/115337 §4: perc_damp, default 0.01, diagonal damping against a singular H.
  * hncyxsy.com/news/243429 §2.4 and §3.1 step 2: use a Cholesky factorisation instead of
    repeated inversion, and drive the column updates from the factor.

Reading: λ = percdamp · mean(diag H), added to every diagonal entry. The factor the column
loop consumes is the upper-triangular U with UᵀU = H_d⁻¹ (row q of U, divided by U_qq, is the
row of the inverse Hessian restricted to the not-yet-quantized columns q, q+1, …).

``upper_chol_of_inverse`` takes the textbook route (Cholesky of H_d, explicit inverse, Cholesky
of the inverse). ``upper_chol_of_inverse_reversed`` takes the one-factorisation route through
the index reversal P: U = P·chol_lower(P H_d P)⁻¹·P. The tests check that the two agree.
"""

import numpy as np
import scipy.linalg


class NotPositiveDefinite(ArithmeticError):
    pass


def damping(H, percdamp):
    """λ = percdamp · mean(diag H); NotPositiveDefinite unless it is positive and finite."""
    H = np.asarray(H, dtype=np.float64)
    lam = float(percdamp) * float(np.mean(np.diag(H)))
    if not np.isfinite(lam) or lam <= 0.0:
        raise NotPositiveDefinite(f"damping term lambda={lam!r} is not positive")
    return lam


def damp(H, percdamp):
    """Return (H + λI, λ) with λ = percdamp · mean(diag H) (λ added to each diagonal entry)."""
    H = np.asarray(H, dtype=np.float64)
    lam = damping(H, percdamp)
    Hd = H.copy()
    Hd[np.diag_indices(H.shape[0])] += lam
    return Hd, lam


def _cholesky_lower(A):
    """L lower triangular with A = L Lᵀ (LAPACK potrf); NotPositiveDefinite otherwise."""
    try:
        return scipy.linalg.cholesky(A, lower=True, check_finite=False)
    except np.linalg.LinAlgError as exc:
        raise NotPositiveDefinite(str(exc)) from exc


def _inverse_lower(L):
    """L⁻¹ for a lower-triangular L (LAPACK trtri)."""
    Linv, info = scipy.linalg.lapack.dtrtri(L, lower=1)
    if info != 0:
        raise NotPositiveDefinite(f"singular triangular factor (info={info})")
    return np.tril(Linv)


def upper_chol_of_inverse(Hd):
    """U upper triangular with UᵀU = Hd⁻¹, by Cholesky → explicit inverse → Cholesky."""
    Hd = np.asarray(Hd, dtype=np.float64)
    L = _cholesky_lower(Hd)
    Linv = _inverse_lower(L)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    C = _cholesky_lower(Hinv)             # Hinv = C Cᵀ, C lower
    return C.T                            # U = Cᵀ: UᵀU = C Cᵀ


def upper_chol_of_inverse_reversed(Hd):
    """U = P · L⁻¹ · P with P H_d P = L Lᵀ and P the index reversal."""
    Hd = np.asarray(Hd, dtype=np.float64)
    L = _cholesky_lower(np.ascontiguousarray(Hd[::-1, ::-1]))
    return _inverse_lower(L)[::-1, ::-1].copy()

"""Oracle: the calibration Hessian H = 2·XᵀX (test infrastructure only).

Sources
  * hncyxsy.com/news/243429 §3.1 step 1: from the layer's input activations X, form
    H = 2XXᵀ + λI (the "+" is lost in the page's text; λ is the damping term, applied later
    in ``factor.damp``). The page writes X with tokens as columns; here X is stored
    tokens × channels, so the same matrix reads 2·XᵀX.
  * gtnt.cn/news/115337 §4: collect each layer's Hessian from calibration forward passes.

The sum runs over all tokens, unnormalised (GPTQ's result is invariant to a positive scale of
H because the damping is relative to mean(diag H)). Accumulation is additive over calls.
"""

import numpy as np
import scipy.linalg


def hessian(X, chunk=8192):
    """H = 2·Σ_t x_t x_tᵀ in fp64 for X of shape [n_tokens, d_in] (any float dtype).

    Each chunk of tokens is added with the BLAS symmetric rank-k update (one triangle of
    XᵀX, the other is its mirror), accumulated in fp64."""
    X = np.asarray(X)
    n, d = X.shape
    S = np.zeros((d, d), dtype=np.float64, order="F")
    for t0 in range(0, n, chunk):
        Xc = X[t0:t0 + chunk].astype(np.float64)
        # S (upper triangle) += Xcᵀ·Xc; Xc.T is a Fortran-ordered d x chunk view
        S = scipy.linalg.blas.dsyrk(1.0, Xc.T, beta=1.0, c=S, trans=0, lower=0,
                                    overwrite_c=1)
    H = S + S.T                           # the lower triangle of S is zero
    H[np.diag_indices(d)] -= np.diag(S)   # the diagonal was counted twice (exact)
    return 2.0 * H


def hessian_entries(X, rows, cols):
    """H[rows][:, cols] only, for sampled parity checks of large Hessians."""
    X = np.asarray(X)
    Xr = X[:, rows].astype(np.float64)
    Xc = X[:, cols].astype(np.float64)
    return 2.0 * (Xr.T @ Xc)

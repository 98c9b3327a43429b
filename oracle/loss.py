"""Oracle: layer reconstruction loss (test infrastructure only).

Sources
  * 0539edu.com/news/6111416 §3.1: GPTQ minimises ‖WX − W_qX‖² for the layer.
  * hncyxsy.com/news/243429 §2.1–2.2: the second-order term δᵀHδ with H the Hessian of that
    objective.

With H = 2·XᵀX (undamped) and Δ = W − Ŵ, tr(ΔHΔᵀ) = 2‖ΔXᵀ‖²_F, so the ratio
tr(ΔHΔᵀ)/tr(WHWᵀ) equals ‖(W − Ŵ)Xᵀ‖²_F / ‖WXᵀ‖²_F.
"""

import numpy as np


def recon_loss(W, What, H):
    """tr(ΔHΔᵀ)/tr(WHWᵀ) in fp64."""
    W = np.asarray(W, dtype=np.float64)
    D = W - np.asarray(What, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    num = np.einsum("ij,ij->", D @ H, D)
    den = np.einsum("ij,ij->", W @ H, W)
    return num / den


def recon_loss_from_x(W, What, X):
    """‖(W − Ŵ)Xᵀ‖²_F / ‖WXᵀ‖²_F computed directly from the activations."""
    W = np.asarray(W, dtype=np.float64)
    Xf = np.asarray(X, dtype=np.float64)
    D = W - np.asarray(What, dtype=np.float64)
    return np.sum((D @ Xf.T) ** 2) / np.sum((W @ Xf.T) ** 2)

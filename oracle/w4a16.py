"""Oracle: the W4A16 layer that consumes GPTQ's output (test infrastructure only).

Sources
  * 0539edu.com/news/6111416 §3.2 and §5.2: a GPTQ/AWQ INT4 checkpoint is served as 4-bit
    weights with fp16 activations; at run time the codes are expanded with their group's scale
    and zero point and multiplied with the fp16 activations.
  * hncyxsy.com/news/243429 §3.3: with desc_act (act_order) the columns were quantized in another
    order, so inference needs the group index of every column (g_idx) to find its scale and
    zero.
  * 0539edu.com §2.1 and §4.2: ŵ = scale·(q − zero) with one fp16 scale and zero per group.

Reading: the reconstructed weight is held in fp16, as the weights of a W4A16 layer are,
Ŵ16[r][c] = fp16(s[r][k]·(q[r][c] − z[r][k])), k = g_idx[c] (one rounding of the exact
product), and the layer computes Y = X·Ŵ16ᵀ (+ R, a residual input) exactly in fp64 before one
rounding to fp16: Y16 = fp16(X·Ŵ16ᵀ + R). X, R and Y are [tokens × features] (PyTorch Linear
layout); codes are [d_out × d_in] in the original column order.
"""

import numpy as np


def dequant_fp16(codes, scales, zeros, g_idx):
    """Ŵ16 [d_out, d_in] as fp64 values: fp16(s·(q − z)) with each column's group from g_idx."""
    g_idx = np.asarray(g_idx, dtype=np.int64)
    s = np.asarray(scales, np.float64)[:, g_idx]
    z = np.asarray(zeros, np.float64)[:, g_idx]
    exact = s * (np.asarray(codes, np.float64) - z)      # exact: 11-bit scale x 9-bit integer
    return exact.astype(np.float16).astype(np.float64)


def w4a16_linear(X, codes, scales, zeros, g_idx, R=None):
    """Y16 = fp16(X·Ŵ16ᵀ + R) in fp64 before the final rounding; returned as fp64 values."""
    Wh = dequant_fp16(codes, scales, zeros, g_idx)
    Y = np.asarray(X, np.float64) @ Wh.T
    if R is not None:
        Y = Y + np.asarray(R, np.float64)
    return Y.astype(np.float16).astype(np.float64), Y


def abs_products(X, codes, scales, zeros, g_idx):
    """Σ_k |x_k·ŵ_k| per output (the scale of the accumulation error of the sum)."""
    Wh = dequant_fp16(codes, scales, zeros, g_idx)
    return np.abs(np.asarray(X, np.float64)) @ np.abs(Wh).T

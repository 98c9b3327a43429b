"""Oracle: AWQ-lite activation-aware channel scaling, a grid search over α (test
infrastructure only).

Sources
  * gtnt.cn/news/115337 §3 (awq_lite): the input channels get a scale s, the weights the same
    scale the other way, which leaves the output unchanged and moves the rounding error; α is
    searched in [0, 1] with step alpha_step (default 0.1), by the MSE of the scaled output
    against the true output; s = x_max^α / w_max^(1−α), with x_max and w_max the per-channel
    mean absolute values of the activations and of the weights.
  * 0539edu.com/news/6111416 §3.2: channels with large activations carry the important
    weights; scaling them up before quantization protects them.

Readings:
  * Direction: the weights of channel c are multiplied by s_c and its activations divided by
    it (the page's sentence names the two the other way round, which would shrink the
    important weights and enlarge their relative rounding error, the opposite of the stated
    purpose). The layer then computes (X/s)·Q(W·s)ᵀ = X·(Q(W·s)/s)ᵀ.
  * x_max_c = mean over tokens of |x_tc|; w_max_c = mean over output rows of |w_rc|.
  * s is held in fp16 (it is folded into the preceding layer, whose weights are fp16):
    s_c = fp16(x_max_c^α / w_max_c^(1−α)), and 1 where that is not a positive finite fp16
    value or where x_max_c or w_max_c is 0.
  * The quantizer is the group min-max RTN of ``rtn`` applied to W·s (exact: an fp16 weight
    times an fp16 scale), and the criterion is the layer's output error for the calibration
    activations, ‖(W − Q(W·s)/s)·Xᵀ‖² = tr(ΔHΔᵀ)/2 with H = 2XᵀX; the smallest wins, ties to the
    smaller α.
"""

import numpy as np

from . import rtn


def channel_mean_abs(X):
    """Per input channel, the mean over tokens of |x| (fp64)."""
    X = np.asarray(X)
    return np.mean(np.abs(X.astype(np.float64)), axis=0)


def awq_scales(x_mean, w_mean, alpha):
    """s_c = fp16(x_mean^α / w_mean^(1−α)) as fp64 values; 1 where degenerate."""
    x_mean = np.asarray(x_mean, np.float64)
    w_mean = np.asarray(w_mean, np.float64)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        s = np.power(x_mean, alpha) / np.power(w_mean, 1.0 - alpha)
        s16 = s.astype(np.float16).astype(np.float64)
    ok = (x_mean > 0) & (w_mean > 0) & np.isfinite(s16) & (s16 > 0)
    return np.where(ok, s16, 1.0)


def alpha_grid(alpha_step=0.1):
    """α = i·alpha_step for i = 0 … round(1/alpha_step) (0, 0.1, …, 1.0 by default)."""
    n = int(round(1.0 / alpha_step)) + 1
    return np.array([i * alpha_step for i in range(n)])


def awq_lite(W, x_mean, H, bits, group_size, alpha_step=0.1, sym=False):
    """Grid search of α. W [d_out, d_in] (fp16 values), x_mean [d_in], H = 2XᵀX [d_in, d_in].

    Returns dict(best (index), alpha, s [d_in], codes, scales, zeros (RTN of W·s),
    losses [grid] = tr(ΔHΔᵀ) per α)."""
    W = np.asarray(W, np.float64)
    H = np.asarray(H, np.float64)
    w_mean = np.mean(np.abs(W), axis=0)
    alphas = alpha_grid(alpha_step)
    losses = np.empty(len(alphas))
    cands = []
    for i, a in enumerate(alphas):
        s = awq_scales(x_mean, w_mean, a)
        codes, scales, zeros = rtn.rtn_minmax(W * s[None, :], bits, group_size, sym=sym)
        D = W - rtn.rtn_dequant(codes, scales, zeros, group_size) / s[None, :]
        losses[i] = np.einsum("ij,ij->", D @ H, D)
        cands.append((s, codes, scales, zeros))
    best = int(np.argmin(losses))
    s, codes, scales, zeros = cands[best]
    return dict(best=best, alpha=alphas[best], s=s, codes=codes, scales=scales, zeros=zeros,
                losses=losses)

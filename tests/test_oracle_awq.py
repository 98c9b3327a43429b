"""Pins for the AWQ-lite oracle.

* The grid is 0, 0.1, …, 1.0 (gtnt.cn §3's default alpha_step).
* Closed forms at the ends of the grid: α = 0 gives s = fp16(1/w_max), α = 1 gives
  s = fp16(x_max); degenerate channels get 1.
* The criterion of every α equals the layer's output error computed from the activations,
  2·‖(W − Q(W·s)/s)·Xᵀ‖² (the folded layer (X/s)·Q(W·s)ᵀ evaluated directly), and the choice is
  the brute-force argmin.
* On activations with outlier channels the search beats plain RTN (s = 1), as the pages claim.
"""

import numpy as np
import pytest

from oracle import awq, hessian, loss, rtn
from post_weight_quantization_24_b200 import workloads


def _case(seed=0, d_out=48, d_in=128, n=1024):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_out=d_out, d_in=d_in, n_tokens=n, seed=seed)
    W = workloads.make_weights(wl).float().numpy().astype(np.float64)
    X = workloads.make_activations(wl).numpy()
    return W, X


def test_grid_and_channel_means():
    assert np.allclose(awq.alpha_grid(), np.arange(11) / 10, rtol=0, atol=1e-15)
    X = np.array([[1.0, -2.0], [-3.0, 0.5]], dtype=np.float16)
    assert np.array_equal(awq.channel_mean_abs(X), [2.0, 1.25])


def test_scales_at_the_ends_of_the_grid():
    x = np.array([0.5, 3.0, 0.0, 7.0])
    w = np.array([0.02, 0.01, 0.03, 0.0])
    s0 = awq.awq_scales(x, w, 0.0)
    s1 = awq.awq_scales(x, w, 1.0)
    assert s0[0] == np.float16(1 / 0.02) and s0[1] == np.float16(1 / 0.01)
    assert s1[0] == np.float16(0.5) and s1[1] == np.float16(3.0)
    assert s0[2] == 1.0 and s1[3] == 1.0          # x_max or w_max zero


def test_criterion_is_the_folded_layer_output_error_and_choice_is_argmin():
    W, X = _case()
    H = hessian.hessian(X)
    x_mean = awq.channel_mean_abs(X)
    res = awq.awq_lite(W, x_mean, H, 4, 32)
    Xf = X.astype(np.float64)
    w_mean = np.mean(np.abs(W), axis=0)
    direct = []
    for a in awq.alpha_grid():
        s = awq.awq_scales(x_mean, w_mean, a)
        c, sc, z = rtn.rtn_minmax(W * s, 4, 32)
        Qs = rtn.rtn_dequant(c, sc, z, 32)
        Y_true = Xf @ W.T
        Y_folded = (Xf / s) @ Qs.T                 # (X/s)·Q(W·s)ᵀ
        direct.append(2.0 * np.sum((Y_true - Y_folded) ** 2))
    assert np.allclose(res["losses"], direct, rtol=1e-9, atol=0)
    assert res["best"] == int(np.argmin(direct))
    assert res["alpha"] == pytest.approx(awq.alpha_grid()[res["best"]])


def test_search_beats_plain_rtn_on_outlier_channels():
    W, X = _case(seed=3, d_out=64, d_in=256, n=2048)
    H = hessian.hessian(X)
    res = awq.awq_lite(W, awq.channel_mean_abs(X), H, 3, 64)
    c, s, z = rtn.rtn_minmax(W, 3, 64)
    # tr(ΔHΔᵀ) of plain RTN (s = 1): the relative loss times tr(WHWᵀ)
    rtn_loss = loss.recon_loss(W, rtn.rtn_dequant(c, s, z, 64), H) * np.einsum("ij,ij->", W @ H, W)
    assert res["losses"][res["best"]] < rtn_loss

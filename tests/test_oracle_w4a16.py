"""Pins for the W4A16 oracle (the layer that consumes GPTQ's output).

* Ŵ16 is the fp16 rounding of the fp64 reconstruction: within half an fp16 ulp of it, and
  exactly it whenever that value is representable.
* Y = X·Ŵ16ᵀ (+ R) equals a plain triple loop on a tiny case, and Y16 is its fp16 rounding.
* Reordering the input dimension (the act_order gather of GPTQ deep-dive §3.3): permuting
  the columns of X, of the codes and of g_idx together leaves Y unchanged.
* The layer applied to the GPTQ result reproduces the oracle's reconstruction loss: with
  H = 2XᵀX, ‖(W − Ŵ)Xᵀ‖² computed from the layer's outputs equals tr(ΔHΔᵀ)/2.
"""

import numpy as np

from oracle import gptq, hessian, loss, rtn, w4a16


def _layer(seed, d_out=24, d_in=64, g=16, bits=4):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16).astype(np.float64)
    codes, scales, zeros = rtn.rtn_minmax(W, bits, g)
    return W, codes, scales, zeros, np.arange(d_in) // g


def test_dequant_is_fp16_rounding_of_the_reconstruction():
    W, codes, scales, zeros, g_idx = _layer(0)
    Wh = w4a16.dequant_fp16(codes, scales, zeros, g_idx)
    exact = rtn.rtn_dequant(codes, scales, zeros, 16)
    ulp = np.abs(np.spacing(exact.astype(np.float16)).astype(np.float64))
    assert np.all(np.abs(Wh - exact) <= ulp / 2)
    representable = exact.astype(np.float16).astype(np.float64) == exact
    assert np.array_equal(Wh[representable], exact[representable])


def test_linear_equals_triple_loop():
    W, codes, scales, zeros, g_idx = _layer(1, d_out=5, d_in=32, g=8)
    rng = np.random.default_rng(2)
    X = rng.standard_normal((7, 32)).astype(np.float16)
    R = rng.standard_normal((7, 5)).astype(np.float16)
    Y16, Y = w4a16.w4a16_linear(X, codes, scales, zeros, g_idx, R=R)
    for t in range(7):
        for r in range(5):
            acc = float(R[t, r])
            for c in range(32):
                k = g_idx[c]
                wh = float(np.float16(scales[r, k] * (codes[r, c] - zeros[r, k])))
                acc += float(X[t, c]) * wh
            assert abs(Y[t, r] - acc) <= 1e-12 * max(1.0, abs(acc))
            assert Y16[t, r] == float(np.float16(Y[t, r]))


def test_input_order_does_not_matter():
    """The act_order gather: codes reordered to the processing order, X gathered the same way,
    g_idx carried along; the layer's output is unchanged."""
    d_in, g = 64, 16
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((9, d_in)) * np.exp(rng.standard_normal(d_in))).astype(np.float16)
    H = hessian.hessian(X)
    W = (rng.standard_normal((12, d_in)) * 0.02).astype(np.float16).astype(np.float64)
    out = gptq.gptq_blocked_ref(W, H, 4, g, 32, act_order=True)
    perm = out["perm"]
    _, Y = w4a16.w4a16_linear(X, out["codes"], out["scales"], out["zeros"], out["g_idx"])
    _, Yp = w4a16.w4a16_linear(X[:, perm], out["codes"][:, perm], out["scales"],
                               out["zeros"], out["g_idx"][perm])
    assert np.allclose(Y, Yp, rtol=1e-12, atol=1e-12)
    # in the processing order the groups are contiguous: g_idx[perm] = p // g
    assert np.array_equal(out["g_idx"][perm], np.arange(d_in) // g)


def test_layer_output_gives_the_reconstruction_loss():
    rng = np.random.default_rng(4)
    X = (rng.standard_normal((200, 32)) * np.exp(0.5 * rng.standard_normal(32))).astype(np.float16)
    H = hessian.hessian(X)
    W = (rng.standard_normal((10, 32)) * 0.02).astype(np.float16).astype(np.float64)
    out = gptq.gptq_blocked_ref(W, H, 4, 8, 16)
    _, Y = w4a16.w4a16_linear(X, out["codes"], out["scales"], out["zeros"], out["g_idx"])
    Y_fp = X.astype(np.float64) @ W.T
    # Ŵ16 differs from the fp64 reconstruction by fp16 rounding only; compare in the loss
    num = np.sum((Y_fp - Y) ** 2)
    den = np.sum(Y_fp ** 2)
    assert abs(num / den - loss.recon_loss(W, out["What"], H)) <= 1e-3 * loss.recon_loss(W, out["What"], H)

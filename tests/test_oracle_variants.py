"""Pins for the oracle's quantizer variants: symmetric quantizer, per-channel groups, static
groups under act_order, and the clip search.

* Symmetric (0539edu.com §2.3, q = round(x/scale) with the zero point fixed at 0): the signed
  code is the page's rint(x/scale), every code is the nearest level of the symmetric grid
  (brute force), |w - ŵ| <= scale/2, and GPTQ with H = c·I reduces to symmetric RTN.
* Per-channel (one group per row): GPTQ with H = c·I is RTN with group_size = d_in, and the
  blocked reference equals the unblocked one for block sizes that do not divide into groups.
* Static groups: the scales come from the original weights in the original order, so with
  H = c·I GPTQ under act_order is plain RTN of the original groups, g_idx[c] = c // g; blocked
  equals unblocked; and the least-squares re-solve rebuilds every code from the fixed grid.
* Clip search (gtnt.cn §3): the grid runs from amax down to amax·0.5 in steps of 0.05; one
  grid point is plain RTN; the choice is the brute-force argmin; the H criterion equals the
  group's output error computed from the activations; clipping never loses to no clipping.
"""

import numpy as np
import pytest

from oracle import factor, gptq, hessian, quantizer, rtn
from post_weight_quantization_24_b200 import workloads


def _weights(d_out, d_in, seed):
    rng = np.random.default_rng(300 + seed)
    W = rng.standard_normal((d_out, d_in)) * 0.02
    W[:, rng.choice(d_in, max(1, d_in // 50), replace=False)] *= 20   # outlier columns
    return W.astype(np.float16).astype(np.float64)


def _x(n, d, seed, correlated=True):
    if correlated:
        return workloads.correlated_activations(n, d, rank=3, seed=seed).numpy()
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))).astype(np.float16)


# ---------------------------------------------------------------- symmetric quantizer -------
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_symmetric_codes_are_the_pages_rounding_and_nearest_level(bits):
    maxq = 2 ** bits - 1
    rng = np.random.default_rng(bits)
    w = rng.standard_normal((300, 16)) * np.exp(rng.standard_normal((300, 1)))
    s, z = quantizer.group_params_sym(w.min(1), w.max(1), maxq)
    assert np.all(z == 2 ** (bits - 1))
    q = quantizer.quantize(w, s[:, None], z[:, None], maxq)
    # the signed code is rint(x / scale) (the page's formula), clamped to the signed range
    signed = np.clip(np.rint(w / s[:, None]), -2 ** (bits - 1), 2 ** (bits - 1) - 1)
    assert np.array_equal(q - 2 ** (bits - 1), signed)
    wh = quantizer.dequantize(q, s[:, None], z[:, None])
    assert np.all(np.abs(w - wh) <= s[:, None] / 2)
    # brute force: no level of the symmetric grid is closer
    levels = s[:, None, None] * (np.arange(maxq + 1)[None, None, :] - 2 ** (bits - 1))
    best = np.min(np.abs(w[:, :, None] - levels), axis=2)
    assert np.allclose(np.abs(w - wh), best, rtol=0, atol=1e-15)
    # scale = 2m/maxq rounded up to fp16, m the largest magnitude
    m = np.max(np.abs(w), axis=1)
    assert np.array_equal(s, quantizer.fp16_round_up(2 * m / maxq))


def test_symmetric_all_zero_group():
    s, z = quantizer.group_params_sym(np.array([0.0]), np.array([0.0]), 15)
    assert s[0] == 1.0 and z[0] == 8


@pytest.mark.parametrize("act_order", [False, True])
def test_symmetric_gptq_identity_hessian_is_symmetric_rtn(act_order):
    W = _weights(20, 64, 0)
    H = 2.5 * np.eye(64)
    codes, scales, zeros = rtn.rtn_minmax(W, 4, 16, sym=True)
    for out in (gptq.gptq_blocked_ref(W, H, 4, 16, 32, act_order=act_order, sym=True),
                gptq.gptq_obs_ref(W, H, 4, 16, act_order=act_order, sym=True)):
        assert np.array_equal(out["codes"], codes)
        assert np.array_equal(out["scales"], scales) and np.array_equal(out["zeros"], zeros)


@pytest.mark.parametrize("static_groups", [False, True])
def test_symmetric_blocked_equals_unblocked(static_groups):
    H = hessian.hessian(_x(400, 64, 3))
    W = _weights(18, 64, 1)
    ref = gptq.gptq_obs_ref(W, H, 3, 16, act_order=True, sym=True, static_groups=static_groups)
    for B in (16, 32, 64):
        out = gptq.gptq_blocked_ref(W, H, 3, 16, B, act_order=True, sym=True,
                                    static_groups=static_groups)
        assert np.array_equal(out["codes"], ref["codes"])
        assert np.array_equal(out["scales"], ref["scales"])


# ---------------------------------------------------------------- per-channel ---------------
@pytest.mark.parametrize("sym", [False, True])
def test_per_channel_identity_hessian_is_rtn_of_the_row(sym):
    W = _weights(15, 48, 2)
    codes, scales, zeros = rtn.rtn_minmax(W, 4, 48, sym=sym)
    out = gptq.gptq_blocked_ref(W, 4.0 * np.eye(48), 4, 48, block_size=16, sym=sym)
    assert np.array_equal(out["codes"], codes)
    assert np.array_equal(out["scales"], scales) and out["scales"].shape == (15, 1)


@pytest.mark.parametrize("act_order", [False, True])
def test_per_channel_blocked_equals_unblocked(act_order):
    H = hessian.hessian(_x(500, 48, 5))
    W = _weights(12, 48, 3)
    ref = gptq.gptq_obs_ref(W, H, 3, 48, act_order=act_order)
    for B in (8, 16, 40):
        out = gptq.gptq_blocked_ref(W, H, 3, 48, B, act_order=act_order)
        assert np.array_equal(out["codes"], ref["codes"])
        assert np.max(np.abs(out["What"] - ref["What"])) <= 1e-9 * np.max(np.abs(W))
    # the row's grid is the one of the original row (nothing is compensated before column 0)
    s, z = quantizer.group_params(W.min(1), W.max(1), 7)
    assert np.array_equal(ref["scales"][:, 0], s) and np.array_equal(ref["zeros"][:, 0], z)


# ---------------------------------------------------------------- static groups -------------
def test_static_groups_identity_hessian_is_rtn_of_the_original_groups():
    W = _weights(16, 64, 4)
    H = np.diag(np.linspace(1.0, 9.0, 64)[::-1][np.random.default_rng(0).permutation(64)])
    codes, scales, zeros = rtn.rtn_minmax(W, 4, 16)
    out = gptq.gptq_blocked_ref(W, H, 4, 16, 32, act_order=True, static_groups=True)
    assert not np.array_equal(out["perm"], np.arange(64))      # act_order reordered
    assert np.array_equal(out["g_idx"], np.arange(64) // 16)
    assert np.array_equal(out["codes"], codes)
    assert np.array_equal(out["scales"], scales) and np.array_equal(out["zeros"], zeros)


@pytest.mark.parametrize("act_order", [False, True])
def test_static_groups_blocked_equals_unblocked(act_order):
    H = hessian.hessian(_x(400, 64, 6))
    W = _weights(20, 64, 5)
    ref = gptq.gptq_obs_ref(W, H, 4, 16, act_order=act_order, static_groups=True)
    for B in (16, 32, 64):
        out = gptq.gptq_blocked_ref(W, H, 4, 16, B, act_order=act_order, static_groups=True)
        assert np.array_equal(out["codes"], ref["codes"])
    s0, z0 = gptq.static_group_params(W, 4, 16)
    assert np.array_equal(ref["scales"], s0) and np.array_equal(ref["zeros"], z0)


def test_static_groups_least_squares_resolve():
    """Every code is the rounding, on its original group's fixed grid, of the value the
    least-squares re-solve gives the column once the earlier columns are fixed."""
    d, g, bits = 16, 4, 3
    maxq = 2 ** bits - 1
    H = hessian.hessian(_x(60, d, 7))
    W = _weights(5, d, 6)
    out = gptq.gptq_blocked_ref(W, H, bits, g, 8, act_order=True, static_groups=True)
    perm = out["perm"]
    Hd, _ = factor.damp(H[np.ix_(perm, perm)], 0.01)
    W0, What = W[:, perm], out["What"][:, perm]
    for r in range(W.shape[0]):
        for q in range(d):
            Q, R = np.arange(q), np.arange(q, d)
            wR = W0[r, R] - np.linalg.solve(Hd[np.ix_(R, R)], Hd[np.ix_(R, Q)] @ (What[r, Q] - W0[r, Q]))
            k = perm[q] // g
            code = quantizer.quantize(wR[0], out["scales"][r, k], out["zeros"][r, k], maxq)
            assert out["codes"][r, perm[q]] == code


# ---------------------------------------------------------------- clip search ---------------
def test_clip_grid_is_the_pages():
    assert np.allclose(rtn.clip_ratios(), [1.0 - 0.05 * i for i in range(11)], rtol=0, atol=1e-15)
    assert rtn.clip_ratios()[-1] == 0.5


@pytest.mark.parametrize("sym", [False, True])
def test_clip_search_single_point_is_plain_rtn(sym):
    W = _weights(10, 64, 8)
    codes, scales, zeros, best, _ = rtn.rtn_clip_search(W, 4, 16, sym=sym, min_ratio=1.0)
    c, s, z = rtn.rtn_minmax(W, 4, 16, sym=sym)
    assert np.array_equal(codes, c) and np.array_equal(scales, s) and np.all(best == 0)


@pytest.mark.parametrize("sym", [False, True])
def test_clip_search_brute_force(sym):
    """A plain per-group loop over the grid reproduces the choice, and the chosen error never
    exceeds that of the unclipped group."""
    bits, g = 3, 8
    maxq = 2 ** bits - 1
    W = _weights(6, 32, 9)
    X = _x(200, 32, 9)
    H = hessian.hessian(X)
    codes, scales, zeros, best, crit = rtn.rtn_clip_search(W, bits, g, H=H, sym=sym)
    params = quantizer.group_params_sym if sym else quantizer.group_params
    for r in range(6):
        for k in range(4):
            w = W[r, k * g:(k + 1) * g]
            Hk = H[k * g:(k + 1) * g, k * g:(k + 1) * g]
            errs = []
            for rho in rtn.clip_ratios():
                c = rho * np.max(np.abs(w))
                wc = np.clip(w, -c, c)
                s, z = params(wc.min(), wc.max(), maxq)
                d = w - quantizer.dequantize(quantizer.quantize(wc, s, z, maxq), s, z)
                errs.append(d @ Hk @ d)
            assert best[r, k] == int(np.argmin(errs))
            assert np.allclose(crit[:, r, k], errs, rtol=1e-12, atol=0)
            assert min(errs) <= errs[0]
    # the H criterion is the group's output error, from the activations: d·H_gg·d = 2‖X_g dᵀ‖²
    Wh = rtn.rtn_dequant(codes, scales, zeros, g)
    D = (W - Wh).reshape(6, 4, g)
    Xg = X.astype(np.float64).reshape(200, 4, g)
    direct = 2.0 * np.einsum("tkg,rkg->rkt", Xg, D) ** 2
    chosen = np.take_along_axis(crit, best[None], axis=0)[0]
    assert np.allclose(chosen, direct.sum(axis=2), rtol=1e-9, atol=0)


def test_clip_search_without_h_is_weight_mse():
    W = _weights(8, 32, 10)
    a = rtn.rtn_clip_search(W, 4, 16)
    b = rtn.rtn_clip_search(W, 4, 16, H=np.eye(32))
    assert np.array_equal(a[3], b[3]) and np.allclose(a[4], b[4], rtol=1e-12, atol=0)
    assert np.any(a[3] > 0)               # the outlier groups do get clipped


# ---------------------------------------------------- percentile / fixed-range clipping -------
def test_group_quantile_worked_example_and_library():
    """The interpolation between order statistics: [1, 2, 3, 4, 10] at 0.9 sits at position
    0.9·4 = 3.6, so 4 + 0.6·(10 − 4) = 7.6; at 0.1 at 0.4: 1 + 0.4·1 = 1.4. The 0 and 1
    quantiles are the min and the max, and positions that are whole numbers give the order
    statistic itself. It agrees with numpy's default ("linear") quantile to rounding."""
    v = np.array([[1.0, 2.0, 3.0, 4.0, 10.0]])
    assert abs(rtn.group_quantile(v, 0.9)[0] - 7.6) < 1e-14
    assert abs(rtn.group_quantile(v, 0.1)[0] - 1.4) < 1e-14
    assert rtn.group_quantile(v, 1.0)[0] == 10.0 and rtn.group_quantile(v, 0.0)[0] == 1.0
    assert rtn.group_quantile(v, 0.5)[0] == 3.0 and rtn.group_quantile(v, 0.75)[0] == 4.0
    rng = np.random.default_rng(5)
    x = np.sort(rng.standard_normal((300, 128)), axis=1)
    for p in (0.9999, 0.999, 0.99, 0.9, 0.5, 0.0001):
        q = rtn.group_quantile(x, p)
        ref = np.quantile(x, p, axis=1)
        # (rounding relative to the interpolated values, which may cancel towards 0)
        assert np.all(np.abs(q - ref) <= 4 * np.spacing(np.max(np.abs(x), axis=1))), p
        assert np.all(q >= x[:, :1].T[0]) and np.all(q <= x[:, -1])


@pytest.mark.parametrize("sym", [False, True])
def test_range_clip_without_clipping_is_plain_rtn(sym):
    W = _weights(12, 128, 11)
    c, s, z = rtn.rtn_minmax(W, 4, 32, sym=sym)
    for kw in (dict(), dict(abs_range=float(np.max(np.abs(W))))):
        codes, scales, zeros, lo, hi = rtn.rtn_range_clip(W, 4, 32, sym=sym, **kw)
        assert np.array_equal(codes, c) and np.array_equal(scales, s)
        assert np.array_equal(zeros, z)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("percentile,abs_range", [(99.99, 0.0), (99.0, 0.0), (90.0, 0.0),
                                                  (100.0, 0.02), (99.9, 0.05)])
def test_range_clip_codes_are_the_nearest_level_of_the_clamped_weight(sym, percentile,
                                                                      abs_range):
    """Brute force: every code is the nearest level of the clamped weight (ties to the even
    quotient), values beyond a bound take the bound's code, |clip(w) − ŵ| <= scale/2, and the
    bounds are the quantiles (limited by the absolute range)."""
    bits, g = 4, 16
    maxq = 2 ** bits - 1
    W = _weights(9, 64, 12)
    codes, scales, zeros, lo, hi = rtn.rtn_range_clip(W, bits, g, percentile, abs_range, sym)
    Wg = W.reshape(9, 4, g)
    v = np.sort(Wg, axis=2)
    p = percentile / 100.0
    exp_hi, exp_lo = rtn.group_quantile(v, p), rtn.group_quantile(v, 1.0 - p)
    if abs_range > 0:
        exp_hi, exp_lo = np.minimum(exp_hi, abs_range), np.maximum(exp_lo, -abs_range)
    assert np.array_equal(hi, exp_hi) and np.array_equal(lo, exp_lo)
    wc = np.clip(Wg, lo[..., None], hi[..., None])
    s, z = scales[..., None], zeros[..., None]
    levels = np.arange(maxq + 1)
    recon = s[..., None] * (levels - z[..., None])               # [r, k, 1, levels]
    dist = np.abs(wc[..., None] - recon)
    q = codes.reshape(9, 4, g)
    got = np.take_along_axis(dist, q[..., None], axis=3)[..., 0]
    assert np.all(got <= dist.min(axis=3) + 1e-18)
    assert np.all(np.abs(wc - s * (q - z)) <= s / 2 + 1e-18)
    clipped = (Wg > hi[..., None]) | (Wg < lo[..., None])
    if percentile < 100.0:
        assert clipped.any()
    bound = np.where(Wg > hi[..., None], hi[..., None], lo[..., None])
    q_bound = quantizer.quantize(bound, s, z, maxq)
    assert np.array_equal(q[clipped], q_bound[clipped])

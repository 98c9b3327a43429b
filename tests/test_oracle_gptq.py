"""Pins for the oracle's GPTQ references.

* H = c·I: no compensation, so GPTQ equals RTN bit for bit.
* The blocked (lazy-update) reference equals the unblocked OBS reference for every block size.
* Closed form: after the first k columns are quantized, the remaining weights equal the
  least-squares re-solve w_R = w_R⁰ − H_RR⁻¹ H_RQ (ŵ_Q − w_Q⁰). The whole output is rebuilt
  from that formula and the quantizer alone, and must match.
* Loss identity tr(ΔHΔᵀ) = 2‖ΔXᵀ‖², row independence, act_order bookkeeping.
"""

import numpy as np
import pytest

from oracle import factor, gptq, hessian, loss, quantizer, rtn
from post_weight_quantization_24_b200 import workloads


def _hessian(n, d, seed, correlated=False):
    if correlated:
        X = workloads.correlated_activations(n, d, seed=seed).numpy()
    else:
        rng = np.random.default_rng(seed)
        X = (rng.standard_normal((n, d)) * np.exp(0.5 * rng.standard_normal(d))).astype(np.float16)
    return X, hessian.hessian(X)


def _weights(d_out, d_in, seed):
    rng = np.random.default_rng(100 + seed)
    return (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16).astype(np.float64)


@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("bits,g", [(4, 16), (3, 32), (2, 8)])
def test_identity_hessian_reduces_to_rtn(act_order, bits, g):
    W = _weights(24, 64, 0)
    H = 3.7 * np.eye(64)
    codes, scales, zeros = rtn.rtn_minmax(W, bits, g)
    for out in (gptq.gptq_blocked_ref(W, H, bits, g, block_size=2 * g, act_order=act_order),
                gptq.gptq_obs_ref(W, H, bits, g, act_order=act_order)):
        assert np.array_equal(out["codes"], codes)
        assert np.array_equal(out["scales"], scales)
        assert np.array_equal(out["zeros"], zeros)


@pytest.mark.parametrize("correlated", [False, True])
@pytest.mark.parametrize("act_order", [False, True])
def test_blocked_equals_unblocked(correlated, act_order):
    X, H = _hessian(400, 64, 3, correlated)
    W = _weights(20, 64, 1)
    ref = gptq.gptq_obs_ref(W, H, 4, 8, act_order=act_order)
    for B in (8, 16, 32, 64):
        out = gptq.gptq_blocked_ref(W, H, 4, 8, block_size=B, act_order=act_order)
        assert np.array_equal(out["codes"], ref["codes"])
        assert np.array_equal(out["scales"], ref["scales"])
        assert np.array_equal(out["zeros"], ref["zeros"])
        assert np.max(np.abs(out["What"] - ref["What"])) <= 1e-9 * np.max(np.abs(W))


@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_least_squares_resolve_closed_form(act_order, seed):
    """Rebuild GPTQ's output from the LS re-solve: every column is quantized at the value the
    remaining weights take when the already-quantized columns are fixed and the layer error
    (w − w⁰)ᵀ H_d (w − w⁰) is minimised over the rest."""
    d, g, bits = 16, 4, 3
    maxq = 2 ** bits - 1
    X, H = _hessian(60, d, 10 + seed, correlated=True)
    W = _weights(6, d, seed)
    out = gptq.gptq_blocked_ref(W, H, bits, g, block_size=8, act_order=act_order)
    perm = out["perm"]
    Hd, _ = factor.damp(H[np.ix_(perm, perm)], 0.01)
    W0 = W[:, perm]
    What = out["What"][:, perm]
    for r in range(W.shape[0]):
        for q in range(d):
            Q, R = np.arange(q), np.arange(q, d)
            wR = W0[r, R] - np.linalg.solve(Hd[np.ix_(R, R)], Hd[np.ix_(R, Q)] @ (What[r, Q] - W0[r, Q]))
            if q % g == 0:
                grp = wR[:g]
                s, z = quantizer.group_params(grp.min(), grp.max(), maxq)
                assert out["scales"][r, q // g] == s
                assert out["zeros"][r, q // g] == z
            s, z = out["scales"][r, q // g], out["zeros"][r, q // g]
            code = quantizer.quantize(wR[0], s, z, maxq)
            assert out["codes"][r, perm[q]] == code
            assert abs(What[r, q] - quantizer.dequantize(code, s, z)) == 0.0


@pytest.mark.parametrize("act_order", [False, True])
def test_trace_values_are_the_least_squares_resolve(act_order):
    """The traced pre-rounding weight of every column equals the closed-form LS re-solve given
    the earlier quantized columns, and the traced group quantities are the ones the scale and
    zero are rounded from: fp16 round-up of the step, rint of the zero quotient, the group's
    widened range."""
    d, g, bits = 24, 8, 3
    maxq = 2 ** bits - 1
    X, H = _hessian(80, d, 31, correlated=True)
    W = _weights(5, d, 7)
    out = gptq.gptq_blocked_ref(W, H, bits, g, block_size=16, act_order=act_order, trace=True)
    perm = out["perm"]
    Hd, _ = factor.damp(H[np.ix_(perm, perm)], 0.01)
    W0 = W[:, perm]
    What = out["What"][:, perm]
    for r in range(W.shape[0]):
        for q in range(d):
            Q, R = np.arange(q), np.arange(q, d)
            wR = W0[r, R] - np.linalg.solve(Hd[np.ix_(R, R)], Hd[np.ix_(R, Q)] @ (What[r, Q] - W0[r, Q]))
            assert abs(out["pre"][r, q] - wR[0]) <= 1e-9 * np.max(np.abs(W))
            if q % g == 0:
                lo, hi = min(wR[:g].min(), 0.0), max(wR[:g].max(), 0.0)
                assert out["step"][r, q // g] == pytest.approx((hi - lo) / maxq, rel=1e-9)
                assert out["zquot"][r, q // g] == pytest.approx(-lo / out["scales"][r, q // g],
                                                                rel=1e-9, abs=1e-12)
    assert np.array_equal(out["scales"], quantizer.fp16_round_up(out["step"]))
    assert np.array_equal(out["zeros"], np.rint(out["zquot"]))
    assert np.array_equal(out["codes_p"], out["codes"][:, perm])


def test_factorisation_routes_drive_the_same_gptq():
    """prepare_u's two routes give U within rounding of each other, and the GPTQ outputs they
    drive are identical on a layer with no near ties."""
    X, H = _hessian(500, 96, 41)
    W = _weights(40, 96, 8)
    _, U1 = gptq.prepare_u(H, 0.01, True, route="textbook")
    _, U2 = gptq.prepare_u(H, 0.01, True, route="reversed")
    assert np.max(np.abs(U1 - U2)) <= 1e-10 * np.max(np.abs(U1))
    a = gptq.gptq_blocked_ref(W, H, 4, 32, act_order=True, U=U1)
    b = gptq.gptq_blocked_ref(W, H, 4, 32, act_order=True, U=U2)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    with pytest.raises(ValueError):
        gptq.prepare_u(H, route="other")


def test_single_column_update_closed_form():
    d = 9
    X, H = _hessian(50, d, 21, correlated=True)
    W = _weights(3, d, 5)
    Hd, _ = factor.damp(H, 0.01)
    U = factor.upper_chol_of_inverse(Hd)
    # OBS step for column 0 with the U row, as the blocked loop applies it
    s, z = quantizer.group_params(W[:, :d].min(1), W[:, :d].max(1), 15)
    wh0 = quantizer.dequantize(quantizer.quantize(W[:, 0], s, z, 15), s, z)
    e = (W[:, 0] - wh0) / U[0, 0]
    Wn = W[:, 1:] - np.outer(e, U[0, 1:])
    R = np.arange(1, d)
    ls = W[:, 1:] - np.linalg.solve(Hd[np.ix_(R, R)], Hd[np.ix_(R, [0])] @ (wh0 - W[:, 0])[None, :]).T
    assert np.max(np.abs(Wn - ls)) <= 1e-10 * np.max(np.abs(W))


def test_rows_are_independent():
    X, H = _hessian(300, 48, 4, correlated=True)
    W = _weights(30, 48, 2)
    full = gptq.gptq_blocked_ref(W, H, 4, 16, block_size=32, act_order=True)
    rows = np.array([29, 3, 17])
    sub = gptq.gptq_blocked_ref(W, H, 4, 16, block_size=32, act_order=True, rows=rows)
    assert np.array_equal(sub["codes"], full["codes"][rows])
    assert np.array_equal(sub["scales"], full["scales"][rows])


def test_block_diagonal_hessian_keeps_compensation_inside_blocks():
    d, g = 32, 8
    _, H1 = _hessian(200, 16, 5, correlated=True)
    _, H2 = _hessian(200, 16, 6, correlated=True)
    H = np.zeros((d, d))
    H[:16, :16], H[16:, 16:] = H1, H2 * (np.trace(H1) / np.trace(H2))  # equal mean diag
    W = _weights(10, d, 3)
    full = gptq.gptq_blocked_ref(W, H, 4, g, block_size=16)
    lam = 0.01 * np.mean(np.diag(H))
    for lo in (0, 16):
        Hb = H[lo:lo + 16, lo:lo + 16]
        # same absolute damping as in the full problem: percdamp relative to this block's mean
        pd = lam / np.mean(np.diag(Hb))
        part = gptq.gptq_blocked_ref(W[:, lo:lo + 16], Hb, 4, g, block_size=16, percdamp=pd)
        assert np.array_equal(part["codes"], full["codes"][:, lo:lo + 16])


def test_act_order_permutation_and_bookkeeping():
    H = np.diag([1.0, 5.0, 5.0, 2.0, 7.0, 1.0, 3.0, 5.0])
    assert gptq.act_order_perm(H).tolist() == [4, 1, 2, 7, 6, 3, 0, 5]
    W = _weights(4, 8, 9)
    out = gptq.gptq_blocked_ref(W, H, 4, 4, block_size=4, act_order=True)
    perm = out["perm"]
    assert out["g_idx"][perm].tolist() == [0, 0, 0, 0, 1, 1, 1, 1]
    s = out["scales"][:, out["g_idx"]]
    z = out["zeros"][:, out["g_idx"]]
    assert np.array_equal(out["What"], quantizer.dequantize(out["codes"], s, z))


def test_loss_identity_with_activations():
    X, H = _hessian(256, 32, 8)
    W = _weights(12, 32, 4)
    out = gptq.gptq_blocked_ref(W, H, 4, 16, block_size=32)
    a = loss.recon_loss(W, out["What"], H)
    b = loss.recon_loss_from_x(W, out["What"], X)
    assert a == pytest.approx(b, rel=1e-10)


def test_gptq_beats_rtn_on_correlated_inputs():
    X, H = _hessian(1024, 128, 12, correlated=True)
    W = _weights(64, 128, 6)
    out = gptq.gptq_blocked_ref(W, H, 3, 32, block_size=64)
    codes, scales, zeros = rtn.rtn_minmax(W, 3, 32)
    W_rtn = rtn.rtn_dequant(codes, scales, zeros, 32)
    assert loss.recon_loss(W, out["What"], H) < 0.8 * loss.recon_loss(W, W_rtn, H)


def test_argument_checks():
    H = np.eye(16)
    W = np.zeros((2, 16))
    with pytest.raises(ValueError):
        gptq.gptq_blocked_ref(W, H, 4, 5)
    with pytest.raises(ValueError):
        gptq.gptq_blocked_ref(W, H, 4, 8, block_size=12)
    with pytest.raises(ValueError):
        gptq.gptq_blocked_ref(W, H, 9, 8)
    with pytest.raises(factor.NotPositiveDefinite):
        gptq.gptq_blocked_ref(W, np.zeros((16, 16)), 4, 8)

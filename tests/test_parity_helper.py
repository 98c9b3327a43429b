"""The near-tie parity criterion (tests/gptq_parity.py) on the CPU, with mistakes planted in a
copy of the oracle's own result: a flip far from a tie must be caught wherever it sits (code,
scale, zero), a flip at a near tie must be accepted together with the cascade after it, and
the derived window must be small and positive."""

import numpy as np
import pytest

from gptq_parity import (first_divergence, near_tie_report, perturbed_hessian,
                         window_from_h_sensitivity)
from oracle import gptq, hessian
from post_weight_quantization_24_b200 import workloads

BITS, G, B = 3, 16, 32


@pytest.fixture(scope="module")
def case():
    X = workloads.correlated_activations(600, 64, rank=3, seed=9).numpy()
    H = hessian.hessian(X)
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((40, 64)) * 0.02).astype(np.float16).astype(np.float64)
    ref = gptq.gptq_blocked_ref(W, H, BITS, G, B, act_order=True, trace=True)
    return W, H, ref


def _report(ref, codes, scales=None, zeros=None, eps=1e-3):
    return near_tie_report(codes, ref["scales"] if scales is None else scales,
                           ref["zeros"] if zeros is None else zeros, ref["perm"], ref, G, BITS,
                           eps)


def _tie_dist(ref):
    gi = np.arange(ref["pre"].shape[1]) // G
    t = ref["pre"] / ref["scales"][:, gi]
    return t, np.abs(np.abs(t - np.floor(t)) - 0.5)


def test_identical_result_passes(case):
    _, _, ref = case
    rep = _report(ref, ref["codes"])
    assert rep["rows_diverged"] == 0 and rep["bad_origin"] == 0 and rep["agree"] == 1.0


def test_flip_far_from_a_tie_is_caught(case):
    _, _, ref = case
    t, dist = _tie_dist(ref)
    maxq = 2 ** BITS - 1
    r, q = np.argwhere((dist > 0.3) & (ref["codes_p"] < maxq))[0]
    codes = ref["codes"].copy()
    codes[r, ref["perm"][q]] += 1
    rep = _report(ref, codes)
    assert rep["bad_origin"] == 1 and rep["bad_examples"][0]["row"] == r


def test_flip_at_a_near_tie_and_its_cascade_are_accepted(case):
    _, _, ref = case
    t, dist = _tie_dist(ref)
    maxq = 2 ** BITS - 1
    inside = (ref["codes_p"] > 0) & (ref["codes_p"] < maxq)
    r, q = np.unravel_index(np.argmin(np.where(inside, dist, np.inf)), dist.shape)
    eps = 1.5 * dist[r, q] + 1e-12
    codes_p = ref["codes_p"].copy()
    codes_p[r, q] += 1 if t[r, q] - np.floor(t[r, q]) < 0.5 else -1
    # the cascade: later columns of that row move, some by two levels
    later = np.arange(q + 1, codes_p.shape[1])
    codes_p[r, later] = np.clip(codes_p[r, later] + 2, 0, maxq)
    codes = np.empty_like(codes_p)
    codes[:, ref["perm"]] = codes_p
    rep = _report(ref, codes, eps=eps)
    assert rep["rows_diverged"] == 1 and rep["bad_origin"] == 0
    assert rep["max_abs_diff"] == 2
    # the same flip with a window below its distance is not a tie
    rep = _report(ref, codes, eps=0.5 * dist[r, q])
    assert rep["bad_origin"] == 1


def test_scale_and_zero_flips_far_from_ties_are_caught(case):
    _, _, ref = case
    sc, step = ref["scales"], ref["step"]
    below = np.nextafter(sc.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    gap = np.minimum(sc - step, step - below) / (sc - below)
    r, k = np.argwhere(gap > 0.3)[0]          # the step sits well inside its fp16 interval
    s = sc.copy()
    s[r, k] = np.nextafter(np.float16(s[r, k]), np.float16(np.inf)).astype(np.float64)
    rep = _report(ref, ref["codes"], scales=s, eps=1e-4)
    assert rep["bad_origin"] == 1 and rep["bad_examples"][0]["kind"] == "param"
    zq = ref["zquot"]
    r, k = np.argwhere(np.abs(np.abs(zq - np.floor(zq)) - 0.5) > 0.3)[0]
    z = ref["zeros"].copy()
    z[r, k] += 1
    rep = _report(ref, ref["codes"], zeros=z, eps=1e-4)
    assert rep["bad_origin"] == 1 and rep["bad_examples"][0]["kind"] == "param"


def test_first_divergence_orders_params_before_codes():
    a = np.zeros((2, 8), np.int64)
    b = a.copy()
    b[0, 5] = 1
    b[1, 4] = 1
    sa = np.ones((2, 2))
    sb = sa.copy()
    sb[1, 1] = 2.0                      # group 1 starts at column 4: same column as the code
    first, kind = first_divergence(a, b, sa, sa, sb, sa, 4)
    assert first.tolist() == [5, 4] and kind.tolist() == ["code", "param"]


def test_window_is_positive_and_small(case):
    W, H, ref = case
    rows = np.arange(0, 40, 2)
    sub = {k: ref[k][rows] for k in ("pre", "codes_p", "scales", "zeros", "step", "zquot")}
    sub["perm"] = ref["perm"]
    eps, detail = window_from_h_sensitivity(W, H, BITS, G, B, 0.01, True, sub, rows)
    assert 0.0 < eps < 0.01, detail
    assert detail["entries_compared"] > 0


def test_perturbation_has_the_requested_size():
    X = workloads.correlated_activations(400, 96, rank=3, seed=2).numpy()
    H = hessian.hessian(X)
    Hp = perturbed_hessian(H, 1e-5, block=40)
    assert np.array_equal(Hp, Hp.T)
    rel = np.linalg.norm(Hp - H) / np.linalg.norm(H)
    assert rel == pytest.approx(1e-5, rel=1e-6)
    assert np.allclose(np.abs(Hp - H), 1e-5 * np.abs(H), rtol=1e-6, atol=0)

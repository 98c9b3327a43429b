"""Pins for the oracle's quantizer and RTN: the pages' worked example, storage arithmetic,
brute force over all levels, and exact bounds."""

import os

import numpy as np
import pytest

from oracle import quantizer, rtn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _is_fp16(x):
    x = np.asarray(x, np.float64)
    return np.all(x.astype(np.float16).astype(np.float64) == x)


def test_fp16_round_up_exact_cases():
    assert quantizer.fp16_round_up(1.0) == 1.0
    # above 1 by less than half an fp16 ulp: nearest would give 1.0, upward gives 1 + 2^-10
    assert quantizer.fp16_round_up(1.0 + 2.0 ** -30) == 1.0 + 2.0 ** -10
    # exactly half an ulp above 1: nearest-even gives 1.0, upward gives 1 + 2^-10
    assert quantizer.fp16_round_up(1.0 + 2.0 ** -11) == 1.0 + 2.0 ** -10
    assert quantizer.fp16_round_up(0.0) == 0.0
    # fp16 subnormal range
    assert quantizer.fp16_round_up(2.0 ** -30) == 2.0 ** -24


def test_fp16_round_up_is_smallest_fp16_above():
    rng = np.random.default_rng(1)
    x = np.exp(rng.uniform(np.log(1e-6), np.log(6e4), 20000))
    r = quantizer.fp16_round_up(x)
    assert _is_fp16(r)
    assert np.all(r >= x)
    below = np.nextafter(r.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    assert np.all(below < x)


def test_worked_example_int8():
    (bits, xmin, xmax, printed, digits), = _rows("worked_example_int8.txt")
    bits, xmin, xmax, printed, digits = int(bits), float(xmin), float(xmax), float(printed), int(digits)
    maxq = 2 ** bits - 1
    s, z = quantizer.group_params(xmin, xmax, maxq)
    # the page's value to its printed precision (3 significant digits)
    assert abs(s - printed) <= 0.5 * 10.0 ** (np.floor(np.log10(printed)) - digits + 1)
    # and the reading: the exact (max-min)/(qmax-qmin) rounded up to the next fp16 value
    exact = (xmax - xmin) / maxq
    assert _is_fp16(s) and exact <= s < exact + 2.0 ** -16
    # the range endpoints land on the first and last level
    q = quantizer.quantize([xmin, xmax], s, z, maxq)
    assert q[0] == 0 and q[1] == maxq


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_quantizer_error_bound_and_nearest_level(bits):
    rng = np.random.default_rng(bits)
    maxq = 2 ** bits - 1
    for trial in range(200):
        g = rng.integers(2, 40)
        w = rng.standard_t(3, g) * 0.02
        if trial % 3 == 0:
            w = np.abs(w) + 0.01                 # a group that does not contain 0
        w = w.astype(np.float16).astype(np.float64)
        s, z = quantizer.group_params(w.min(), w.max(), maxq)
        q = quantizer.quantize(w, s, z, maxq)
        wh = quantizer.dequantize(q, s, z)
        assert np.all((q >= 0) & (q <= maxq))
        assert np.all(np.abs(w - wh) <= s / 2)
        # brute force: no level is closer
        levels = quantizer.dequantize(np.arange(maxq + 1), s, z)
        best = np.min(np.abs(w[:, None] - levels[None, :]), axis=1)
        assert np.all(np.abs(w - wh) <= best)
        # the zero point is a code and real 0 sits exactly on it
        assert z == np.rint(z) and 0 <= z <= maxq and not np.signbit(z)
        assert quantizer.dequantize(np.array([z]), s, z)[0] == 0.0
        # the widened range's lower end maps to code 0 (rint(-x) = -rint(x) under half-even;
        # the upper end may land one code short because z is rounded)
        lo = min(w.min(), 0.0)
        assert quantizer.quantize(np.array([lo]), s, z, maxq)[0] == 0
        if w.min() >= 0:
            assert z == 0 and q[np.argmin(w)] == np.clip(np.rint(w.min() / s), 0, maxq)
        else:
            assert q[np.argmin(w)] == 0


def test_quantizer_ties_round_half_even():
    s, z, maxq = 0.5, 3.0, 15
    w = np.array([0.25, 0.75, 1.25, -0.25, -0.75])   # w/s = 0.5, 1.5, 2.5, -0.5, -1.5
    q = quantizer.quantize(w, s, z, maxq)
    assert list(q) == [3, 5, 5, 3, 1]


def test_degenerate_group_scale_one():
    s, z = quantizer.group_params(0.0, 0.0, 15)
    assert s == 1.0 and z == 0.0 and not np.signbit(z)
    assert quantizer.quantize(np.array([0.0]), s, z, 15)[0] == 0


def test_one_signed_groups_widen_to_zero():
    # a constant positive group: range [0, 0.3], the value lands on the top code
    s, z = quantizer.group_params(0.3, 0.3, 15)
    assert z == 0.0 and s == quantizer.fp16_round_up(0.3 / 15)
    assert quantizer.quantize(np.array([0.3]), s, z, 15)[0] == 15
    # a negative group [-0.7, -0.2]: range [-0.7, 0], zero point at the top code
    s, z = quantizer.group_params(-0.7, -0.2, 7)
    assert s == quantizer.fp16_round_up(0.7 / 7) and z == 7.0
    assert list(quantizer.quantize(np.array([-0.7, 0.0]), s, z, 7)) == [0, 7]
    # a tiny span far from 0 no longer gives a zero point beyond fp16's exact integers
    s, z = quantizer.group_params(1.0, 1.0 + 2.0 ** -20, 7)
    assert z == 0.0 and np.float16(z) == z


def test_rtn_matches_per_group_brute_force():
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((16, 64)) * 0.02).astype(np.float16).astype(np.float64)
    codes, scales, zeros = rtn.rtn_minmax(W, 4, 16)
    for r in range(16):
        for gi in range(4):
            w = W[r, gi * 16:(gi + 1) * 16]
            span = max(w.max(), 0.0) - min(w.min(), 0.0)
            s = quantizer.fp16_round_up(span / 15)
            assert scales[r, gi] == s
            levels = s * (np.arange(16) - zeros[r, gi])
            for k, wv in enumerate(w):
                c = codes[r, gi * 16 + k]
                assert abs(wv - levels[c]) <= np.min(np.abs(wv - levels))


def test_pack_int4_nibble_order():
    codes = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    packed = rtn.pack_int4(codes)
    assert packed.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(rtn.unpack_int4(packed), codes)


def test_storage_accounting_matches_pages():
    for bits, g, bpw in _rows("storage_bits.txt"):
        bits, g, bpw = int(bits), int(g), float(bpw)
        assert rtn.storage_bits_per_weight(bits, g) == bpw
        # and the buffers the layout actually uses: packed codes + fp16 scales + fp16 zeros
        d_out, d_in = 8, 4 * g
        W = np.random.default_rng(0).standard_normal((d_out, d_in))
        codes, scales, zeros = rtn.rtn_minmax(W, bits, g)
        packed = rtn.pack_int4(codes)
        nbytes = packed.nbytes + scales.astype(np.float16).nbytes + zeros.astype(np.float16).nbytes
        assert nbytes * 8 / (d_out * d_in) == bpw


def test_model_size_arithmetic_matches_pages():
    for n, bits, gb, digits in _rows("model_sizes.txt"):
        n, bits, gb, digits = float(n), int(bits), float(gb), int(digits)
        if bits == 4:
            nbytes = n / 2                       # two codes per byte
        else:
            nbytes = n * bits / 8
        assert round(nbytes / 1e9, digits) == gb

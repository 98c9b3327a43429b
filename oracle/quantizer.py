"""Oracle: the asymmetric per-group min-max quantizer (test infrastructure only).

Sources
  * 0539edu.com/news/6111416 §2.1: q = round(x/scale) + zero_point; the worked example maps the
    range [-2.5, 3.7] onto the 256 INT8 levels with scale = (max - min)/(qmax - qmin) ≈ 0.0243.
  * 0539edu.com/news/6111416 §4.2: one fp16 scale and one fp16 zero point per group.
  * hncyxsy.com/news/243429 §3.1 step 3: per column, pick the quantization scale, round, keep
    the error.

Readings taken where the pages are silent:
  * Codes use the unsigned range [0, maxq], maxq = 2**bits - 1 (the INT8 example's signed range
    differs only by an offset of 2**(bits-1)).
  * The range is the group's min and max widened to contain 0. §2.1's formula sends the real
    value 0 to the code zero_point, so zero_point is itself a code in [0, maxq] and, with
    §4.2's fp16 storage, exact; a group entirely above (below) 0 gets the range [0, max]
    ([min, 0]). For groups that contain 0 (the worked example's [-2.5, 3.7]) this is the
    literal min and max.
  * scale = (xmax - xmin)/maxq rounded UP to fp16, so that the stored scale is what the codes
    are computed with and |w - ŵ| <= scale/2 holds exactly for every entry.
  * zero = rint(-xmin/scale), round half to even; an integer in [0, maxq] (+0, never -0),
    stored as an fp16 value.
  * An all-zero group (xmax == xmin == 0 after widening) gets scale 1.
  * q = clamp(rint(w/scale) + zero, 0, maxq), round half to even; ŵ = scale·(q - zero).
"""

import numpy as np


def fp16_round_up(x):
    """Smallest fp16 value >= x, element-wise, returned as fp64.

    ``np.float16`` converts fp64 with one round-to-nearest-even step; where that landed below
    x, the next fp16 value up is taken. Values above the fp16 range become +inf.
    """
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    below = h.astype(np.float64) < x
    h = np.where(below, np.nextafter(h, np.float16(np.inf)), h)
    return h.astype(np.float64)


def group_params(xmin, xmax, maxq, trace=False):
    """(scale, zero) for groups with the given minima and maxima (fp64 arrays).

    The range [xmin, xmax] is first widened to contain 0. scale is fp16-representable (held
    in fp64), zero is an integer in [0, maxq] (held in fp64).

    With ``trace`` the two quantities before their rounding come back as well: the unrounded
    step (xmax - xmin)/maxq (before the round-up to fp16) and the zero quotient -xmin/scale
    (before rint). They locate the group's rounding decisions: a scale whose unrounded step
    sits on an fp16 value, or a zero whose quotient sits on a half-integer, is a tie.
    """
    xmin = np.minimum(np.asarray(xmin, dtype=np.float64), 0.0)
    xmax = np.maximum(np.asarray(xmax, dtype=np.float64), 0.0)
    span = xmax - xmin
    with np.errstate(divide="ignore", invalid="ignore"):
        step = span / maxq
        scale = fp16_round_up(step)
        scale = np.where(span == 0.0, 1.0, scale)
        zquot = -xmin / scale
        zero = np.rint(zquot) + 0.0
    if trace:
        return scale, zero, step, zquot
    return scale, zero


def group_params_sym(xmin, xmax, maxq, trace=False):
    """(scale, zero) of the symmetric quantizer for groups with the given minima and maxima.

    0539edu.com/news/6111416 §2.3: a symmetric quantizer fixes the zero point at 0, so
    q = round(x/scale). Reading: the range is [-m, m] with m = max(|min|, |max|), split into
    maxq steps like the asymmetric range: scale = 2m/maxq rounded up to fp16 (1 for an all-zero
    group). Codes stay unsigned: the zero point 0 of the signed code is stored as the code
    offset 2**(bits-1) = (maxq + 1)/2, so q = clamp(rint(w/scale) + (maxq+1)/2, 0, maxq) and
    |w - ŵ| <= scale/2 still holds for every entry.
    """
    m = np.maximum(np.abs(np.asarray(xmin, dtype=np.float64)),
                   np.abs(np.asarray(xmax, dtype=np.float64)))
    step = 2.0 * m / maxq
    scale = np.where(m == 0.0, 1.0, fp16_round_up(step))
    zero = np.full_like(scale, (maxq + 1) // 2, dtype=np.float64)
    if trace:
        return scale, zero, step, np.full_like(scale, np.nan)
    return scale, zero


def quantize(w, scale, zero, maxq):
    """Integer codes q = clamp(rint(w/scale) + zero, 0, maxq) (fp64 in, int64 out)."""
    w = np.asarray(w, dtype=np.float64)
    q = np.rint(w / scale) + zero
    return np.clip(q, 0, maxq).astype(np.int64)


def dequantize(q, scale, zero):
    """ŵ = scale·(q - zero) in fp64."""
    return np.asarray(scale, np.float64) * (np.asarray(q, np.float64) - zero)

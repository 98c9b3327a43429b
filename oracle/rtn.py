"""Oracle: group min-max round-to-nearest (RTN) weight quantization (test infrastructure only).

Sources
  * bhfrc.com/news/5741 §2.2: independent min-max per group of ``group_size`` weights.
  * 0539edu.com/news/6111416 §4.2: with fp16 scale and zero per group, 4-bit storage costs
    4 + 32/group_size bits per weight (4.25 / 4.5 / 5 at 128 / 64 / 32).
  * hncyxsy.com/news/243429 §1.2: RTN rounds every weight independently, with no compensation.
  * gtnt.cn/news/115337 §3 (awq_clip) and bhfrc.com/news/5741 §4.3: the range can be clipped
    before the min-max scale is taken, by a searched ratio of the block's absolute maximum or
    by a percentile (99.99 %) or a fixed absolute range.

Layout: W is [d_out, d_in] (PyTorch Linear layout); groups are ``group_size`` consecutive
input columns of one row. scales and zeros are [d_out, d_in/group_size]. For 4-bit codes the
packed form holds two codes per byte, the even column in the low nibble.
"""

import numpy as np

from .quantizer import group_params, group_params_sym, quantize, dequantize


def rtn_minmax(W, bits, group_size, sym=False):
    """Return (codes int64 [d_out, d_in], scales fp64, zeros fp64 [d_out, d_in/g]).
    ``sym`` takes the symmetric quantizer (0539edu.com §2.3) instead of the asymmetric one."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    if d_in % group_size:
        raise ValueError("d_in must be a multiple of group_size")
    maxq = 2 ** bits - 1
    Wg = W.reshape(d_out, d_in // group_size, group_size)
    params = group_params_sym if sym else group_params
    scale, zero = params(Wg.min(axis=2), Wg.max(axis=2), maxq)
    q = quantize(Wg, scale[..., None], zero[..., None], maxq)
    return q.reshape(d_out, d_in), scale, zero


def clip_ratios(min_ratio=0.5, step=0.05):
    """The clip grid of gtnt.cn/news/115337 §3 (awq_clip): ratios of the block's amax from 1
    down to min_ratio (default 0.5) in steps of `step` (default 0.05), largest first:
    ρ_i = 1 − i·step, i = 0 … round((1 − min_ratio)/step)."""
    n = int(round((1.0 - min_ratio) / step)) + 1
    return np.array([1.0 - i * step for i in range(n)])


def rtn_clip_search(W, bits, group_size, H=None, sym=False, min_ratio=0.5, step=0.05):
    """Group RTN with a clip search per group (gtnt.cn §3: search each quantization block's
    clip bound c in [amax·min_ratio, amax], amax = max |w| of the block, truncating the
    weights to [-c, c] before their min-max scale is taken).

    For each group and each grid ratio ρ (``clip_ratios(min_ratio, step)``), c = ρ·amax; the group's weights
    are clamped to [-c, c] and quantized with the scale and zero of the clamped group; the
    criterion is the group's share of the layer output error, d·H_gg·d with d = w − ŵ (the
    original weights minus the reconstruction) and H_gg the group's diagonal block of
    H = 2XᵀX; without H it is the weight error d·d. The smallest criterion wins, ties to the
    larger ratio (less clipping).

    Returns (codes [d_out, d_in], scales, zeros [d_out, d_in/g], ratio index [d_out, d_in/g],
    criteria [grid points, d_out, d_in/g])."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    if d_in % group_size:
        raise ValueError("d_in must be a multiple of group_size")
    maxq = 2 ** bits - 1
    ng = d_in // group_size
    Wg = W.reshape(d_out, ng, group_size)
    amax = np.max(np.abs(Wg), axis=2)
    params = group_params_sym if sym else group_params
    if H is not None:
        H = np.asarray(H, dtype=np.float64)
        Hb = np.stack([H[k * group_size:(k + 1) * group_size, k * group_size:(k + 1) * group_size]
                       for k in range(ng)])
    ratios = clip_ratios(min_ratio, step)
    crit = np.empty((len(ratios), d_out, ng))
    cand = []
    for i, rho in enumerate(ratios):
        c = rho * amax
        Wc = np.clip(Wg, -c[..., None], c[..., None])
        s, z = params(Wc.min(axis=2), Wc.max(axis=2), maxq)
        q = quantize(Wc, s[..., None], z[..., None], maxq)
        D = Wg - dequantize(q, s[..., None], z[..., None])
        if H is None:
            crit[i] = np.sum(D * D, axis=2)
        else:
            crit[i] = np.einsum("rkg,kgh,rkh->rk", D, Hb, D)
        cand.append((q, s, z))
    best = np.argmin(crit, axis=0)                # first index among equal minima
    codes = np.empty((d_out, ng, group_size), dtype=np.int64)
    scales = np.empty((d_out, ng))
    zeros = np.empty((d_out, ng))
    for i, (q, s, z) in enumerate(cand):
        m = best == i
        codes[m], scales[m], zeros[m] = q[m], s[m], z[m]
    return codes.reshape(d_out, d_in), scales, zeros, best, crit


def group_quantile(v_sorted, frac):
    """The frac-quantile of each group's values (last axis, sorted ascending), by linear
    interpolation between the order statistics around position frac·(g − 1), every operation
    in fp64 and rounded on its own: h = frac·(g − 1), k = floor(h), t = h − k,
    q = v[k] + t·(v[k+1] − v[k]) (q = v[g−1] at the top)."""
    v = np.asarray(v_sorted, dtype=np.float64)
    g = v.shape[-1]
    h = float(frac) * float(g - 1)
    k = int(np.floor(h))
    if k >= g - 1:
        return v[..., g - 1].copy()
    t = h - k
    return v[..., k] + t * (v[..., k + 1] - v[..., k])


def rtn_range_clip(W, bits, group_size, percentile=100.0, abs_range=0.0, sym=False):
    """Group RTN of clipped weights (bhfrc.com/news/5741 §4.3: instead of the group's extreme
    values, take a percentile of its values such as 99.99 %, or an absolute range such as
    [-10, 10], and truncate what lies outside before the min-max range is formed).

    Per group: lo and hi are the (1 − p) and p quantiles of its weights (``group_quantile``,
    p = percentile/100; percentile 100 gives the min and the max); with abs_range a > 0 they
    are further limited to [−a, a]. The weights are clamped to [lo, hi] and quantized with the
    quantizer of the range [lo, hi] (widened to contain 0, or symmetric with
    m = max(|lo|, |hi|)). Returns (codes [d_out, d_in], scales, zeros [d_out, d_in/g],
    lo, hi [d_out, d_in/g])."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    if d_in % group_size:
        raise ValueError("d_in must be a multiple of group_size")
    if not (50.0 <= percentile <= 100.0) or abs_range < 0:
        raise ValueError("percentile must lie in [50, 100] and abs_range >= 0")
    maxq = 2 ** bits - 1
    Wg = W.reshape(d_out, d_in // group_size, group_size)
    v = np.sort(Wg, axis=2)
    p = percentile / 100.0
    hi = group_quantile(v, p)
    lo = group_quantile(v, 1.0 - p)
    if abs_range > 0:
        lo = np.maximum(lo, -abs_range)
        hi = np.minimum(hi, abs_range)
    Wc = np.clip(Wg, lo[..., None], hi[..., None])
    params = group_params_sym if sym else group_params
    scale, zero = params(lo, hi, maxq)
    q = quantize(Wc, scale[..., None], zero[..., None], maxq)
    return q.reshape(d_out, d_in), scale, zero, lo, hi


def rtn_dequant(codes, scales, zeros, group_size):
    d_out, d_in = codes.shape
    s = np.repeat(scales, group_size, axis=1)
    z = np.repeat(zeros, group_size, axis=1)
    return dequantize(codes, s, z)


def pack_int4(codes):
    """Two 4-bit codes per byte along the input dimension: even column in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    if codes.shape[1] % 2:
        raise ValueError("d_in must be even to pack INT4")
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_int4(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def storage_bits_per_weight(bits, group_size, scale_bits=16, zero_bits=16):
    """Average storage per weight: the code plus the group's scale and zero spread over it."""
    return bits + (scale_bits + zero_bits) / group_size

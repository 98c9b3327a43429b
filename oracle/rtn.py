"""Oracle: group min-max round-to-nearest (RTN) weight quantization (test infrastructure only).

Sources
  * bhfrc.com/news/5741 §2.2: independent min-max per group of ``group_size`` weights.
  * 0539edu.com/news/6111416 §4.2: with fp16 scale and zero per group, 4-bit storage costs
    4 + 32/group_size bits per weight (4.25 / 4.5 / 5 at 128 / 64 / 32).
  * hncyxsy.com/news/243429 §1.2: RTN rounds every weight independently, with no compensation.

Layout: W is [d_out, d_in] (PyTorch Linear layout); groups are ``group_size`` consecutive
input columns of one row. scales and zeros are [d_out, d_in/group_size]. For 4-bit codes the
packed form holds two codes per byte, the even column in the low nibble.
"""

import numpy as np

from .quantizer import group_params, quantize, dequantize


def rtn_minmax(W, bits, group_size):
    """Return (codes int64 [d_out, d_in], scales fp64, zeros fp64 [d_out, d_in/g])."""
    W = np.asarray(W, dtype=np.float64)
    d_out, d_in = W.shape
    if d_in % group_size:
        raise ValueError("d_in must be a multiple of group_size")
    maxq = 2 ** bits - 1
    Wg = W.reshape(d_out, d_in // group_size, group_size)
    scale, zero = group_params(Wg.min(axis=2), Wg.max(axis=2), maxq)
    q = quantize(Wg, scale[..., None], zero[..., None], maxq)
    return q.reshape(d_out, d_in), scale, zero


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

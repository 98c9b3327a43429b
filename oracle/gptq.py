"""Oracle: GPTQ layer-wise quantization with OBS error compensation (test infrastructure only).

Sources
  * hncyxsy.com/news/243429 §2.2: when a column is quantized, the not-yet-quantized columns F
    are corrected with the inverse Hessian restricted to F,
        δ_F = −(w_q − quant(w_q)) / [H_F⁻¹]_qq · (H_F⁻¹)_{q,F}
    (the page's text drops the quantized value from the numerator; this is the OBS/OBQ form it
    names in §1.3 and §2.3).
  * hncyxsy.com/news/243429 §2.4: a fixed column order instead of OBQ's greedy choice; lazy
    batch updates (accumulate the errors of a block of columns, then update all later columns
    at once); a Cholesky factorisation instead of repeated inversion.
  * hncyxsy.com/news/243429 §3.1 steps 1–4: Hessian with damping; Cholesky; per block of 128
    columns, column by column: choose the scale, round, accumulate the error; after the block,
    update the remaining columns; store codes, scales and zeros.
  * hncyxsy.com/news/243429 §3.3 and bhfrc.com/news/5741 §2.3: desc_act / act_order processes
    columns in descending order of the Hessian diagonal (the activation energy 2Σx²).
  * gtnt.cn/news/115337 §4: block_size (default 128) is a multiple of group_size; perc_damp 0.01.

Readings taken where the pages are silent or garbled:
  * Groups are ``group_size`` consecutive columns in processing order; the group's scale and
    zero come from the group's current (already compensated) weights at its first column.
  * act_order sorts diag(H) descending, ties by lower column index first, on the undamped H.
  * Codes come back in the original column order; g_idx[c] is the processing-order group of
    column c; scales/zeros are [d_out, d_in/group_size] in processing-group order.

Two references:
  ``gptq_obs_ref``     column by column with the explicit inverse over the remaining columns,
                       eliminated one column at a time (no Cholesky, no blocking).
  ``gptq_blocked_ref`` the algorithm as the pages lay it out: rows of U (UᵀU = H_d⁻¹), in-block
                       rank-1 updates and one lazy update per block. The GPU is compared
                       against this one; the tests check that both references agree.

Rows of W are independent given H, so both accept ``rows`` to run a subset of rows exactly.
"""

import numpy as np

from .factor import damp, damping, upper_chol_of_inverse, upper_chol_of_inverse_reversed
from .quantizer import group_params, group_params_sym, quantize, dequantize


def act_order_perm(H):
    """Processing order: columns by descending diag(H), ties by lower index (stable)."""
    diag = np.diag(np.asarray(H, dtype=np.float64))
    return np.argsort(-diag, kind="stable")


def _prepare(W, H, percdamp, act_order, rows, need_hd=True):
    """Rows of W, W in the processing order, the order, and (when asked for) the damped
    Hessian in that order; λ always (it does not depend on the order)."""
    W = np.asarray(W, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    if rows is not None:
        W = W[np.asarray(rows)]
    d_in = H.shape[0]
    perm = act_order_perm(H) if act_order else np.arange(d_in)
    if need_hd:
        Hd, lam = damp(H[np.ix_(perm, perm)] if act_order else H, percdamp)
    else:
        Hd, lam = None, damping(H, percdamp)
    return W, W[:, perm].copy(), perm, Hd, lam


def _assemble(codes_p, What_p, scales, zeros, perm, group_size, static_groups=False):
    d_out, d_in = codes_p.shape
    codes = np.empty_like(codes_p)
    codes[:, perm] = codes_p
    What = np.empty_like(What_p)
    What[:, perm] = What_p
    g_idx = np.empty(d_in, dtype=np.int64)
    if static_groups:
        g_idx[:] = np.arange(d_in) // group_size
    else:
        g_idx[perm] = np.arange(d_in) // group_size
    return dict(codes=codes, scales=scales, zeros=zeros, g_idx=g_idx, perm=perm, What=What)


def _check_args(d_in, bits, group_size, block_size=None):
    if not 2 <= bits <= 8:
        raise ValueError("bits must be in [2, 8]")
    if group_size <= 0 or d_in % group_size:
        raise ValueError("d_in must be a multiple of group_size")
    # one group per row (per-channel) has no group boundary inside a block
    if block_size is not None and (block_size <= 0 or
                                   (block_size % group_size and group_size != d_in)):
        raise ValueError("block_size must be a multiple of group_size")


def _params_fn(sym):
    return group_params_sym if sym else group_params


def static_group_params(W0, bits, group_size, sym=False):
    """Scale and zero of every group of the ORIGINAL weights in the original column order
    (groups of ``group_size`` consecutive original columns), as static groups fix them before
    any column is quantized. Returns fp64 arrays [rows, d_in/group_size]."""
    W0 = np.asarray(W0, dtype=np.float64)
    d_out, d_in = W0.shape
    Wg = W0.reshape(d_out, d_in // group_size, group_size)
    return _params_fn(sym)(Wg.min(axis=2), Wg.max(axis=2), 2 ** bits - 1)


def gptq_obs_ref(W, H, bits, group_size, percdamp=0.01, act_order=False, rows=None,
                 sym=False, static_groups=False):
    """Unblocked reference: OBS update with the inverse over the remaining columns. The
    quantizer variants are those of ``gptq_blocked_ref``."""
    d_in = np.asarray(H).shape[0]
    _check_args(d_in, bits, group_size)
    maxq = 2 ** bits - 1
    _, Wp, perm, Hd, _ = _prepare(W, H, percdamp, act_order, rows)
    d_out = Wp.shape[0]
    params = _params_fn(sym)
    Hinv = np.linalg.inv(Hd)                       # inverse over F = all columns
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    What = np.zeros((d_out, d_in))
    if static_groups:
        scales, zeros = static_group_params(np.asarray(W, np.float64)[rows] if rows is not None
                                            else W, bits, group_size, sym)
        col_group = perm // group_size
    else:
        scales = np.zeros((d_out, d_in // group_size))
        zeros = np.zeros((d_out, d_in // group_size))
        col_group = np.arange(d_in) // group_size
    for q in range(d_in):
        if not static_groups and q % group_size == 0:
            grp = Wp[:, q:q + group_size]
            s, z = params(grp.min(axis=1), grp.max(axis=1), maxq)
            scales[:, q // group_size], zeros[:, q // group_size] = s, z
        s, z = scales[:, col_group[q]], zeros[:, col_group[q]]
        w = Wp[:, q].copy()
        codes[:, q] = quantize(w, s, z, maxq)
        What[:, q] = dequantize(codes[:, q], s, z)
        err = (w - What[:, q]) / Hinv[q, q]
        Wp[:, q + 1:] -= np.outer(err, Hinv[q, q + 1:])
        Wp[:, q] = What[:, q]
        # remove column q from F: inverse of H restricted to F \ {q}
        Hinv = Hinv - np.outer(Hinv[:, q], Hinv[q, :]) / Hinv[q, q]
    return _assemble(codes, What, scales, zeros, perm, group_size, static_groups)


def gptq_blocked_ref(W, H, bits, group_size, block_size=128, percdamp=0.01, act_order=False,
                     rows=None, U=None, trace=False, sym=False, static_groups=False):
    """Blocked reference with lazy batch updates, driven by U (UᵀU = H_d⁻¹).

    ``U`` may be passed in when it was already computed by ``prepare_u`` for the same
    (H, percdamp, act_order); rows of W are processed independently either way.

    Quantizer variants: ``sym`` takes the symmetric quantizer (``quantizer.group_params_sym``);
    ``group_size == d_in`` is one group per row (per-channel), whose scale and zero come from
    the whole row before its first column is quantized; ``static_groups`` fixes every group's
    scale and zero from the original weights, groups of consecutive ORIGINAL columns, before
    any column is quantized, and each column then uses the group of its original position
    (g_idx[c] = c // group_size, scales indexed by that group), whatever order act_order gives.

    With ``trace`` the result also holds the values each rounding decision was taken on, in
    the processing order: ``pre`` [d_out, d_in], the compensated weight of every column just
    before it is quantized; ``step`` and ``zquot`` [d_out, d_in/g], each group's unrounded
    step (max − min)/maxq and zero quotient −min/scale (see ``quantizer.group_params``).
    """
    d_in = np.asarray(H).shape[0]
    _check_args(d_in, bits, group_size, block_size)
    maxq = 2 ** bits - 1
    _, Wp, perm, Hd, lam = _prepare(W, H, percdamp, act_order, rows, need_hd=U is None)
    if U is None:
        U = upper_chol_of_inverse(Hd)
    d_out = Wp.shape[0]
    params = _params_fn(sym)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    What = np.zeros((d_out, d_in))
    scales = np.zeros((d_out, d_in // group_size))
    zeros = np.zeros((d_out, d_in // group_size))
    if trace:
        pre = np.zeros((d_out, d_in))
        steps = np.zeros((d_out, d_in // group_size))
        zquots = np.zeros((d_out, d_in // group_size))
    if static_groups:
        W0 = np.empty_like(Wp)
        W0[:, perm] = Wp                          # the original weights, original order
        G0 = W0.reshape(d_out, d_in // group_size, group_size)
        s0, z0, step0, zquot0 = params(G0.min(axis=2), G0.max(axis=2), maxq, trace=True)
        scales[:], zeros[:] = s0, z0
        if trace:
            steps[:], zquots[:] = step0, zquot0
        col_group = perm // group_size            # the group of each processing position
    else:
        col_group = np.arange(d_in) // group_size
    for j0 in range(0, d_in, block_size):
        j1 = min(j0 + block_size, d_in)
        Err = np.zeros((d_out, j1 - j0))
        for q in range(j0, j1):
            if not static_groups and q % group_size == 0:
                grp = Wp[:, q:q + group_size]
                s, z, step, zquot = params(grp.min(axis=1), grp.max(axis=1), maxq, trace=True)
                scales[:, q // group_size], zeros[:, q // group_size] = s, z
                if trace:
                    steps[:, q // group_size], zquots[:, q // group_size] = step, zquot
            s, z = scales[:, col_group[q]], zeros[:, col_group[q]]
            w = Wp[:, q].copy()
            if trace:
                pre[:, q] = w
            codes[:, q] = quantize(w, s, z, maxq)
            What[:, q] = dequantize(codes[:, q], s, z)
            err = (w - What[:, q]) / U[q, q]
            Wp[:, q + 1:j1] -= np.outer(err, U[q, q + 1:j1])
            Wp[:, q] = What[:, q]
            Err[:, q - j0] = err
        Wp[:, j1:] -= Err @ U[j0:j1, j1:]          # lazy batch update of all later columns
    out = _assemble(codes, What, scales, zeros, perm, group_size, static_groups)
    out["lam"] = lam
    if trace:
        out.update(pre=pre, step=steps, zquot=zquots, codes_p=codes)
    return out


def prepare_u(H, percdamp=0.01, act_order=False, route="textbook"):
    """(perm, U) for a Hessian: the processing order and the factor the blocked loop uses.

    ``route`` picks one of the two factorisations in ``factor`` (they agree to rounding, which
    the oracle's tests check): "textbook" (Cholesky, explicit inverse, Cholesky again) or
    "reversed" (one Cholesky of the index-reversed matrix and one triangular solve), the
    cheaper one for the widest layers.
    """
    H = np.asarray(H, dtype=np.float64)
    perm = act_order_perm(H) if act_order else np.arange(H.shape[0])
    Hd, _ = damp(H[np.ix_(perm, perm)] if act_order else H, percdamp)
    if route == "reversed":
        return perm, upper_chol_of_inverse_reversed(Hd)
    if route != "textbook":
        raise ValueError(f"unknown route {route!r}")
    return perm, upper_chol_of_inverse(Hd)

"""Near-tie analysis of GPU GPTQ outputs against the oracle (test helper, CPU side).

GPTQ is a greedy chain over the columns of each row: every rounding decision moves the
not-yet-quantized weights of its row. Two correct implementations that differ only in
rounding order (fp32 on the GPU, fp64 in the oracle) therefore agree bit for bit on a row until
the first column whose value lies so close to a rounding boundary that the two sides may
legitimately round it differently (a near tie). From there on the row follows another, equally
valid, trajectory, and later codes can differ by more than one level.

The criterion applied here, per row, in the processing order:
  * either the row is identical to the oracle's (codes, scales, zeros), or
  * its first difference is an oracle-side near tie: the oracle's own pre-rounding value of
    that decision (``gptq_blocked_ref(..., trace=True)``) lies within the window ``eps`` of
    its rounding boundary. The decisions are the code (t = w/scale near a half-integer), the
    group scale (the unrounded step (max - min)/maxq near an fp16 value) and the group zero
    (-min/scale near a half-integer).

The window is derived, not chosen: it is the largest move of any pre-rounding value (in units
of its group's scale) that a perturbation of H at the Hessian tolerance causes in the oracle
itself, measured before each row's own first divergence, times a safety factor of 2. The rows
it is measured on are a random sample plus every row in which the two results differ, i.e.
every row the criterion is applied to: a maximum taken over a small random sample alone
misses the tail of the rows' sensitivities (a layer's rows differ in their outlier weights
and in how far their compensation reaches). The perturbation moves every entry of H by 1e-5 of its value with a random sign (so its
relative Frobenius norm is the tolerance, 1e-5). That is five times the GPU's measured error
on the diagonal (about 2e-6, a truncation bias of the tensor cores' accumulation) and far above
its error on the off-diagonal entries, whose fp32 partial sums have random signs; the GPU's
fp32 factorisation and column steps add rounding below both.
"""

from __future__ import annotations

import numpy as np

from oracle import gptq as ogptq


def perturbed_hessian(H, rel=1e-5, seed=0, block=2048):
    """H + E with E symmetric and E_ij = rel * H_ij * R_ij, R_ij = +-1 at random: every entry
    moved by the relative tolerance, so ||E||_F = rel * ||H||_F exactly."""
    H = np.asarray(H, dtype=np.float64)
    d = H.shape[0]
    Hp = H.copy()
    rng = np.random.default_rng(seed)
    for i0 in range(0, d, block):
        i1 = min(i0 + block, d)
        for j0 in range(i0, d, block):
            j1 = min(j0 + block, d)
            R = np.where(rng.random((i1 - i0, j1 - j0)) < 0.5, -rel, rel)
            if j0 == i0:
                R = np.triu(R) + np.triu(R, 1).T
            E = H[i0:i1, j0:j1] * R
            Hp[i0:i1, j0:j1] += E
            if j0 != i0:
                Hp[j0:j1, i0:i1] += E.T
    return Hp


def first_divergence(codes_a, codes_b, sc_a, zr_a, sc_b, zr_b, g):
    """Per row: (position, kind) of the first difference in the processing order, kind "none",
    "code" or "param" (a group's scale or zero; its position is the group's first column).
    Codes are [rows, d] in the processing order, scales/zeros [rows, d/g]."""
    d = codes_a.shape[1]
    code_diff = codes_a != codes_b
    par_diff = (sc_a != sc_b) | (zr_a != zr_b)
    fc = np.where(code_diff.any(1), code_diff.argmax(1), d)
    fp = np.where(par_diff.any(1), par_diff.argmax(1) * g, d)
    first = np.minimum(fc, fp)
    kind = np.where(first == d, "none", np.where(fp <= fc, "param", "code"))
    return first, kind


def _code_tie_dist(t):
    """Distance of t to the nearest half-integer (the rounding boundaries of rint)."""
    return np.abs(np.abs(t - np.floor(t)) - 0.5)


def _fp16_below(s):
    return np.nextafter(np.asarray(s, np.float64).astype(np.float16),
                        np.float16(-np.inf)).astype(np.float64)


def window_from_h_sensitivity(W, H, bits, g, B, percdamp, act_order, ref_trace, rows,
                              U_pert=None, H_pert=None, route="textbook", rel=1e-5,
                              safety=2.0, cache=None, **variant):
    """The tie window eps (see the module docstring), from the oracle run on H and on a
    perturbed H over the ``rows``. ``ref_trace`` is the oracle's traced result for those rows
    on H; ``variant`` are the quantizer switches of ``gptq_blocked_ref``. ``cache`` (a dict),
    if given, keeps the perturbed H and its factor for a later call. Returns (eps, detail)."""
    if cache is not None:
        H_pert = cache.get("H_pert", H_pert)
        U_pert = cache.get("U_pert", U_pert)
    if U_pert is None:
        if H_pert is None:
            H_pert = perturbed_hessian(H, rel)
        _, U_pert = ogptq.prepare_u(H_pert, percdamp, act_order, route=route)
    if H_pert is None:
        H_pert = perturbed_hessian(H, rel)
    if cache is not None:
        cache["H_pert"], cache["U_pert"] = H_pert, U_pert
    alt = ogptq.gptq_blocked_ref(W, H_pert, bits, g, B, percdamp, act_order, rows=rows,
                                 U=U_pert, trace=True, **variant)
    first, _ = first_divergence(ref_trace["codes_p"], alt["codes_p"], ref_trace["scales"],
                                ref_trace["zeros"], alt["scales"], alt["zeros"], g)
    moved = np.flatnonzero(alt["perm"] != ref_trace["perm"])
    if moved.size:
        # a perturbation that reorders act_order's keys changes the columns from the first
        # moved position on: compare only the positions before it
        first = np.minimum(first, int(moved[0]))
    if variant.get("static_groups"):
        gi = np.asarray(ref_trace["perm"]) // g
    else:
        gi = np.arange(ref_trace["pre"].shape[1]) // g
    s_col = ref_trace["scales"][:, gi]
    dev = np.abs(ref_trace["pre"] - alt["pre"]) / s_col
    mask = np.arange(dev.shape[1])[None, :] < first[:, None]
    eps_meas = float(np.max(dev[mask])) if mask.any() else 0.0
    detail = dict(eps_measured=eps_meas, rows=int(len(rows)), rel=rel,
                  oracle_rows_diverged=int(np.sum(first < dev.shape[1])),
                  entries_compared=int(mask.sum()))
    return safety * eps_meas, detail


def near_tie_report(codes, scales, zeros, perm, ref_trace, g, bits, eps, rows=None,
                    static_groups=False):
    """Check every row of a GPU result against the oracle's traced result (same rows).

    codes: GPU codes [rows, d] in the ORIGINAL column order; scales/zeros [rows, d/g]; perm the
    GPU's processing order (must equal the oracle's). With static groups every grid is fixed
    from the original weights before the first column, so a grid difference is the row's
    first divergence. Returns a dict of statistics; the parity criterion is
    ``bad_origin == 0``."""
    maxq = 2 ** bits - 1
    codes = np.asarray(codes).astype(np.int64)
    cg = codes[:, perm]
    co = ref_trace["codes_p"].astype(np.int64)
    sg = np.asarray(scales, np.float64)
    zg = np.asarray(zeros, np.float64)
    so, zo = ref_trace["scales"], ref_trace["zeros"]
    first, kind = first_divergence(cg, co, sg, zg, so, zo, g)
    d = cg.shape[1]
    if static_groups:
        grid_diff = np.any((sg != so) | (zg != zo), axis=1)
        kind = np.where(grid_diff, "param", kind)
        k_static = np.where(grid_diff, ((sg != so) | (zg != zo)).argmax(1), 0)
        first = np.where(grid_diff, 0, first)
    diff = cg - co
    bad_rows = []
    for r in np.flatnonzero(first < d):
        q = int(first[r])
        k = int(k_static[r]) if static_groups and kind[r] == "param" else q // g
        if kind[r] == "code":
            kk = int(perm[q]) // g if static_groups else k
            t = ref_trace["pre"][r, q] / so[r, kk]
            ok = _code_tie_dist(t) <= eps
            why = dict(t=float(t), dist=float(_code_tie_dist(t)))
        else:
            s, step, zq = so[r, k], ref_trace["step"][r, k], ref_trace["zquot"][r, k]
            if sg[r, k] != s:
                dist = min(s - step, step - _fp16_below(s))
                ok = dist <= 2.0 * eps * s / maxq
                why = dict(step=float(step), scale=float(s), dist=float(dist))
            else:
                ok = _code_tie_dist(zq) <= eps
                why = dict(zquot=float(zq), dist=float(_code_tie_dist(zq)))
        if not ok:
            bad_rows.append(dict(row=int(r if rows is None else rows[r]), col=q,
                                 kind=str(kind[r]), **why))
    gi = (np.asarray(perm) // g) if static_groups else np.arange(d) // g
    t_all = ref_trace["pre"] / so[:, gi]
    n_near = int(np.sum(_code_tie_dist(t_all) <= eps))
    hist = {int(k): int(v) for k, v in zip(*np.unique(diff, return_counts=True))}
    return dict(rows=int(cg.shape[0]), rows_diverged=int(np.sum(first < d)),
                bad_origin=len(bad_rows), bad_examples=bad_rows[:5],
                agree=float(np.mean(diff == 0)), max_abs_diff=int(np.max(np.abs(diff))),
                beyond_one_level=int(np.sum(np.abs(diff) > 1)), diff_hist=hist,
                oracle_near_ties=n_near, eps=float(eps))

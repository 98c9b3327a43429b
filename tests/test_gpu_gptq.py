"""GPTQ on the GPU against the fp64 oracle.

Tolerances: codes agree on >= 99 % of entries and every mismatch is one level; the layer
reconstruction loss is within 1 % (relative) of the oracle's. With H = c·I the GPU must
reproduce RTN bit for bit. The oracle always starts from X (its own fp64 Hessian); the GPU
path starts from the same X through its tensor-core Hessian.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import factor as ofac
from oracle import gptq as ogptq
from oracle import hessian as ohess
from oracle import loss as oloss
from oracle import rtn as ortn
from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def gpu_hessian(lib, X):
    h = lib.Hessian(X.shape[1])
    h.accumulate(X)
    return h.get()


def log_parity(**rec):
    """Append parity statistics to $GPTQ_PARITY_LOG (a JSON-lines file) when it is set."""
    path = os.environ.get("GPTQ_PARITY_LOG")
    if path:
        rec["test"] = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def compare_codes(got, ref, frac=0.99, max_diff=1):
    diff = got.astype(np.int64) - ref.astype(np.int64)
    agree = float(np.mean(diff == 0))
    hist = {int(k): int(v) for k, v in zip(*np.unique(diff, return_counts=True))}
    log_parity(agree=agree, diff_hist=hist)
    assert agree >= frac, f"codes agree on {agree:.5f}, differences {hist}"
    if max_diff is not None:
        assert np.max(np.abs(diff)) <= max_diff, f"code differences {hist}"
    return agree


def self_consistency(W0p, Whp, codes_p, scales, zeros, Hd, g, bits, tie_tol=0.05):
    """Check every GPU decision against exact arithmetic given the GPU's own earlier decisions.

    With the first q columns (processing order) fixed at the GPU's quantized values, the
    compensated weights of the rest are the least-squares re-solve
        w_R = w_R0 - H_RR^-1 H_RQ (What_Q - w_Q0)
    (fp64, damped H). Column q's code must be the rounding of its re-solved value with the
    GPU's group scale and zero, unless that value lies within `tie_tol` of a rounding boundary;
    group scales must match the re-solved group range to within one fp16 step.
    Returns (non-tie mismatches, near-tie cases, scale mismatches).
    """
    from oracle import quantizer
    maxq = 2 ** bits - 1
    d = W0p.shape[1]
    bad = near = sbad = 0
    for q in range(d):
        if q == 0:
            wR = W0p
        else:
            rhs = Hd[q:, :q] @ (Whp[:, :q] - W0p[:, :q]).T
            wR = W0p[:, q:] - np.linalg.solve(Hd[q:, q:], rhs).T
        if q % g == 0:
            grp = wR[:, :g]
            s_exact, _ = quantizer.group_params(grp.min(1), grp.max(1), maxq)
            s_gpu = scales[:, q // g]
            up = np.nextafter(s_exact.astype(np.float16), np.float16(np.inf)).astype(np.float64)
            dn = np.nextafter(s_exact.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
            sbad += int(np.sum((s_gpu != s_exact) & (s_gpu != up) & (s_gpu != dn)))
        s, z = scales[:, q // g], zeros[:, q // g]
        t = wR[:, 0] / s
        want = np.clip(np.rint(t) + z, 0, maxq)
        dist = np.abs(np.abs(t - np.floor(t)) - 0.5)
        mism = want != codes_p[:, q]
        tie = dist < tie_tol
        bad += int(np.sum(mism & ~tie))
        near += int(np.sum(mism & tie))
    return bad, near, sbad


def recurrence_consistency(Wn, H, out, g, bits, percdamp, rows, tie_tol=0.05):
    """Replay GPTQ in fp64 on `rows` with the GPU's processing order and the GPU's own
    quantization decisions, and check each decision is the rounding of the exactly compensated
    weight (test-side numpy: U is the upper Cholesky factor of the inverse of the damped,
    permuted H built from the fp64 Hessian). Returns (non-tie mismatches, near ties,
    group-scale mismatches beyond one fp16 step)."""
    maxq = 2 ** bits - 1
    perm = out["perm"].cpu().numpy().astype(np.int64)
    d = len(perm)
    Hp = H[np.ix_(perm, perm)]
    lam = percdamp * np.mean(np.diag(Hp))
    L = np.linalg.cholesky(Hp + lam * np.eye(d))
    Linv = np.linalg.solve(L, np.eye(d))
    U = np.linalg.cholesky(Linv.T @ Linv).T
    codes = out["codes"].cpu().numpy()[np.ix_(rows, perm)].astype(np.float64)
    sc = out["scales"].float().cpu().numpy()[rows].astype(np.float64)
    zr = out["zeros"].float().cpu().numpy()[rows].astype(np.float64)
    w = Wn[np.ix_(rows, perm)].copy()
    bad = near = sbad = 0
    for q in range(d):
        gi = q // g
        if q % g == 0:
            grp = w[:, q:q + g]
            span = np.maximum(grp.max(1), 0.0) - np.minimum(grp.min(1), 0.0)
            s_ex = (span / maxq).astype(np.float16).astype(np.float64)
            lo = np.nextafter(s_ex.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
            hi = np.nextafter(np.nextafter(s_ex.astype(np.float16), np.float16(np.inf)),
                              np.float16(np.inf)).astype(np.float64)
            sbad += int(np.sum((sc[:, gi] < lo) | (sc[:, gi] > hi)))
        s, z = sc[:, gi], zr[:, gi]
        t = w[:, q] / s
        want = np.clip(np.rint(t) + z, 0, maxq)
        mism = want != codes[:, q]
        tie = np.abs(np.abs(t - np.floor(t)) - 0.5) < tie_tol
        bad += int(np.sum(mism & ~tie))
        near += int(np.sum(mism & tie))
        what = s * (codes[:, q] - z)
        e = (w[:, q] - what) / U[q, q]
        w[:, q + 1:] -= np.outer(e, U[q, q + 1:])
        w[:, q] = what
    return bad, near, sbad


def adjacent_level(out, ref, g):
    """Largest |What_gpu - What_ref| in units of the oracle's step (<= 1.5 means every mismatch
    is on an adjacent level, also where the two sides' group grids differ)."""
    codes = out["codes"].cpu().numpy().astype(np.float64)
    gi = out["g_idx"].cpu().numpy()
    sc = out["scales"].float().cpu().numpy().astype(np.float64)
    zr = out["zeros"].float().cpu().numpy().astype(np.float64)
    Wg = sc[:, gi] * (codes - zr[:, gi])
    return float(np.max(np.abs(Wg - ref["What"]) / ref["scales"][:, ref["g_idx"]]))


def full_size_checks(out, ref, Wn, Href, g, bits, percdamp=0.01, n_rows=48, rows=None):
    """Parity for full-size layers.

    Target tolerances: >= 99 % identical codes; loss within 1 %; every mismatch one level
    (read as: the reconstructed weight lies within 1.5 oracle steps, which is exactly +-1 code
    where both sides use the same group grid).
    At full size GPTQ's greedy chain makes a few entries cascade: one legitimate near-tie flip
    (fp32 vs fp64) changes that row's compensation for every later column, which can move a
    group's min/max and so its grid. For those the one-level bound is held for >= 99.99 % of
    entries, and a replay proves every GPU decision exact given the GPU's own earlier decisions
    (on the rows with the largest deviations plus random rows), i.e. the rest are cascades,
    not wrong arithmetic."""
    codes = out["codes"].cpu().numpy().astype(np.int64)
    diff = codes - ref["codes"]
    agree = compare_codes(codes, ref["codes"], max_diff=None)
    cg = out["codes"].cpu().numpy().astype(np.float64)
    gi = out["g_idx"].cpu().numpy()
    sc = out["scales"].float().cpu().numpy().astype(np.float64)
    zr = out["zeros"].float().cpu().numpy().astype(np.float64)
    steps = np.abs(sc[:, gi] * (cg - zr[:, gi]) - ref["What"]) / ref["scales"][:, ref["g_idx"]]
    beyond = float(np.mean(steps > 1.5))
    grid_diff = float(np.mean((sc != ref["scales"]) | (zr != ref["zeros"])))
    if rows is None:
        worst = np.argsort(-steps.max(1))[: n_rows // 2]
        rng = np.random.default_rng(0)
        rows = np.unique(np.concatenate([worst, rng.choice(len(codes), n_rows // 2, replace=False)]))
    bad, near, sbad = recurrence_consistency(Wn, Href, out, g, bits, percdamp, rows)
    l_ref = oloss.recon_loss(Wn, ref["What"], Href)
    log_parity(agree=agree, max_steps=float(steps.max()), frac_beyond_one_level=beyond,
               grid_diff_frac=grid_diff, recurrence_bad=bad, recurrence_near=near,
               scale_bad=sbad, loss_lib=out["loss"], loss_ref=l_ref)
    assert beyond <= 1e-4, beyond
    assert bad == 0 and sbad == 0, (bad, near, sbad)
    assert abs(out["loss"] - l_ref) <= 0.01 * l_ref, (out["loss"], l_ref)


def run_case(lib, W, X, bits, g, B, act_order, percdamp=0.01, rows=None):
    H = gpu_hessian(lib, X)
    out = lib.quantize_layer(W, H, bits=bits, group_size=g, block_size=B, percdamp=percdamp,
                             act_order=act_order, compute_loss=True)
    torch.cuda.synchronize()
    Wn = W.float().cpu().numpy().astype(np.float64)
    Href = ohess.hessian(X.cpu().numpy())
    ref = ogptq.gptq_blocked_ref(Wn, Href, bits, g, block_size=B, percdamp=percdamp,
                                 act_order=act_order, rows=rows)
    return out, ref, Wn, Href


def check_outputs(out, ref, Wn, Href, g, perm_must_match=True, max_diff=1):
    perm_gpu = out["perm"].cpu().numpy()
    if perm_must_match:
        assert np.array_equal(perm_gpu, ref["perm"])
    assert np.array_equal(out["g_idx"].cpu().numpy(), ref["g_idx"])
    codes = out["codes"].cpu().numpy()
    agree = compare_codes(codes, ref["codes"], max_diff=max_diff)
    # the GPU's reconstruction, scored with the oracle's loss on the oracle's Hessian
    s = out["scales"].float().cpu().numpy().astype(np.float64)
    z = out["zeros"].float().cpu().numpy().astype(np.float64)
    gi = out["g_idx"].cpu().numpy()
    What = s[:, gi] * (codes - z[:, gi])
    l_gpu = oloss.recon_loss(Wn, What, Href)
    l_ref = oloss.recon_loss(Wn, ref["What"], Href)
    assert abs(l_gpu - l_ref) <= 0.01 * l_ref, (l_gpu, l_ref)
    # the loss the library reports for itself
    log_parity(agree=agree, loss_gpu=l_gpu, loss_lib=out["loss"], loss_ref=l_ref)
    assert abs(out["loss"] - l_ref) <= 0.01 * l_ref, (out["loss"], l_ref)
    return agree, l_gpu, l_ref


@pytest.mark.parametrize("bits,g,B,act_order", [
    (4, 128, 128, False), (4, 128, 128, True), (3, 128, 128, True), (4, 64, 128, False),
    (4, 32, 64, True), (2, 128, 128, False), (8, 128, 128, True), (4, 8, 16, False),
    (3, 2, 16, False)])
def test_linear_512(cuda_lib, bits, g, B, act_order):
    wl = workloads.WORKLOADS["linear_512"]
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    out, ref, Wn, Href = run_case(cuda_lib, W, X, bits, g, B, act_order)
    check_outputs(out, ref, Wn, Href, g)


@pytest.mark.parametrize("d_out,d_in,n,g,B,act_order", [
    (77, 384, 1500, 64, 128, True), (31, 200, 800, 8, 64, False), (64, 264, 900, 8, 128, True),
    (5, 136, 300, 8, 64, False), (129, 1024, 3000, 128, 128, True), (37, 120, 600, 6, 24, True)])
def test_ragged_shapes(cuda_lib, d_out, d_in, n, g, B, act_order):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_out=d_out, d_in=d_in, n_tokens=n, seed=d_in)
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    out, ref, Wn, Href = run_case(cuda_lib, W, X, 4, g, B, act_order)
    check_outputs(out, ref, Wn, Href, g)


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
@pytest.mark.parametrize("act_order", [False, True])
def test_identity_hessian_is_rtn_bit_exact(cuda_lib, dtype, act_order):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_out=300, d_in=768)
    W = workloads.make_weights(wl, device="cuda").to(dtype)
    H = 5.0 * torch.eye(768, device="cuda")
    out = cuda_lib.quantize_layer(W, H, bits=4, group_size=128, act_order=act_order)
    packed, scales, zeros = cuda_lib.rtn_minmax_quantize(W, 4, 128)
    torch.cuda.synchronize()
    rtn_codes = ortn.unpack_int4(packed.cpu().numpy())
    assert np.array_equal(out["codes"].cpu().numpy(), rtn_codes)
    assert torch.equal(out["scales"], scales) and torch.equal(out["zeros"], zeros)
    codes, s_ref, _ = ortn.rtn_minmax(W.float().cpu().numpy().astype(np.float64), 4, 128)
    assert np.array_equal(rtn_codes, codes)


def test_correlated_inputs(cuda_lib):
    """Strongly correlated channels (not one of the named workloads): compensation is large, so
    one legitimate near-tie flip upstream can move later codes by more than one level. Here the
    GPU must agree with the oracle on >= 99 % of codes and on the loss within 1 %, and each of
    its decisions must be exact given its own earlier ones (self-consistency in fp64)."""
    X = workloads.correlated_activations(4096, 256, rank=4, seed=3, device="cuda")
    W = workloads.make_weights(workloads.WORKLOADS["mlp_up_7b"].replace(d_out=192, d_in=256),
                               device="cuda")
    out, ref, Wn, Href = run_case(cuda_lib, W, X, 3, 64, 128, True)
    agree, l_gpu, l_ref = check_outputs(out, ref, Wn, Href, 64, max_diff=None)
    perm = out["perm"].cpu().numpy().astype(np.int64)
    codes = out["codes"].cpu().numpy()[:, perm].astype(np.float64)
    sc = out["scales"].float().cpu().numpy().astype(np.float64)
    zr = out["zeros"].float().cpu().numpy().astype(np.float64)
    Whp = sc[:, np.arange(256) // 64] * (codes - zr[:, np.arange(256) // 64])
    Hd, _ = ofac.damp(Href[np.ix_(perm, perm)], 0.01)
    bad, near, sbad = self_consistency(Wn[:, perm], Whp, codes, sc, zr, Hd, 64, 3)
    log_parity(self_consistency_bad=bad, near_ties=near, scale_bad=sbad, loss_gpu=l_gpu,
               loss_ref=l_ref)
    assert bad == 0 and sbad == 0, (bad, near, sbad)
    # compensation did real work here: GPTQ beats RTN clearly
    codes, s, z = ortn.rtn_minmax(Wn, 3, 64)
    assert l_ref < 0.8 * oloss.recon_loss(Wn, ortn.rtn_dequant(codes, s, z, 64), Href)


@pytest.mark.parametrize("act_order", [False, True])
def test_inverse_factor_matches_oracle(cuda_lib, act_order):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_in=1024, n_tokens=8192, seed=4)
    X = workloads.make_activations(wl, device="cuda")
    H = gpu_hessian(cuda_lib, X)
    U, perm = cuda_lib.inverse_factor(H, 0.01, act_order)
    Ug = U.cpu().numpy().astype(np.float64)
    Href = ohess.hessian(X.cpu().numpy())
    perm_ref, Uref = ogptq.prepare_u(Href, 0.01, act_order)
    assert np.array_equal(perm.cpu().numpy(), perm_ref)
    assert np.array_equal(Ug, np.triu(Ug))
    err = np.max(np.abs(Ug - Uref)) / np.max(np.abs(Uref))
    assert err <= 1e-3, err
    Hd, _ = ofac.damp(Href[np.ix_(perm_ref, perm_ref)], 0.01)
    resid = np.max(np.abs(Ug.T @ Ug @ Hd - np.eye(1024)))
    assert resid <= 1e-3, resid


@pytest.mark.slow
def test_full_size_mlp_up_7b(cuda_lib):
    """The timed workload: W 11008x4096 fp16, X 262144x4096, INT4 g128 B128, all rows."""
    wl = workloads.WORKLOADS["mlp_up_7b"]
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    out, ref, Wn, Href = run_case(cuda_lib, W, X, wl.bits, wl.group_size, wl.block_size,
                                  wl.act_order)
    assert np.array_equal(out["perm"].cpu().numpy(), ref["perm"])
    full_size_checks(out, ref, Wn, Href, wl.group_size, wl.bits)


@pytest.fixture(scope="module")
def mlp_down_inputs():
    """W 4096x11008 and X 262144x11008 (the act_order workload) with the oracle's Hessian."""
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = workloads.WORKLOADS["mlp_down_7b"]
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    Href = ohess.hessian(X.cpu().numpy(), chunk=4096)
    return wl, W, X, Href


@pytest.mark.slow
@pytest.mark.parametrize("bits", [4, 3])
def test_mlp_down_7b_act_order(cuda_lib, mlp_down_inputs, bits):
    """d_in = 11008 with act_order, INT4 and INT3, 262144 calibration tokens."""
    wl, W, X, Href = mlp_down_inputs
    H = gpu_hessian(cuda_lib, X)
    out = cuda_lib.quantize_layer(W, H, bits=bits, group_size=128, act_order=True,
                                  compute_loss=True)
    torch.cuda.synchronize()
    Wn = W.float().cpu().numpy().astype(np.float64)
    ref = ogptq.gptq_blocked_ref(Wn, Href, bits, 128, act_order=True)
    perm_gpu = out["perm"].cpu().numpy()
    moved = np.flatnonzero(perm_gpu != ref["perm"])
    log_parity(perm_positions_moved=int(moved.size))
    # near-equal diagonal entries may swap within the fp32 error of H: both orders are valid
    # processing orders (the replay uses the GPU's); swapped columns leave the code comparison
    assert moved.size <= 8, moved.size
    if moved.size == 0:
        full_size_checks(out, ref, Wn, Href, 128, bits)
    else:
        keep = np.ones(Wn.shape[1], dtype=bool)
        keep[perm_gpu[moved]] = False
        keep[ref["perm"][moved]] = False
        compare_codes(out["codes"].cpu().numpy()[:, keep], ref["codes"][:, keep], max_diff=None)
        rows = np.random.default_rng(0).choice(Wn.shape[0], 24, replace=False)
        bad, near, sbad = recurrence_consistency(Wn, Href, out, 128, bits, 0.01, rows)
        assert bad == 0 and sbad == 0, (bad, near, sbad)
        l_ref = oloss.recon_loss(Wn, ref["What"], Href)
        assert abs(out["loss"] - l_ref) <= 0.01 * l_ref, (out["loss"], l_ref)


@pytest.mark.slow
def test_full_size_attn_o_70b(cuda_lib):
    """The 70B attention-output layer: W 8192x8192 fp16, X 65536x8192, INT4 g128 B128, all rows,
    against the full fp64 oracle."""
    wl = workloads.WORKLOADS["attn_o_70b"]
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    out, ref, Wn, Href = run_case(cuda_lib, W, X, wl.bits, wl.group_size, wl.block_size,
                                  wl.act_order)
    assert np.array_equal(out["perm"].cpu().numpy(), ref["perm"])
    assert np.array_equal(out["g_idx"].cpu().numpy(), ref["g_idx"])
    full_size_checks(out, ref, Wn, Href, wl.group_size, wl.bits)


def recurrence_consistency_dev(W, H, out, g, bits, percdamp, rows, tie_tol=0.05):
    """recurrence_consistency for layers whose d_in makes host fp64 linear algebra too slow: the
    same replay, with the fp64 factorisation and the column steps run by torch on the device.
    U is the upper Cholesky factor of the inverse of the damped, permuted H (here by the index
    reversal: U = flip(chol_lower(flip(H_d))^-1), which satisfies U^T U = H_d^-1)."""
    dev = H.device
    maxq = 2 ** bits - 1
    perm = out["perm"].to(dev).long()
    d = perm.numel()
    Hd = H.double()[perm][:, perm]
    Hd.diagonal().add_(percdamp * torch.mean(torch.diagonal(Hd)))
    L = torch.linalg.cholesky(torch.flip(Hd, [0, 1]))
    del Hd
    eye = torch.eye(d, dtype=torch.float64, device=dev)
    U = torch.flip(torch.linalg.solve_triangular(L, eye, upper=False), [0, 1])
    del L, eye
    r = torch.as_tensor(rows, device=dev).long()
    codes = out["codes"][r][:, perm].double()
    sc = out["scales"][r].double()
    zr = out["zeros"][r].double()
    w = W[r].double()[:, perm].clone()
    bad = near = sbad = 0
    for q in range(d):
        gi = q // g
        if q % g == 0:
            grp = w[:, q:q + g]
            span = (torch.clamp(grp.max(1).values, min=0.0) - torch.clamp(grp.min(1).values, max=0.0))
            s_ex = (span / maxq).cpu().numpy().astype(np.float16)
            lo = np.nextafter(s_ex, np.float16(-np.inf)).astype(np.float64)
            hi = np.nextafter(np.nextafter(s_ex, np.float16(np.inf)), np.float16(np.inf))
            sgi = sc[:, gi].cpu().numpy()
            sbad += int(np.sum((sgi < lo) | (sgi > hi.astype(np.float64))))
        s, z = sc[:, gi], zr[:, gi]
        t = w[:, q] / s
        want = torch.clamp(torch.round(t) + z, 0, maxq)   # torch.round: half to even
        mism = want != codes[:, q]
        tie = torch.abs(torch.abs(t - torch.floor(t)) - 0.5) < tie_tol
        bad += int(torch.sum(mism & ~tie))
        near += int(torch.sum(mism & tie))
        what = s * (codes[:, q] - z)
        e = (w[:, q] - what) / U[q, q]
        w[:, q + 1:] -= torch.outer(e, U[q, q + 1:])
        w[:, q] = what
    return bad, near, sbad


@pytest.mark.slow
def test_mlp_down_70b_sampled(cuda_lib, request):
    """The 70B down projection: W 8192x28672 fp16, X 65536x28672 (3.8 GB), INT4 g128 B128. The
    fp64 oracle is too slow for the whole layer in a test, so parity is checked on sampled
    outputs and through properties that hold at any size:
      * H against the oracle on its diagonal and on a sampled 96x96 block (1e-5 relative);
      * every GPU decision on sampled rows is the rounding of its exactly compensated weight
        (fp64 replay driven by the GPU's own decisions, on the GPU's H, which the first check
        ties to the oracle);
      * the loss the library reports equals tr(ΔHΔᵀ)/tr(WHWᵀ) on that H in fp64 within 1 %;
      * RTN of the same W is bit-exact against the oracle."""
    wl = workloads.WORKLOADS["mlp_down_70b"]
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    H = gpu_hessian(cuda_lib, X)
    d = wl.d_in
    # H: sampled block and diagonal against the oracle
    Xc = X.cpu().numpy()
    del X
    rng = np.random.default_rng(0)
    rows_h = np.sort(rng.choice(d, 96, replace=False))
    cols_h = np.sort(rng.choice(d, 96, replace=False))
    ref_blk = ohess.hessian_entries(Xc, rows_h, cols_h)
    got_blk = H[torch.as_tensor(rows_h, device="cuda")][:, torch.as_tensor(cols_h, device="cuda")]
    got_blk = got_blk.cpu().numpy().astype(np.float64)
    ref_diag = np.empty(d)
    for c0 in range(0, d, 1024):
        x64 = Xc[:, c0:c0 + 1024].astype(np.float64)
        ref_diag[c0:c0 + 1024] = 2.0 * np.einsum("ti,ti->i", x64, x64)
    del Xc, x64
    got_diag = torch.diagonal(H).cpu().numpy().astype(np.float64)

    def rel_fro(a, b):
        return float(np.linalg.norm(a - b) / np.linalg.norm(b))

    log_parity(h_rel_fro_diag=rel_fro(got_diag, ref_diag), h_rel_fro_block=rel_fro(got_blk, ref_blk))
    assert rel_fro(got_diag, ref_diag) <= 1e-5
    assert rel_fro(got_blk, ref_blk) <= 1e-5

    out = cuda_lib.quantize_layer(W, H, bits=wl.bits, group_size=wl.group_size,
                                  block_size=wl.block_size, act_order=wl.act_order,
                                  compute_loss=True)
    torch.cuda.synchronize()
    assert np.array_equal(out["perm"].cpu().numpy(), np.arange(d))
    assert np.array_equal(out["g_idx"].cpu().numpy(), np.arange(d) // wl.group_size)
    codes = out["codes"]
    assert int(codes.max()) <= 2 ** wl.bits - 1
    # the library's loss against tr(ΔHΔᵀ)/tr(WHWᵀ) in fp64 on the same H
    gi = out["g_idx"].long()
    What = out["scales"].double()[:, gi] * (codes.double() - out["zeros"].double()[:, gi])
    W64, H64 = W.double(), H.double()
    D = W64 - What
    l64 = float(torch.sum((D @ H64) * D) / torch.sum((W64 @ H64) * W64))
    del D, What, H64
    log_parity(loss_lib=out["loss"], loss_fp64_same_h=l64)
    assert abs(out["loss"] - l64) <= 0.01 * l64, (out["loss"], l64)
    # replay on sampled rows
    rows = np.sort(rng.choice(wl.d_out, 16, replace=False))
    bad, near, sbad = recurrence_consistency_dev(W, H, out, wl.group_size, wl.bits, 0.01, rows)
    log_parity(recurrence_bad=bad, recurrence_near=near, scale_bad=sbad)
    assert bad == 0 and sbad == 0, (bad, near, sbad)
    # RTN of the same weights, bit-exact
    packed, scales, zeros = cuda_lib.rtn_minmax_quantize(W, wl.bits, wl.group_size)
    torch.cuda.synchronize()
    c_ref, s_ref, z_ref = ortn.rtn_minmax(W.float().cpu().numpy().astype(np.float64), wl.bits,
                                          wl.group_size)
    assert np.array_equal(ortn.unpack_int4(packed.cpu().numpy()), c_ref)
    assert np.array_equal(scales.float().cpu().numpy().astype(np.float64), s_ref)
    assert np.array_equal(zeros.float().cpu().numpy().astype(np.float64), z_ref)

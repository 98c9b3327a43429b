"""Layer-by-layer GPTQ of an MLP block stack on the GPU against the oracle's sequential run.

Both sides run their own chain from the same calibration activations and weights: the GPU
with its tensor-core Hessians, GPTQ kernels, W4A16 layers, RMS pre-norm and SiLU gate; the
oracle in fp64. Only the first layer sees identical inputs on both sides. After it, a
legitimate near-tie flip of one code (one weight moved by one step of its group) changes the
next layers' activations, and so their Hessians, by much more than the Hessian tolerance, and
those layers follow another valid trajectory. So: the first layer is held to the criteria of the
single-layer tests (>= 99 % identical codes, every differing row starting at an oracle-side
near tie, loss within 1 %); every layer's reconstruction loss, a statistic of the whole layer,
is within 1 % of the oracle's; the final activations are within 1e-2 relative Frobenius error;
the code agreement of the later layers is logged. The silu gate and the RMS pre-norm alone are
within one fp16 ulp of the oracle's.
"""

import numpy as np
import pytest
import torch

from gptq_parity import near_tie_report
from oracle import sequential as oseq
from test_gpu_gptq import oracle_ref
from post_weight_quantization_24_b200 import sequential, workloads

pytestmark = pytest.mark.gpu


def _blocks(n_blocks, d, d_ff, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    f = lambda r, c: (0.05 * torch.randn(r, c, generator=g, device="cuda")).to(torch.float16)
    return [(f(d_ff, d), f(d_ff, d), f(d, d_ff)) for _ in range(n_blocks)]


def test_silu_gate_matches_oracle(cuda_lib):
    GU = (3.0 * torch.randn(700, 2 * 264, device="cuda")).to(torch.float16)
    A = cuda_lib.silu_mul(GU)
    torch.cuda.synchronize()
    ref = oseq.silu_mul(GU[:, :264].cpu().numpy(), GU[:, 264:].cpu().numpy())
    got = A.float().cpu().numpy().astype(np.float64)
    ulp = np.abs(np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64))
    assert np.all(np.abs(got - ref) <= ulp)


def test_rms_norm_matches_oracle(cuda_lib):
    X = workloads.make_activations(workloads.WORKLOADS["mlp_up_7b"].replace(
        d_in=520, n_tokens=333, seed=23), device="cuda")
    Y = cuda_lib.rms_norm(X)
    torch.cuda.synchronize()
    ref = oseq.rms_norm(X.cpu().numpy())
    got = Y.float().cpu().numpy().astype(np.float64)
    ulp = np.abs(np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64))
    assert np.all(np.abs(got - ref) <= ulp)


@pytest.mark.parametrize("act_order", [False, True])
def test_sequential_stack_matches_oracle(cuda_lib, act_order):
    d, d_ff, n = 256, 512, 2048
    X0 = workloads.make_activations(workloads.WORKLOADS["mlp_up_7b"].replace(
        d_in=d, n_tokens=n, seed=21), device="cuda")
    blocks = _blocks(2, d, d_ff, seed=22)
    X, recs = sequential.quantize_mlp_stack(X0, blocks, bits=4, group_size=128,
                                            act_order=act_order)
    torch.cuda.synchronize()
    Xr, rrecs = oseq.sequential_mlp_stack(
        X0.cpu().numpy(), [tuple(w.float().cpu().numpy() for w in b) for b in blocks],
        bits=4, group_size=128, act_order=act_order)
    assert len(recs) == len(rrecs) == 4
    stats = []
    for i, (rec, ref) in enumerate(zip(recs, rrecs)):
        codes = rec["codes"].cpu().numpy().astype(np.int64)
        agree = float(np.mean(codes == ref["out"]["codes"]))
        stats.append((rec["name"], agree, rec["loss"], ref["loss"]))
        if i == 0:
            assert agree >= 0.99, (rec["name"], agree)
            g = 128
            W0 = torch.cat([blocks[0][0], blocks[0][1]]).float().cpu().numpy().astype(np.float64)
            tr, eps, _ = oracle_ref(W0, ref["H"], 4, g, 128, act_order)
            rep = near_tie_report(codes, rec["scales"].float().cpu().numpy(),
                                  rec["zeros"].float().cpu().numpy(),
                                  rec["perm"].cpu().numpy().astype(np.int64), tr, g, 4, eps)
            assert rep["bad_origin"] == 0, rep["bad_examples"]
        assert abs(rec["loss"] - ref["loss"]) <= 0.01 * ref["loss"], stats
    got = X.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(got - Xr) / np.linalg.norm(Xr)
    print("sequential stack:", stats, "final rel", rel)
    assert rel <= 1e-2, (rel, stats)

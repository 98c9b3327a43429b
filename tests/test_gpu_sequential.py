"""Layer-by-layer GPTQ of an MLP block stack on the GPU against the oracle's sequential run.

Both sides run their own chain from the same calibration activations and weights: the GPU
with its tensor-core Hessians, GPTQ kernels, W4A16 layers and SiLU gate; the oracle in fp64.
The first layer sees identical inputs on both sides; later layers see activations that differ
by the fp16 roundings of the two chains (the GPU accumulates in fp32), so their Hessians, and
through near ties their codes, can differ slightly. Criteria per layer: >= 99 % identical codes
and the reconstruction loss within 1 % of the oracle's; the final activations within 1e-2
relative Frobenius error (a flipped code moves one weight by one step of its group); the
silu gate alone within one fp16 ulp of the oracle's.
"""

import numpy as np
import pytest
import torch

from oracle import sequential as oseq
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
    for rec, ref in zip(recs, rrecs):
        codes = rec["codes"].cpu().numpy().astype(np.int64)
        agree = float(np.mean(codes == ref["out"]["codes"]))
        assert agree >= 0.99, (rec["name"], agree)
        assert abs(rec["loss"] - ref["loss"]) <= 0.01 * ref["loss"], (rec["name"], rec["loss"],
                                                                       ref["loss"])
    got = X.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(got - Xr) / np.linalg.norm(Xr)
    assert rel <= 1e-2, rel

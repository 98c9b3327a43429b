"""H = 2·XᵀX on the tensor cores against the fp64 oracle.

Integer-valued X makes every product and partial sum exact in fp32, so those cases compare
bit for bit and pin the operand layouts, tile indexing, ragged edges and token tails.
Real-valued X is held to 1e-5 relative Frobenius error."""

import json
import os

import numpy as np
import pytest
import torch

from oracle import hessian as orc
from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def _int_x(n, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randint(-3, 4, (n, d), generator=g, device="cuda").to(torch.float16)


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def log_error(request, **fields):
    """Append the measured errors to $GPTQ_PARITY_LOG (one JSON line), when it is set."""
    path = os.environ.get("GPTQ_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(test=request.node.nodeid, **fields)) + "\n")


@pytest.mark.parametrize("n,d", [(4096, 512), (1000, 200), (77, 8), (130, 264), (64, 128),
                                 (3000, 640), (1, 256)])
def test_integer_inputs_exact(cuda_lib, n, d):
    X = _int_x(n, d, n + d)
    h = cuda_lib.Hessian(d)
    h.accumulate(X)
    H = h.get().cpu().numpy().astype(np.float64)
    ref = orc.hessian(X.cpu().numpy())
    assert np.array_equal(H, ref), f"max abs diff {np.max(np.abs(H - ref))}"
    assert h.tokens == n


def test_accumulates_across_calls_and_reset(cuda_lib):
    X1, X2 = _int_x(700, 136, 1), _int_x(333, 136, 2)
    h = cuda_lib.Hessian(136)
    h.accumulate(X1)
    h.accumulate(X2)
    h.accumulate(X1[:0])
    ref = orc.hessian(np.concatenate([X1.cpu().numpy(), X2.cpu().numpy()]))
    assert np.array_equal(h.get().cpu().numpy().astype(np.float64), ref)
    assert h.tokens == 1033
    h.reset()
    assert torch.count_nonzero(h.get()) == 0


@pytest.mark.parametrize("unit_tokens", [0, 64, 1024, 16384])
def test_linear_512_relative_error(cuda_lib, unit_tokens, request):
    wl = workloads.WORKLOADS["linear_512"]
    X = workloads.make_activations(wl, device="cuda")
    H = torch.zeros(512, 512, device="cuda")
    cuda_lib.hessian_accumulate_into(H, X, unit_tokens=unit_tokens)
    Hg = np.triu(H.cpu().numpy().astype(np.float64))
    ref = np.triu(orc.hessian(X.cpu().numpy()))
    log_error(request, rel_fro=rel_fro(Hg, ref))
    assert rel_fro(Hg, ref) <= 1e-5


def test_full_size_mlp_up_sampled(cuda_lib, request):
    """262144 tokens x 4096 channels, as timed: diagonal plus sampled rows/columns."""
    wl = workloads.WORKLOADS["mlp_up_7b"]
    X = workloads.make_activations(wl, device="cuda")
    h = cuda_lib.Hessian(wl.d_in)
    h.accumulate(X)
    H = h.get()
    Xc = X.cpu().numpy()
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(wl.d_in, 96, replace=False))
    cols = np.sort(rng.choice(wl.d_in, 96, replace=False))
    ref_blk = orc.hessian_entries(Xc, rows, cols)
    got_blk = H[torch.as_tensor(rows, device="cuda")][:, torch.as_tensor(cols, device="cuda")]
    got_blk = got_blk.cpu().numpy().astype(np.float64)
    x64 = Xc.astype(np.float64)
    ref_diag = 2.0 * np.einsum("ti,ti->i", x64, x64)
    got_diag = torch.diagonal(H).cpu().numpy().astype(np.float64)
    scale = np.sqrt(np.outer(ref_diag[rows], ref_diag[cols]))
    log_error(request, rel_fro_diag=rel_fro(got_diag, ref_diag), rel_fro_block=rel_fro(got_blk, ref_blk),
              max_entry_rel=float(np.max(np.abs(got_blk - ref_blk) / scale)),
              mean_rel_bias_diag=float(np.mean((got_diag - ref_diag) / ref_diag)))
    assert rel_fro(got_diag, ref_diag) <= 1e-5
    assert rel_fro(got_blk, ref_blk) <= 1e-5
    # every sampled entry individually, relative to its row/column scale
    assert np.max(np.abs(got_blk - ref_blk) / scale) <= 2e-5


def test_symmetric_mirror(cuda_lib):
    X = _int_x(500, 392, 5)
    h = cuda_lib.Hessian(392)
    h.accumulate(X)
    H = h.get()
    assert torch.equal(H, H.T)
    raw = h.raw()
    assert torch.equal(torch.triu(raw), torch.triu(H))

"""AWQ-lite on the GPU against the oracle.

The channel means are fp64 sums on both sides, so the fp16 scales s agree bit for bit. The
losses are accumulated in fp32 (3xTF32 GEMM) against fp64: within 1e-4 relative. The chosen α
equals the oracle's unless the oracle's own losses of the two choices lie within that
tolerance of each other (a near tie of the search); for the chosen α the codes, scales, zeros
and s are bit-exact (RTN of W·s with exact products)."""

import numpy as np
import pytest
import torch

from oracle import awq as oawq
from oracle import hessian as ohess
from oracle import rtn as ortn
from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def test_channel_abs_sum(cuda_lib):
    X = workloads.make_activations(workloads.WORKLOADS["mlp_up_7b"].replace(
        d_in=1000, n_tokens=3001, seed=3), device="cuda")
    sums = cuda_lib.channel_abs_sum(X)
    sums = cuda_lib.channel_abs_sum(X[:1000], sums)      # accumulates over batches
    torch.cuda.synchronize()
    Xn = X.cpu().numpy().astype(np.float64)
    ref = np.sum(np.abs(Xn), axis=0) + np.sum(np.abs(Xn[:1000]), axis=0)
    assert np.allclose(sums.cpu().numpy(), ref, rtol=1e-12, atol=0)


@pytest.mark.parametrize("bits,g,sym", [(4, 128, False), (3, 64, False), (4, 32, True)])
def test_awq_lite_matches_oracle(cuda_lib, bits, g, sym):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_out=512, d_in=1024, n_tokens=8192, seed=g)
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    h = cuda_lib.Hessian(1024)
    h.accumulate(X)
    H = h.get()
    sums = cuda_lib.channel_abs_sum(X)
    res = cuda_lib.awq_lite_search(W, sums, X.shape[0], H, bits=bits, group_size=g, sym=sym)
    torch.cuda.synchronize()
    Xn = X.cpu().numpy()
    Href = ohess.hessian(Xn)
    Wn = W.float().cpu().numpy().astype(np.float64)
    ref = oawq.awq_lite(Wn, oawq.channel_mean_abs(Xn), Href, bits, g, sym=sym)
    L = np.array(res["losses"])
    assert np.allclose(L, ref["losses"], rtol=1e-4, atol=0), (L, ref["losses"])
    b = res["best"]
    if b != ref["best"]:
        la, lb = ref["losses"][b], ref["losses"][ref["best"]]
        assert abs(la - lb) <= 1e-4 * lb, (b, ref["best"], la, lb)
        return
    assert np.array_equal(res["s"].float().cpu().numpy().astype(np.float64), ref["s"])
    codes = res["packed"].cpu().numpy()
    if bits == 4:
        codes = ortn.unpack_int4(codes)
    assert np.array_equal(codes, ref["codes"])
    assert np.array_equal(res["scales"].float().cpu().numpy().astype(np.float64), ref["scales"])
    assert np.array_equal(res["zeros"].float().cpu().numpy().astype(np.float64), ref["zeros"])

"""The W4A16 layer (w4a16_pack, w4a16_linear) against the oracle's fp64 layer.

Tolerance, derived from the arithmetic: the reconstructed fp16 weights and the fp16 x fp16
products are exact in fp32, the tensor cores accumulate d_in products in fp32 (at most about
d_in/16 accumulator additions per output, each with a relative error below 2^-22 allowing for
truncation), the residual is added in fp32, and both sides round once to fp16. So
|Y_gpu - Y_ref| <= (d_in/16 + 2)·2^-22·Σ|x·ŵ| + 2^-23·|R| + one fp16 ulp of |Y_ref|.
The packing is compared byte for byte with the codes in the processing order.
"""

import numpy as np
import pytest
import torch

from oracle import hessian as ohess
from oracle import w4a16 as ow4
from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def _quantized_layer(lib, d_out, d_in, n_cal, g, act_order, seed, static_groups=False):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_out=d_out, d_in=d_in, n_tokens=n_cal,
                                                  seed=seed)
    W = workloads.make_weights(wl, device="cuda")
    Xc = workloads.make_activations(wl, device="cuda")
    h = lib.Hessian(d_in)
    h.accumulate(Xc)
    out = lib.quantize_layer(W, h.get(), bits=4, group_size=g, act_order=act_order,
                             static_groups=static_groups)
    return W, out


def _check(Y, X, codes, scales, zeros, g_idx, R=None):
    Xn = X.cpu().numpy()
    Rn = None if R is None else R.cpu().numpy()
    Y16, Yx = ow4.w4a16_linear(Xn, codes, scales, zeros, g_idx, R=Rn)
    mag = ow4.abs_products(Xn, codes, scales, zeros, g_idx)
    d_in = Xn.shape[1]
    tol = (d_in / 16 + 2) * 2.0 ** -22 * mag
    if Rn is not None:
        tol += 2.0 ** -23 * np.abs(Rn.astype(np.float64))
    tol += np.abs(np.spacing(np.abs(Yx).astype(np.float16)).astype(np.float64))
    got = Y.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - Y16)
    assert np.all(np.isfinite(got))
    assert np.all(err <= tol), (float(np.max(err / tol)), int(np.sum(err > tol)))
    return float(np.max(err / np.maximum(np.abs(Y16), 1e-30)))


@pytest.mark.parametrize("n,d_out,d_in,g,act_order", [
    (300, 264, 512, 128, False),       # ragged token and channel tiles
    (1000, 512, 1024, 64, True),       # act_order: perm gather on both sides
    (129, 1024, 768, 32, True),
    (64, 4096, 4096, 128, False),
])
def test_w4a16_matches_oracle(cuda_lib, n, d_out, d_in, g, act_order):
    W, out = _quantized_layer(cuda_lib, d_out, d_in, 4096, g, act_order, seed=n)
    perm = out["perm"] if act_order else None
    packed = cuda_lib.w4a16_pack(out["codes"], perm)
    X = workloads.make_activations(
        workloads.WORKLOADS["mlp_up_7b"].replace(d_in=d_in, n_tokens=n, seed=n + 1), device="cuda")
    Y = cuda_lib.w4a16_linear(X, packed, out["scales"], out["zeros"], g, perm=perm)
    torch.cuda.synchronize()
    codes = out["codes"].cpu().numpy()
    p = np.arange(d_in) if perm is None else perm.cpu().numpy()
    ref_packed = (codes[:, p][:, 0::2] & 0xF) | ((codes[:, p][:, 1::2] & 0xF) << 4)
    assert np.array_equal(packed.cpu().numpy(), ref_packed)
    _check(Y, X, codes, out["scales"].float().cpu().numpy(), out["zeros"].float().cpu().numpy(),
           out["g_idx"].cpu().numpy())


def test_w4a16_residual_in_place_and_static_groups(cuda_lib):
    """Y = X·Ŵᵀ + R written over R, with static groups (original-order groups, no gather)."""
    n, d_out, d_in, g = 500, 768, 768, 128
    W, out = _quantized_layer(cuda_lib, d_out, d_in, 4096, g, True, seed=5, static_groups=True)
    packed = cuda_lib.w4a16_pack(out["codes"])
    X = workloads.make_activations(
        workloads.WORKLOADS["mlp_up_7b"].replace(d_in=d_in, n_tokens=n, seed=6), device="cuda")
    R = torch.randn(n, d_out, device="cuda").to(torch.float16)
    R0 = R.clone()
    cuda_lib.w4a16_linear(X, packed, out["scales"], out["zeros"], g, R=R, out=R)
    torch.cuda.synchronize()
    _check(R, X, out["codes"].cpu().numpy(), out["scales"].float().cpu().numpy(),
           out["zeros"].float().cpu().numpy(), out["g_idx"].cpu().numpy(), R=R0)


def test_w4a16_rtn_packing_is_the_rtn_layout(cuda_lib):
    """RTN's packed output (even column in the low nibble) is the layout w4a16_pack writes
    without a perm, so an RTN checkpoint feeds the layer directly."""
    W = workloads.make_weights(workloads.WORKLOADS["mlp_up_7b"].replace(d_out=512, d_in=1024),
                               device="cuda")
    packed, scales, zeros = cuda_lib.rtn_minmax_quantize(W, 4, 128)
    from oracle import rtn as ortn
    codes = torch.from_numpy(ortn.unpack_int4(packed.cpu().numpy())).cuda()
    assert torch.equal(cuda_lib.w4a16_pack(codes), packed)
    X = workloads.make_activations(
        workloads.WORKLOADS["mlp_up_7b"].replace(d_in=1024, n_tokens=256, seed=8), device="cuda")
    Y = cuda_lib.w4a16_linear(X, packed, scales, zeros, 128)
    torch.cuda.synchronize()
    _check(Y, X, codes.cpu().numpy(), scales.float().cpu().numpy(),
           zeros.float().cpu().numpy(), np.arange(1024) // 128)


def test_w4a16_argument_checks(cuda_lib):
    X = torch.zeros(16, 100, dtype=torch.float16, device="cuda")
    packed = torch.zeros(64, 50, dtype=torch.uint8, device="cuda")
    s = torch.ones(64, 1, dtype=torch.float16, device="cuda")
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.w4a16_linear(X, packed, s, s, 100)        # d_in not a multiple of 64
    assert e.value.name == "GPTQ_ERR_ARG"

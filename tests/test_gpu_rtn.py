"""RTN on the GPU against the fp64 oracle: codes, scales and zeros bit-exact."""

import numpy as np
import pytest
import torch

from oracle import rtn as orc
from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def check_rtn(gptq, W, bits, g):
    packed, scales, zeros = gptq.rtn_minmax_quantize(W, bits, g)
    torch.cuda.synchronize()
    Wn = W.float().cpu().numpy().astype(np.float64)
    codes, s_ref, z_ref = orc.rtn_minmax(Wn, bits, g)
    got = packed.cpu().numpy()
    if bits == 4:
        got = orc.unpack_int4(got)
    assert got.shape == codes.shape
    mism = np.count_nonzero(got != codes)
    assert mism == 0, f"{mism} code mismatches"
    assert np.array_equal(scales.float().cpu().numpy().astype(np.float64), s_ref)
    assert np.array_equal(zeros.cpu().numpy(), z_ref.astype(np.float16))


def _w(d_out, d_in, dtype, seed, outliers=True):
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = torch.randn(d_out, d_in, generator=g, device="cuda") * 0.02
    if outliers:
        W[:, : max(1, d_in // 100)] *= 20
    return W.to(dtype)


def test_linear_512_fp32(cuda_lib):
    wl = workloads.WORKLOADS["linear_512"]
    W = workloads.make_weights(wl, device="cuda")
    check_rtn(cuda_lib, W, 4, 128)


@pytest.mark.parametrize("bits,g", [(4, 128), (4, 64), (4, 32), (4, 16), (4, 8), (3, 128),
                                    (2, 64), (8, 128), (4, 256), (5, 32)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
def test_ragged_rows_all_group_sizes(cuda_lib, bits, g, dtype):
    check_rtn(cuda_lib, _w(77, 512, dtype, bits * 1000 + g), bits, g)


@pytest.mark.parametrize("d_in,g,bits", [(96, 24, 4), (120, 40, 3), (72, 72, 4), (80, 10, 2)])
def test_generic_group_sizes(cuda_lib, d_in, g, bits):
    check_rtn(cuda_lib, _w(33, d_in, torch.float16, d_in + g), bits, g)


def test_degenerate_and_tie_groups(cuda_lib):
    rows = []
    rows.append(np.full(32, 0.3))                                   # constant: scale 1
    rows.append(np.abs(np.random.default_rng(0).standard_normal(32)) + 4.0)   # no zero in range
    rows.append(np.random.default_rng(1).standard_normal(32) * 1e-6)  # fp16 subnormal scale
    tie = np.array([0.0, 15 / 16] + [(k + 0.5) / 16 for k in range(15)] + [k / 16 for k in range(15)])
    rows.append(tie)                                                # exact halves: scale 1/16
    rows.append(-np.abs(np.random.default_rng(2).standard_normal(32)) - 100.0)
    W = torch.tensor(np.stack(rows), dtype=torch.float16, device="cuda")
    W = torch.cat([W, W.float().neg().half()], 0).contiguous()
    for bits in (2, 4, 8):
        check_rtn(cuda_lib, W, bits, 32)
        check_rtn(cuda_lib, W.float().contiguous(), bits, 16)


@pytest.mark.parametrize("name,bits", [("mlp_up_7b", 4), ("mlp_down_7b", 4), ("mlp_down_7b", 3)])
def test_full_size_weights(cuda_lib, name, bits):
    wl = workloads.WORKLOADS[name]
    W = workloads.make_weights(wl, device="cuda")
    check_rtn(cuda_lib, W, bits, 128)


def test_empty_rows_rejected(cuda_lib):
    W = torch.empty(0, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(cuda_lib.GPTQError):
        cuda_lib.rtn_minmax_quantize(W, 4, 128)

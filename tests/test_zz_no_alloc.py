"""gptq_quantize_layer_noalloc, the quantizer for callers that may not allocate device memory.

Such callers (a runtime whose pools already hold nearly all of the GPU, a deployment that
forbids allocation after start-up) cannot pass a workspace, so this entry point uses the
library's fixed 32 MiB device scratch instead. The test calls it through the C ABI twice on
one layer, with another layer through the same scratch in between, and checks each result
against the workspace-taking gptq_quantize_layer on the same inputs: codes, scales, zeros,
g_idx and perm bit for bit (the same deterministic kernels run on the same H), the loss to
1e-5. It also checks that a layer too large for the scratch is refused.
This file is collected last so a stop-at-first-failure run has run everything else first.
"""

import ctypes

import numpy as np
import pytest
import torch

from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def _inputs(lib, d_out, d_in, n, seed):
    wl = workloads.WORKLOADS["mlp_up_7b"].replace(d_out=d_out, d_in=d_in, n_tokens=n, seed=seed)
    W = workloads.make_weights(wl, device="cuda")
    X = workloads.make_activations(wl, device="cuda")
    h = lib.Hessian(d_in)
    h.accumulate(X)
    return W, h.get()


def _noalloc_via_abi(lib, W, H, bits, g, B, act_order):
    """Call the C entry point directly with caller-owned output buffers."""
    d_out, d_in = W.shape
    codes = torch.empty(d_out, d_in, dtype=torch.uint8, device="cuda")
    scales = torch.empty(d_out, d_in // g, dtype=torch.float16, device="cuda")
    zeros = torch.empty(d_out, d_in // g, dtype=torch.float16, device="cuda")
    g_idx = torch.empty(d_in, dtype=torch.int32, device="cuda")
    perm = torch.empty(d_in, dtype=torch.int32, device="cuda")
    loss = ctypes.c_float(float("nan"))
    st = lib.lib().gptq_quantize_layer_noalloc(
        W.data_ptr(), lib.DTYPE_F16 if W.dtype == torch.float16 else lib.DTYPE_F32, d_out, d_in,
        H.data_ptr(), bits, g, B, 0.01, int(act_order), codes.data_ptr(), scales.data_ptr(),
        zeros.data_ptr(), g_idx.data_ptr(), perm.data_ptr(), ctypes.byref(loss),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.status_string(st)
    return dict(codes=codes, scales=scales, zeros=zeros, g_idx=g_idx, perm=perm,
                loss=float(loss.value))


def _workspace_call(lib, W, H, bits, g, B, act_order):
    """The workspace-taking entry point, with a fresh workspace filled with NaN bytes: any
    scratch byte read before it is written would show up in the result."""
    ws = torch.full((lib.quantize_layer_workspace(*W.shape, B),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    return lib.quantize_layer(W, H, bits=bits, group_size=g, block_size=B, act_order=act_order,
                              compute_loss=True, workspace=ws)


def _identical(a, b):
    """Both entry points run the same deterministic kernels on the same H: outputs are
    bit-identical. The loss sums fp64 partial sums with atomics, whose order may differ."""
    for k in ("codes", "scales", "zeros", "g_idx", "perm"):
        assert torch.equal(a[k], b[k]), k
    assert abs(a["loss"] - b["loss"]) <= 1e-5 * b["loss"]


@pytest.mark.parametrize("d_out,d_in,n,bits,g,B,act_order", [
    (512, 512, 2048, 4, 128, 128, False),
    (1000, 1024, 4096, 3, 64, 128, True),
])
def test_noalloc_matches_workspace_entry_point_twice(cuda_lib, d_out, d_in, n, bits, g, B,
                                                     act_order):
    """Two no-allocation calls with a different layer (another shape, group size, bit width and
    act_order setting) run through the same scratch in between: each equals the workspace
    entry point's result bit for bit, so nothing left in the scratch leaks into a call."""
    W, H = _inputs(cuda_lib, d_out, d_in, n, seed=d_in)
    W2, H2 = _inputs(cuda_lib, 700, 768, 3000, seed=77)
    ref = _workspace_call(cuda_lib, W, H, bits, g, B, act_order)
    ref2 = _workspace_call(cuda_lib, W2, H2, 2, 32, 64, not act_order)
    first = _noalloc_via_abi(cuda_lib, W, H, bits, g, B, act_order)
    other = _noalloc_via_abi(cuda_lib, W2, H2, 2, 32, 64, not act_order)
    second = _noalloc_via_abi(cuda_lib, W, H, bits, g, B, act_order)
    torch.cuda.synchronize()
    _identical(first, ref)
    _identical(other, ref2)
    _identical(second, ref)


def test_noalloc_refuses_layers_larger_than_its_scratch(cuda_lib):
    W = torch.zeros(4096, 4096, dtype=torch.float16, device="cuda")
    H = torch.eye(4096, device="cuda")
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.quantize_layer_noalloc(W, H)
    assert e.value.name == "GPTQ_ERR_WORKSPACE"

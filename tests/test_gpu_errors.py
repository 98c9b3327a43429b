"""Device-detected failures come back as status codes (no GPU fault is ever provoked)."""

import pytest
import torch

from post_weight_quantization_24_b200 import workloads

pytestmark = pytest.mark.gpu


def _w(d_out=64, d_in=256):
    return workloads.make_weights(workloads.WORKLOADS["mlp_up_7b"].replace(d_out=d_out, d_in=d_in),
                                  device="cuda")


def test_zero_activations_not_pd(cuda_lib):
    h = cuda_lib.Hessian(256)
    h.accumulate(torch.zeros(512, 256, dtype=torch.float16, device="cuda"))
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.quantize_layer(_w(), h.get())
    assert e.value.name == "GPTQ_ERR_NOT_PD"
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.inverse_factor(h.get())
    assert e.value.name == "GPTQ_ERR_NOT_PD"


def test_indefinite_hessian_not_pd_from_cholesky_pivot(cuda_lib):
    d = 256
    H = torch.eye(d, device="cuda")
    H[0, 1] = H[1, 0] = 3.0          # 2x2 block [[1,3],[3,1]] is indefinite; mean diag stays 1
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.quantize_layer(_w(d_in=d), H, percdamp=0.01)
    assert e.value.name == "GPTQ_ERR_NOT_PD"


def test_nonfinite_inputs(cuda_lib):
    X = workloads.make_activations(workloads.WORKLOADS["linear_512"].replace(d_in=256),
                                   device="cuda", n_tokens=1024, d_in=256)
    h = cuda_lib.Hessian(256)
    h.accumulate(X)
    H = h.get()
    W = _w()
    W[3, 7] = float("nan")
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.quantize_layer(W, H)
    assert e.value.name == "GPTQ_ERR_NONFINITE"
    H2 = H.clone()
    H2[5, 9] = float("inf")
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.quantize_layer(_w(), H2)
    assert e.value.name == "GPTQ_ERR_NONFINITE"
    # the library recovers: a clean call right after succeeds
    out = cuda_lib.quantize_layer(_w(), H)
    assert out["codes"].shape == (64, 256)


def test_workspace_too_small(cuda_lib):
    H = torch.eye(256, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(cuda_lib.GPTQError) as e:
        cuda_lib.quantize_layer(_w(), H, workspace=ws)
    assert e.value.name == "GPTQ_ERR_WORKSPACE"


def test_bad_arguments(cuda_lib):
    H = torch.eye(256, device="cuda")
    for kw in (dict(bits=1), dict(group_size=96), dict(block_size=96, group_size=64),
               dict(percdamp=-0.5)):
        with pytest.raises(cuda_lib.GPTQError) as e:
            cuda_lib.quantize_layer(_w(), H, **kw)
        assert e.value.name == "GPTQ_ERR_ARG"


def test_bounded_wait_gives_timeout_and_the_library_recovers(cuda_lib):
    """The factorisation's diagonal-block kernel is switched to wait on an mbarrier that nothing
    arrives at. Its bounded wait gives up after about 1 ms: the call returns GPTQ_ERR_TIMEOUT
    (no hang, no fault), and with the switch off again the next call succeeds and matches a
    call made before the stall."""
    X = workloads.make_activations(workloads.WORKLOADS["linear_512"].replace(d_in=256),
                                   device="cuda", n_tokens=2048, d_in=256)
    h = cuda_lib.Hessian(256)
    h.accumulate(X)
    H = h.get()
    W = _w()
    before = cuda_lib.quantize_layer(W, H, compute_loss=True)
    codes_before = before["codes"].clone()
    cuda_lib.test_stall_factor(True)
    try:
        with pytest.raises(cuda_lib.GPTQError) as e:
            cuda_lib.inverse_factor(H)
        assert e.value.name == "GPTQ_ERR_TIMEOUT"
        with pytest.raises(cuda_lib.GPTQError) as e:
            cuda_lib.quantize_layer(W, H)
        assert e.value.name == "GPTQ_ERR_TIMEOUT"
    finally:
        cuda_lib.test_stall_factor(False)
    after = cuda_lib.quantize_layer(W, H, compute_loss=True)
    assert torch.equal(after["codes"], codes_before)
    assert torch.equal(after["scales"], before["scales"])

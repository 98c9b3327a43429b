"""The seeded input generators hold to their recipe (CPU): weight outlier columns, per-channel
activation magnitudes with outlier channels, fp16 storage, determinism per seed, and the named
layer shapes."""

import numpy as np
import pytest
import torch

from post_weight_quantization_24_b200 import workloads as wk


def test_named_workloads_have_the_documented_shapes():
    W = wk.WORKLOADS
    assert (W["linear_512"].d_out, W["linear_512"].d_in, W["linear_512"].n_tokens) == (512, 512, 2048)
    assert (W["mlp_up_7b"].d_out, W["mlp_up_7b"].d_in, W["mlp_up_7b"].n_tokens) == (11008, 4096, 262144)
    assert (W["mlp_down_7b"].d_out, W["mlp_down_7b"].d_in) == (4096, 11008) and W["mlp_down_7b"].act_order
    assert (W["attn_o_70b"].d_out, W["attn_o_70b"].d_in, W["attn_o_70b"].n_tokens) == (8192, 8192, 65536)
    assert (W["mlp_down_70b"].d_out, W["mlp_down_70b"].d_in) == (8192, 28672)
    for wl in W.values():
        assert (wl.bits, wl.group_size, wl.block_size, wl.percdamp) == (4, 128, 128, 0.01)
    # one 7B decoder layer: 7 linears reading 4 distinct inputs
    assert len(wk.DECODER_7B_LINEARS) == 7
    assert {src for *_, src in wk.DECODER_7B_LINEARS} == set(wk.DECODER_7B_INPUTS)
    for _, d_out, d_in, src in wk.DECODER_7B_LINEARS:
        assert wk.DECODER_7B_INPUTS[src] == d_in


def test_weights_outlier_columns_and_scale():
    wl = wk.WORKLOADS["mlp_up_7b"].replace(d_out=2048, d_in=4096)
    W = wk.make_weights(wl).float()
    assert W.dtype == torch.float32 and wk.make_weights(wl).dtype == torch.float16
    col_std = W.std(dim=0).numpy()
    k = int(round(wl.w_outlier_frac * wl.d_in))
    assert k == 4
    big = np.flatnonzero(col_std > 5 * wl.w_std)
    assert big.size == k                                   # exactly round(0.1 % d_in) columns
    assert np.allclose(col_std[big], wl.w_std * wl.w_outlier_scale, rtol=0.1)
    rest = np.delete(col_std, big)
    assert abs(rest.mean() - wl.w_std) < 0.02 * wl.w_std


def test_channel_magnitudes_lognormal_with_outlier_channels():
    base = wk.channel_magnitudes(4096, 1.0, 0, 50.0, seed=3)
    m = wk.channel_magnitudes(4096, 1.0, 6, 50.0, seed=3)
    ratio = (m / base).numpy()
    assert np.sum(np.isclose(ratio, 50.0)) == 6 and np.sum(np.isclose(ratio, 1.0)) == 4090
    logm = np.log(base.numpy())
    assert abs(logm.mean()) < 0.06 and abs(logm.std() - 1.0) < 0.05


def test_activations_are_fp16_with_per_channel_magnitudes():
    wl = wk.WORKLOADS["mlp_up_7b"].replace(d_in=64, n_tokens=20000)
    X = wk.make_activations(wl)
    assert X.dtype == torch.float16 and X.shape == (20000, 64)
    mags = wk.channel_magnitudes(64, wl.x_sigma, wl.x_outlier_channels, wl.x_outlier_scale, wl.seed)
    est = X.float().std(dim=0) / mags
    assert torch.all((est > 0.97) & (est < 1.03)), est


def test_generators_are_deterministic_per_seed():
    wl = wk.WORKLOADS["linear_512"]
    assert torch.equal(wk.make_weights(wl), wk.make_weights(wl))
    assert torch.equal(wk.make_activations(wl), wk.make_activations(wl))
    assert not torch.equal(wk.make_weights(wl), wk.make_weights(wl, seed=1))
    assert not torch.equal(wk.make_activations(wl), wk.make_activations(wl, seed=1))
    assert wk.make_weights(wl).dtype == torch.float32      # linear_512 keeps fp32 weights


@pytest.mark.parametrize("rank", [2, 4])
def test_correlated_activations_are_strongly_correlated(rank):
    X = wk.correlated_activations(4096, 64, rank=rank, seed=3).double().numpy()
    C = np.corrcoef(X.T)
    off = np.abs(C[~np.eye(64, dtype=bool)])
    assert np.median(off) > 0.2                             # independent channels: about 0.01

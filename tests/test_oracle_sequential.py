"""Pins for the sequential (layer-by-layer) GPTQ oracle.

* silu: silu(0) = 0, silu(g) − silu(−g) = g, and silu(g) → g for large g; the fp16 result is
  the rounding of the fp64 one.
* Near-lossless quantization (8 bits, small groups) makes the sequential stack follow the
  unquantized stack closely, block after block.
* The error propagates: the Hessian of the down projection, and the input of the next block,
  change when the gate/up projection of the same block is quantized more coarsely, and with
  8-bit layers they approach the ones of the unquantized forward pass.
"""

import numpy as np

from oracle import hessian, sequential
from post_weight_quantization_24_b200 import workloads


def _stack(n_blocks=2, d=64, d_ff=128, n=512, seed=0):
    rng = np.random.default_rng(seed)
    X = workloads.make_activations(workloads.WORKLOADS["mlp_up_7b"].replace(
        d_in=d, n_tokens=n, seed=seed, x_outlier_channels=2)).numpy()
    blocks = []
    for _ in range(n_blocks):
        f = lambda r, c: (rng.standard_normal((r, c)) * 0.05).astype(np.float16).astype(np.float64)
        blocks.append((f(d_ff, d), f(d_ff, d), f(d, d_ff)))
    return X, blocks


def test_silu_closed_forms():
    g = np.array([0.0, 1.5, -1.5, 30.0, -30.0], dtype=np.float16)
    one = np.ones_like(g)
    s = sequential.silu_mul(g, one)
    assert s[0] == 0.0
    assert abs((s[1] - s[2]) - 1.5) <= 2e-3            # silu(g) - silu(-g) = g (fp16 outputs)
    assert s[3] == 30.0 and abs(s[4]) < 1e-10
    exact = g.astype(np.float64) / (1 + np.exp(-g.astype(np.float64)))
    assert np.array_equal(s, exact.astype(np.float16).astype(np.float64))


def test_rms_norm_closed_forms():
    X = np.array([[3.0, 4.0], [0.0, 0.0], [-2.0, 2.0]], dtype=np.float16)
    Nx = sequential.rms_norm(X)
    # rms of (3, 4) is sqrt(12.5): outputs 3/sqrt(12.5), 4/sqrt(12.5); an all-zero row stays 0
    assert np.allclose(Nx[0], np.array([3, 4]) / np.sqrt(12.5 + 1e-6), rtol=1e-3)
    assert np.array_equal(Nx[1], [0.0, 0.0])
    assert np.allclose(np.mean(Nx[2] ** 2), 1.0, rtol=1e-3)


def test_eight_bit_stack_follows_the_float_stack():
    X, blocks = _stack()
    Xq, recs = sequential.sequential_mlp_stack(X, blocks, bits=8, group_size=32, block_size=32)
    Xf = np.asarray(X, np.float64)
    for Wg, Wu, Wd in blocks:
        Xf = sequential.mlp_block_float(Xf, Wg, Wu, Wd)
    rel = np.linalg.norm(Xq - Xf) / np.linalg.norm(Xf)
    # 8-bit steps of about range/255 per 32 weights: a relative weight error near 5e-3 per
    # layer, plus fp16 rounding of every activation
    assert rel < 1e-2, rel
    assert len(recs) == 4 and all(r["loss"] < 1e-3 for r in recs)
    X2, _ = sequential.sequential_mlp_stack(X, blocks, bits=2, group_size=32, block_size=32)
    assert np.linalg.norm(X2 - Xf) / np.linalg.norm(Xf) > 10 * rel


def test_quantization_error_propagates_to_later_hessians():
    X, blocks = _stack(n_blocks=2, seed=1)
    _, r8 = sequential.sequential_mlp_stack(X, blocks, bits=8, group_size=32, block_size=32)
    _, r2 = sequential.sequential_mlp_stack(X, blocks, bits=2, group_size=32, block_size=32)
    # block 0's gate/up sees the same input either way; everything after it does not
    assert np.array_equal(r8[0]["H"], r2[0]["H"])
    for k in (1, 2, 3):
        rel = np.linalg.norm(r8[k]["H"] - r2[k]["H"]) / np.linalg.norm(r8[k]["H"])
        assert rel > 1e-3, (k, rel)
    # with 8-bit layers the down projection's Hessian is close to the float forward's
    Wg, Wu, _ = blocks[0]
    Xf = np.asarray(X, np.float64)
    Xf = Xf / np.sqrt(np.mean(Xf * Xf, axis=1, keepdims=True) + sequential.RMS_EPS)
    G, U = Xf @ Wg.T, Xf @ Wu.T
    Af = G / (1 + np.exp(-G)) * U
    Hf = hessian.hessian(Af)
    assert np.linalg.norm(r8[1]["H"] - Hf) / np.linalg.norm(Hf) < 2e-2

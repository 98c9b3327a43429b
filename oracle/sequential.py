"""Oracle: sequential layer-by-layer GPTQ with error propagation (test infrastructure only).

Sources
  * gtnt.cn/news/115337 §4: GPTQ collects each layer's Hessian from calibration forward passes
    and quantizes layer by layer, in order.
  * 0539edu.com/news/6111416 §3.1: GPTQ quantizes layer by layer, minimising each layer's
    output error ‖WX − W_qX‖²; hncyxsy.com/news/243429 §3.1 step 4: the layers are processed
    one after another.

Reading: "in order" means the input of every layer is produced by the layers before it in
their QUANTIZED form, so the error each layer leaves is seen by the Hessians of the layers after
it. The pages name no block architecture for a synthetic run; the block here is the gated MLP of
the 7B decoder shapes the configs use, with its pre-normalisation (RMS norm with unit weight,
which keeps the products of the gate in range) and a residual connection (attention is left
out):

    N_b = rms_norm(X_b),   X_{b+1} = X_b + down( silu(gate(N_b)) ⊙ up(N_b) )

quantized in the order gate and up (one Hessian, from N_b), then down (its Hessian from the
activations A = silu(G) ⊙ U computed with the already-quantized gate and up). Every layer
output is the W4A16 layer of ``w4a16`` (fp16 weights reconstructed from the codes, exact
fp64 accumulation, one rounding to fp16); N and A are rounded to fp16 after fp64 arithmetic.
"""

import numpy as np

from . import gptq, hessian, loss, w4a16


def silu_mul(G, U):
    """fp16(silu(g)·u), silu(g) = g/(1 + e^(−g)), computed in fp64 from the fp16 values."""
    g = np.asarray(G, np.float64)
    u = np.asarray(U, np.float64)
    return (g / (1.0 + np.exp(-g)) * u).astype(np.float16).astype(np.float64)


RMS_EPS = 1e-6


def rms_norm(X, eps=RMS_EPS):
    """fp16(x / sqrt(mean(x²) + eps)) per token (row), unit weight, in fp64."""
    X = np.asarray(X, np.float64)
    r = np.sqrt(np.mean(X * X, axis=1, keepdims=True) + eps)
    return (X / r).astype(np.float16).astype(np.float64)


def mlp_block_float(X, W_gate, W_up, W_down):
    """The unquantized block in fp64 from fp16 inputs (for comparison)."""
    X = np.asarray(X, np.float64)
    Nx = X / np.sqrt(np.mean(X * X, axis=1, keepdims=True) + RMS_EPS)
    G = Nx @ np.asarray(W_gate, np.float64).T
    U = Nx @ np.asarray(W_up, np.float64).T
    A = G / (1.0 + np.exp(-G)) * U
    return X + A @ np.asarray(W_down, np.float64).T


def sequential_mlp_stack(X0, blocks, bits=4, group_size=128, block_size=128, percdamp=0.01,
                         act_order=False):
    """Quantize a stack of MLP blocks in order. ``blocks`` is a list of (W_gate, W_up, W_down)
    with W_gate, W_up [d_ff, d] and W_down [d, d_ff]. Returns (final activations (fp16 values,
    fp64), per-layer records: dict(name, out (gptq_blocked_ref result), loss, H))."""
    X = np.asarray(X0, np.float64)
    records = []
    for b, (Wg, Wu, Wd) in enumerate(blocks):
        d_ff = np.asarray(Wg).shape[0]
        Nx = rms_norm(X)
        H1 = hessian.hessian(Nx)
        W_gu = np.vstack([np.asarray(Wg, np.float64), np.asarray(Wu, np.float64)])
        o1 = gptq.gptq_blocked_ref(W_gu, H1, bits, group_size, block_size, percdamp, act_order)
        records.append(dict(name=f"block{b}.gate_up", out=o1, H=H1,
                            loss=loss.recon_loss(W_gu, o1["What"], H1)))
        Y16, _ = w4a16.w4a16_linear(Nx, o1["codes"], o1["scales"], o1["zeros"], o1["g_idx"])
        A = silu_mul(Y16[:, :d_ff], Y16[:, d_ff:])
        H2 = hessian.hessian(A)
        Wd = np.asarray(Wd, np.float64)
        o2 = gptq.gptq_blocked_ref(Wd, H2, bits, group_size, block_size, percdamp, act_order)
        records.append(dict(name=f"block{b}.down", out=o2, H=H2,
                            loss=loss.recon_loss(Wd, o2["What"], H2)))
        X, _ = w4a16.w4a16_linear(A, o2["codes"], o2["scales"], o2["zeros"], o2["g_idx"], R=X)
    return X, records

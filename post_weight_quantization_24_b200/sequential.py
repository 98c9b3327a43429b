"""Layer-by-layer GPTQ of a stack of MLP blocks, each layer's Hessian taken from the outputs
of the already-quantized layers before it (gtnt.cn/news/115337 §4: Hessians from calibration
forward passes, layers quantized in order; hncyxsy.com/news/243429 §3.1 step 4).

Block: N_b = rms_norm(X_b), X_{b+1} = X_b + down(silu(gate(N_b)) ⊙ up(N_b)), the gated MLP of
the 7B decoder shapes with its unit-weight RMS pre-norm and a residual (attention left out). Per
block, in order:
  1. N_b = rms_norm(X_b), H = 2·N_bᵀN_b (tensor-core Hessian);
  2. GPTQ of the row-stacked gate;up weights (one Hessian, one factorisation);
  3. the W4A16 layer on N_b with the quantized gate;up -> G;U, then A = silu(G)·U;
  4. H = 2·AᵀA, GPTQ of down;
  5. X_{b+1} = X_b + the W4A16 layer on A with the quantized down (residual added before the
     fp16 rounding).
This module only sequences library calls; every step runs in the library's kernels.
"""

from __future__ import annotations

import torch

from . import gptq


def _quantize_and_pack(W, H, bits, group_size, block_size, percdamp, act_order, workspace):
    out = gptq.quantize_layer(W, H, bits=bits, group_size=group_size, block_size=block_size,
                              percdamp=percdamp, act_order=act_order, compute_loss=True,
                              workspace=workspace)
    perm = out["perm"] if act_order else None
    out["packed"] = gptq.w4a16_pack(out["codes"], perm)
    out["perm_gather"] = perm
    return out


def quantize_mlp_stack(X0: torch.Tensor, blocks, bits: int = 4, group_size: int = 128,
                       block_size: int = 128, percdamp: float = 0.01, act_order: bool = False,
                       timings: dict | None = None):
    """Quantize `blocks` = [(W_gate [d_ff, d], W_up [d_ff, d], W_down [d, d_ff]), ...] (fp16
    CUDA tensors) in order, starting from the calibration activations X0 (fp16 [n, d]).

    Returns (final activations fp16 [n, d], per-layer records dict(name, codes, scales, zeros,
    g_idx, perm, packed, loss)). With `timings` (a dict), CUDA-event milliseconds per step kind
    are added to it: norm, hessian, gptq, w4a16, silu."""
    if bits != 4:
        raise ValueError("the W4A16 layer serves 4-bit codes")
    X = X0
    records = []
    ev = []

    def mark(kind):
        if timings is not None:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            ev.append((kind, e))

    for b, (Wg, Wu, Wd) in enumerate(blocks):
        d_ff, d = Wg.shape
        n = X.shape[0]
        W_gu = torch.cat([Wg, Wu], dim=0)
        ws = torch.empty(max(gptq.quantize_layer_workspace(2 * d_ff, d, block_size),
                             gptq.quantize_layer_workspace(d, d_ff, block_size)),
                         dtype=torch.uint8, device=X.device)
        mark("start")
        Nx = gptq.rms_norm(X)
        mark("norm")
        h1 = gptq.Hessian(d)
        h1.accumulate(Nx)
        mark("hessian")
        o1 = _quantize_and_pack(W_gu, h1.raw(), bits, group_size, block_size, percdamp,
                                act_order, ws)
        mark("gptq")
        GU = gptq.w4a16_linear(Nx, o1["packed"], o1["scales"], o1["zeros"], group_size,
                               perm=o1["perm_gather"])
        del Nx
        mark("w4a16")
        A = gptq.silu_mul(GU)
        del GU
        mark("silu")
        h2 = gptq.Hessian(d_ff)
        h2.accumulate(A)
        mark("hessian")
        o2 = _quantize_and_pack(Wd, h2.raw(), bits, group_size, block_size, percdamp,
                                act_order, ws)
        mark("gptq")
        X = gptq.w4a16_linear(A, o2["packed"], o2["scales"], o2["zeros"], group_size,
                              perm=o2["perm_gather"], R=X)
        mark("w4a16")
        records.append(dict(name=f"block{b}.gate_up", **o1))
        records.append(dict(name=f"block{b}.down", **o2))
        del A, h1, h2
    if timings is not None:
        torch.cuda.synchronize()
        for (_, a), (kind, b) in zip(ev[:-1], ev[1:]):
            if kind != "start":
                timings[kind] = timings.get(kind, 0.0) + a.elapsed_time(b)
    return X, records

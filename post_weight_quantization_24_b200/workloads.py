"""Seeded synthetic layer inputs for GPTQ calibration workloads.

This module only draws random numbers: it holds no quantization, Hessian or factorisation
arithmetic, so both the CUDA library's callers and the fp64 checker can take their inputs from
it. Every tensor comes from its own stream keyed by (seed, tensor id).

Recipe (the shapes are those of LLM linear layers; the value distributions follow the pages'
description of LLM weights and activations: near-zero-mean weights with a few outlier input
columns, activations with per-channel magnitudes spread over orders of magnitude and a few
outlier channels):

* W: N(0, w_std²) in fp32; ``round(w_outlier_frac · d_in)`` randomly chosen input columns
  multiplied by ``w_outlier_scale``; stored as ``w_dtype``.
* X: z ~ N(0, 1) per entry times a per-channel magnitude exp(N(0, x_sigma²));
  ``x_outlier_channels`` randomly chosen channels multiplied by ``x_outlier_scale``; rounded to
  fp16 (round to nearest even).

Named workloads:

* ``linear_512``       W 512×512 fp32, X 2048×512, x_sigma 0.5, no outliers; INT4 g128 B128.
* ``mlp_up_7b``        W 11008×4096 fp16 with 4 outlier columns ×20; X 262144×4096 (128 sequences
                       of 2048 tokens), x_sigma 1, 6 outlier channels ×50; INT4 g128 B128.
* ``mlp_down_7b``      W 4096×11008 fp16 (11 outlier columns); X 262144×11008; act_order on;
                       INT4 and INT3, g128.
* ``attn_o_70b``       W 8192×8192 fp16 (8 outlier columns); X 65536×8192; INT4 g128 B128.
* ``mlp_down_70b``     W 8192×28672 fp16 (29 outlier columns); X 65536×28672; INT4 g128 B128.
* ``decoder_7b``       one 7B decoder layer: q,k,v,o 4096×4096, gate,up 11008×4096,
                       down 4096×11008; per-layer inputs of 131072 tokens.

No public dataset is used: the synthetic activations stand in for the WikiText-2 / C4
calibration text the pages mention.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    name: str
    d_out: int
    d_in: int
    n_tokens: int
    w_dtype: str = "f16"            # "f16" or "f32"
    w_std: float = 0.02
    w_outlier_frac: float = 0.001
    w_outlier_scale: float = 20.0
    x_sigma: float = 1.0
    x_outlier_channels: int = 6
    x_outlier_scale: float = 50.0
    bits: int = 4
    group_size: int = 128
    block_size: int = 128
    percdamp: float = 0.01
    act_order: bool = False
    seed: int = 0

    def replace(self, **kw) -> "LayerWorkload":
        return dataclasses.replace(self, **kw)

    @property
    def n_weights(self) -> int:
        return self.d_out * self.d_in


WORKLOADS = {
    "linear_512": LayerWorkload("linear_512", 512, 512, 2048, w_dtype="f32",
                                w_outlier_frac=0.0, x_sigma=0.5, x_outlier_channels=0),
    "mlp_up_7b": LayerWorkload("mlp_up_7b", 11008, 4096, 262144),
    "mlp_down_7b": LayerWorkload("mlp_down_7b", 4096, 11008, 262144, act_order=True),
    "attn_o_70b": LayerWorkload("attn_o_70b", 8192, 8192, 65536),
    "mlp_down_70b": LayerWorkload("mlp_down_70b", 8192, 28672, 65536),
}

# One 7B decoder layer: (name, d_out, d_in, which input it reads).
DECODER_7B_LINEARS = (
    ("q_proj", 4096, 4096, "attn_in"), ("k_proj", 4096, 4096, "attn_in"),
    ("v_proj", 4096, 4096, "attn_in"), ("o_proj", 4096, 4096, "o_in"),
    ("gate_proj", 11008, 4096, "mlp_in"), ("up_proj", 11008, 4096, "mlp_in"),
    ("down_proj", 4096, 11008, "down_in"),
)
DECODER_7B_INPUTS = {"attn_in": 4096, "o_in": 4096, "mlp_in": 4096, "down_in": 11008}
# The same layer with the linears that read one input stacked row-wise (q;k;v and gate;up), as
# fused projections store them: (name, parts, d_in, input).
DECODER_7B_FUSED = (
    ("qkv_proj", ("q_proj", "k_proj", "v_proj"), 4096, "attn_in"),
    ("o_proj", ("o_proj",), 4096, "o_in"),
    ("gate_up_proj", ("gate_proj", "up_proj"), 4096, "mlp_in"),
    ("down_proj", ("down_proj",), 11008, "down_in"),
)

_TID_W, _TID_W_OUTLIER, _TID_X, _TID_X_SCALE, _TID_X_OUTLIER = 1, 2, 3, 4, 5


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + tensor_id * 7919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _dtype(name: str) -> torch.dtype:
    return {"f16": torch.float16, "f32": torch.float32}[name]


def make_weights(wl: LayerWorkload, device="cpu", seed: int | None = None) -> torch.Tensor:
    """W [d_out, d_in] with the workload's distribution, stored as ``wl.w_dtype``."""
    seed = wl.seed if seed is None else seed
    W = torch.randn(wl.d_out, wl.d_in, generator=_gen(seed, _TID_W, device), device=device,
                    dtype=torch.float32)
    W.mul_(wl.w_std)
    k = int(round(wl.w_outlier_frac * wl.d_in))
    if k:
        cols = torch.randperm(wl.d_in, generator=_gen(seed, _TID_W_OUTLIER, "cpu"))[:k]
        W[:, cols.to(device)] *= wl.w_outlier_scale
    return W.to(_dtype(wl.w_dtype))


def channel_magnitudes(d_in: int, sigma: float, n_outliers: int, outlier_scale: float,
                       seed: int) -> torch.Tensor:
    """Per-channel activation magnitudes exp(N(0, sigma²)) with outlier channels (fp32, CPU)."""
    m = torch.exp(sigma * torch.randn(d_in, generator=_gen(seed, _TID_X_SCALE, "cpu")))
    if n_outliers:
        ch = torch.randperm(d_in, generator=_gen(seed, _TID_X_OUTLIER, "cpu"))[:n_outliers]
        m[ch] *= outlier_scale
    return m


def make_activations(wl: LayerWorkload, device="cpu", seed: int | None = None,
                     n_tokens: int | None = None, d_in: int | None = None,
                     chunk_tokens: int = 16384) -> torch.Tensor:
    """X [n_tokens, d_in] fp16: N(0,1) entries times per-channel magnitudes."""
    seed = wl.seed if seed is None else seed
    n = wl.n_tokens if n_tokens is None else n_tokens
    d = wl.d_in if d_in is None else d_in
    mags = channel_magnitudes(d, wl.x_sigma, wl.x_outlier_channels, wl.x_outlier_scale, seed)
    mags = mags.to(device)
    X = torch.empty(n, d, dtype=torch.float16, device=device)
    g = _gen(seed, _TID_X, device)
    for t0 in range(0, n, chunk_tokens):
        t1 = min(n, t0 + chunk_tokens)
        z = torch.randn(t1 - t0, d, generator=g, device=device, dtype=torch.float32)
        X[t0:t1] = (z * mags).to(torch.float16)
    return X


def correlated_activations(n: int, d: int, rank: int = 4, seed: int = 0,
                           device="cpu") -> torch.Tensor:
    """X = Z·M with a low-rank-plus-identity mixing M: strongly correlated channels.

    A test input (not a named workload): it makes the error compensation do visible work.
    """
    g = _gen(seed, 11, "cpu")
    A = torch.randn(d, rank, generator=g)
    M = torch.eye(d) + 0.9 * (A @ A.T) / np.sqrt(rank) + 0.05 * torch.randn(d, d, generator=g)
    Z = torch.randn(n, d, generator=g)
    return (Z @ M).to(torch.float16).to(device)


def make_decoder_layer(layer: int, n_tokens: int, device="cpu", seed_base: int = 1000):
    """One synthetic 7B decoder layer of a stack: its four distinct inputs (n_tokens each, the
    7B activation recipe) and its weights (the 7B weight recipe, fp16), with the linears that
    read one input stacked row-wise. Every tensor has its own seed, distinct per layer.
    Returns (inputs: {input name: X}, fused: [(name, W, input name)])."""
    base = WORKLOADS["mlp_up_7b"]
    seed0 = seed_base + 64 * layer
    inputs = {}
    for idx, (name, d) in enumerate(DECODER_7B_INPUTS.items()):
        inputs[name] = make_activations(base.replace(d_in=d, n_tokens=n_tokens),
                                        device=device, seed=seed0 + idx)
    shapes = {name: (d_out, d_in) for name, d_out, d_in, _ in DECODER_7B_LINEARS}
    order = [name for name, _, _, _ in DECODER_7B_LINEARS]
    fused = []
    for name, parts, d_in, src in DECODER_7B_FUSED:
        rows = sum(shapes[p][0] for p in parts)
        W = torch.empty(rows, d_in, dtype=torch.float16, device=device)
        r0 = 0
        for p in parts:
            d_out = shapes[p][0]
            W[r0:r0 + d_out] = make_weights(base.replace(d_out=d_out, d_in=d_in), device=device,
                                            seed=seed0 + 8 + order.index(p))
            r0 += d_out
        fused.append((name, W, src))
    return inputs, fused

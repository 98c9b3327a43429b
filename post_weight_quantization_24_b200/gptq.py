"""Python binding of ``libgptq_b200.so`` (ctypes; argument marshalling only).

Every computation runs in the library's sm_100a kernels; torch supplies device memory and the
current CUDA stream. If the library is not built, calls raise immediately — there is no CPU or
torch fallback.

Functions (names follow the C ABI in ``include/gptq.h``):
  Hessian(d_in)                    handle: .accumulate(X), .get(), .data_ptr, .tokens, .reset()
  hessian_accumulate_into(H, X)    H += 2·XᵀX on a caller tensor (upper triangle)
  quantize_layer(W, H, ...)        GPTQ one linear layer -> codes, scales, zeros, g_idx, perm, loss
  quantize_layer_workspace(...)    workspace bytes for quantize_layer
  inverse_factor(H, ...)           processing order and U with UᵀU = H_d⁻¹ (stage 2 alone)
  rtn_minmax_quantize(W, ...)      group min-max RTN -> packed codes, scales, zeros
  profile_enable(on), profile_read()  per-stage milliseconds of the last quantize_layer call
"""

from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgptq_b200.so")

STATUS = {0: "GPTQ_OK", -1: "GPTQ_ERR_ARG", -2: "GPTQ_ERR_NOT_PD", -3: "GPTQ_ERR_NONFINITE",
          -4: "GPTQ_ERR_CUDA", -5: "GPTQ_ERR_OOM", -6: "GPTQ_ERR_TIMEOUT",
          -7: "GPTQ_ERR_WORKSPACE", -8: "GPTQ_ERR_UNSUPPORTED"}
DTYPE_F16, DTYPE_F32 = 0, 1
STAGES = ("prepare", "factor", "images", "column_loop", "lazy_update", "assemble", "loss")


class GPTQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name}")


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "gptq_status_string": ([_I], ctypes.c_char_p),
    "gptq_hessian_create": ([_I, ctypes.POINTER(_P)], _I),
    "gptq_hessian_accumulate": ([_P, _P, _I64, _P], _I),
    "gptq_hessian_get": ([_P, _P, _P], _I),
    "gptq_hessian_data": ([_P], _P),
    "gptq_hessian_tokens": ([_P], _I64),
    "gptq_hessian_dim": ([_P], _I),
    "gptq_hessian_reset": ([_P, _P], _I),
    "gptq_hessian_destroy": ([_P], _I),
    "gptq_hessian_accumulate_into": ([_P, _I, _P, _I64, _I, _P, _P], _I),
    "gptq_quantize_layer_workspace": ([_I, _I, _I], _SZ),
    "gptq_quantize_layer": ([_P, _I, _I, _I, _P, _I, _I, _I, _F, _I, _P, _P, _P, _P, _P,
                             ctypes.POINTER(_F), _P, _SZ, _P], _I),
    "gptq_inverse_factor_workspace": ([_I], _SZ),
    "gptq_inverse_factor": ([_P, _I, _F, _I, _P, _P, _P, _SZ, _P], _I),
    "rtn_minmax_quantize": ([_P, _I, _I, _I, _I, _I, _P, _P, _P, _P], _I),
    "gptq_quantize_layer_ex": ([_P, _I, _I, _I, _P, _I, _I, _I, _F, _I, _I, _I, _P, _P, _P, _P,
                                _P, ctypes.POINTER(_F), _P, _SZ, _P], _I),
    "rtn_quantize_ex": ([_P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P], _I),
    "rtn_clip_search": ([_P, _I, _I, _I, _I, _I, _I, _P, ctypes.c_double, ctypes.c_double, _P,
                         _P, _P, _P, _P], _I),
    "rtn_range_clip": ([_P, _I, _I, _I, _I, _I, _I, ctypes.c_double, ctypes.c_double, _P, _P,
                        _P, _P], _I),
    "w4a16_pack": ([_P, _I, _I, _P, _P, _P], _I),
    "w4a16_linear_workspace": ([_I64, _I, _I], _SZ),
    "w4a16_linear": ([_P, _I64, _I, _P, _P, _P, _I, _I, _P, _P, _P, _P, _SZ, _P, _P], _I),
    "gptq_silu_mul": ([_P, _I64, _I, _P, _P], _I),
    "gptq_rms_norm": ([_P, _I64, _I, _F, _P, _P], _I),
    "gptq_channel_abs_sum": ([_P, _I, _I64, _I, _P, _P], _I),
    "awq_lite_workspace": ([_I, _I, ctypes.c_double], _SZ),
    "awq_lite_search": ([_P, _I, _I, _I, _P, _I64, _P, _I, _I, _I, ctypes.c_double, _P, _P, _P,
                         _P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I), _P, _SZ, _P],
                        _I),
    "gptq_quantize_layer_noalloc": ([_P, _I, _I, _I, _P, _I, _I, _I, _F, _I, _P, _P, _P, _P, _P,
                                     ctypes.POINTER(_F), _P], _I),
    "gptq_profile_enable": ([_I], None),
    "gptq_profile_read": ([ctypes.POINTER(_F), _I], _I),
    "gptq_launch_count": ([], ctypes.c_ulonglong),
    "gptq_test_stall_factor": ([_I], _I),
}


def lib() -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m post_weight_quantization_24_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise GPTQError(status, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return DTYPE_F16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"W must be float16 or float32, got {t.dtype}")


def _require_cuda(t: torch.Tensor, name: str) -> None:
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


# ------------------------------------------------------------------------------------------
# Hessian
# ------------------------------------------------------------------------------------------
class Hessian:
    """H = 2·XᵀX accumulated over calls (fp32, d_in x d_in) on the current device."""

    def __init__(self, d_in: int):
        h = _P()
        _check(lib().gptq_hessian_create(d_in, ctypes.byref(h)), "gptq_hessian_create")
        self._h = h
        self.d_in = d_in

    def accumulate(self, X: torch.Tensor) -> None:
        _require_cuda(X, "X")
        if X.dtype != torch.float16 or X.dim() != 2 or X.shape[1] != self.d_in:
            raise ValueError("X must be fp16 [n_tokens, d_in]")
        _check(lib().gptq_hessian_accumulate(self._h, X.data_ptr(), X.shape[0], _stream()),
               "gptq_hessian_accumulate")

    def get(self, out: torch.Tensor | None = None) -> torch.Tensor:
        if out is None:
            out = torch.empty(self.d_in, self.d_in, dtype=torch.float32, device="cuda")
        _check(lib().gptq_hessian_get(self._h, out.data_ptr(), _stream()), "gptq_hessian_get")
        return out

    @property
    def data_ptr(self) -> int:
        return lib().gptq_hessian_data(self._h)

    def raw(self) -> torch.Tensor:
        """The handle's storage viewed as a tensor (upper triangle valid); no copy."""
        return _wrap_device_ptr(self.data_ptr, (self.d_in, self.d_in), owner=self)

    @property
    def tokens(self) -> int:
        return lib().gptq_hessian_tokens(self._h)

    def reset(self) -> None:
        _check(lib().gptq_hessian_reset(self._h, _stream()), "gptq_hessian_reset")

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().gptq_hessian_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _wrap_device_ptr(ptr: int, shape, owner):
    """Zero-copy fp32 tensor over device memory owned by ``owner`` (kept alive by the tensor)."""
    class _CAI:
        def __init__(self):
            self.__cuda_array_interface__ = {
                "shape": tuple(shape), "typestr": "<f4", "data": (ptr, False), "version": 3,
                "strides": None}
            self._owner = owner
    return torch.as_tensor(_CAI(), device="cuda")


def hessian_accumulate_into(H: torch.Tensor, X: torch.Tensor, unit_tokens: int = 0,
                            status: torch.Tensor | None = None) -> None:
    """H (fp32 [d, d], upper triangle) += 2·XᵀX for X fp16 [n, d]."""
    _require_cuda(H, "H")
    _require_cuda(X, "X")
    if H.dtype != torch.float32 or X.dtype != torch.float16:
        raise TypeError("H must be fp32 and X fp16")
    d = H.shape[0]
    if H.shape != (d, d) or X.dim() != 2 or X.shape[1] != d:
        raise ValueError("shape mismatch")
    _check(lib().gptq_hessian_accumulate_into(H.data_ptr(), d, X.data_ptr(), X.shape[0],
                                              unit_tokens, _ptr(status), _stream()),
           "gptq_hessian_accumulate_into")


# ------------------------------------------------------------------------------------------
# GPTQ layer
# ------------------------------------------------------------------------------------------
def quantize_layer_workspace(d_out: int, d_in: int, block_size: int = 128) -> int:
    return int(lib().gptq_quantize_layer_workspace(d_out, d_in, block_size))


def quantize_layer(W: torch.Tensor, H: torch.Tensor, bits: int = 4, group_size: int = 128,
                   block_size: int = 128, percdamp: float = 0.01, act_order: bool = False,
                   compute_loss: bool = False, workspace: torch.Tensor | None = None,
                   out: dict | None = None, sym: bool = False,
                   static_groups: bool = False) -> dict:
    """GPTQ-quantize W [d_out, d_in] (fp16/fp32) with Hessian H [d_in, d_in] (upper read).

    Returns dict(codes uint8 [d_out, d_in] original order, scales/zeros fp16 [d_out, d_in/g],
    g_idx int32 [d_in], perm int32 [d_in], loss float | None). ``sym``, ``static_groups`` and
    group_size == d_in (per-channel) select the quantizer variants of gptq_quantize_layer_ex.
    """
    _require_cuda(W, "W")
    _require_cuda(H, "H")
    d_out, d_in = W.shape
    if H.dtype != torch.float32 or H.shape != (d_in, d_in):
        raise ValueError("H must be fp32 [d_in, d_in]")
    dev = W.device
    if out is None:
        ng = d_in // group_size if group_size > 0 and d_in % group_size == 0 else 1
        out = dict(codes=torch.empty(d_out, d_in, dtype=torch.uint8, device=dev),
                   scales=torch.empty(d_out, ng, dtype=torch.float16, device=dev),
                   zeros=torch.empty(d_out, ng, dtype=torch.float16, device=dev),
                   g_idx=torch.empty(d_in, dtype=torch.int32, device=dev),
                   perm=torch.empty(d_in, dtype=torch.int32, device=dev))
    if workspace is None:
        nbytes = quantize_layer_workspace(d_out, d_in, block_size)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    loss = ctypes.c_float(float("nan"))
    st = lib().gptq_quantize_layer_ex(
        W.data_ptr(), _dtype_code(W), d_out, d_in, H.data_ptr(), bits, group_size, block_size,
        float(percdamp), int(bool(act_order)), int(bool(sym)), int(bool(static_groups)),
        out["codes"].data_ptr(), out["scales"].data_ptr(), out["zeros"].data_ptr(),
        out["g_idx"].data_ptr(), _ptr(out.get("perm")),
        ctypes.byref(loss) if compute_loss else None, workspace.data_ptr(),
        workspace.numel(), _stream())
    _check(st, "gptq_quantize_layer_ex")
    res = dict(out)
    res["loss"] = float(loss.value) if compute_loss else None
    return res


def quantize_layer_noalloc(W: torch.Tensor, H: torch.Tensor, bits: int = 4,
                           group_size: int = 128, block_size: int = 128,
                           percdamp: float = 0.01, act_order: bool = False,
                           compute_loss: bool = False, out: dict | None = None) -> dict:
    """quantize_layer without a workspace: the library uses its fixed 32 MiB device scratch.

    For callers that may not allocate device memory while quantizing. Only ``out`` (the
    caller's output tensors) is allocated here when it is not given. Layers whose workspace
    would exceed 32 MiB raise GPTQError(GPTQ_ERR_WORKSPACE). Calls share the scratch, so they
    must not overlap on the GPU.
    """
    _require_cuda(W, "W")
    _require_cuda(H, "H")
    d_out, d_in = W.shape
    dev = W.device
    if out is None:
        ng = d_in // group_size if group_size > 0 and d_in % group_size == 0 else 1
        out = dict(codes=torch.empty(d_out, d_in, dtype=torch.uint8, device=dev),
                   scales=torch.empty(d_out, ng, dtype=torch.float16, device=dev),
                   zeros=torch.empty(d_out, ng, dtype=torch.float16, device=dev),
                   g_idx=torch.empty(d_in, dtype=torch.int32, device=dev),
                   perm=torch.empty(d_in, dtype=torch.int32, device=dev))
    loss = ctypes.c_float(float("nan"))
    st = lib().gptq_quantize_layer_noalloc(
        W.data_ptr(), _dtype_code(W), d_out, d_in, H.data_ptr(), bits, group_size, block_size,
        float(percdamp), int(bool(act_order)), out["codes"].data_ptr(), out["scales"].data_ptr(),
        out["zeros"].data_ptr(), out["g_idx"].data_ptr(), _ptr(out.get("perm")),
        ctypes.byref(loss) if compute_loss else None, _stream())
    _check(st, "gptq_quantize_layer_noalloc")
    res = dict(out)
    res["loss"] = float(loss.value) if compute_loss else None
    return res


def inverse_factor(H: torch.Tensor, percdamp: float = 0.01, act_order: bool = False):
    """(U, perm): U upper with UᵀU = (P H P + λI)⁻¹ in processing order; perm int32."""
    _require_cuda(H, "H")
    d = H.shape[0]
    U = torch.empty(d, d, dtype=torch.float32, device=H.device)
    perm = torch.empty(d, dtype=torch.int32, device=H.device)
    ws = torch.empty(int(lib().gptq_inverse_factor_workspace(d)), dtype=torch.uint8,
                     device=H.device)
    _check(lib().gptq_inverse_factor(H.data_ptr(), d, float(percdamp), int(bool(act_order)),
                                     U.data_ptr(), perm.data_ptr(), ws.data_ptr(), ws.numel(),
                                     _stream()), "gptq_inverse_factor")
    return U, perm


# ------------------------------------------------------------------------------------------
# RTN
# ------------------------------------------------------------------------------------------
def rtn_minmax_quantize(W: torch.Tensor, bits: int = 4, group_size: int = 128,
                        out: tuple | None = None, sym: bool = False):
    """Group min-max RTN of W [d_out, d_in] -> (packed uint8, scales fp16, zeros fp16).

    bits == 4: packed is [d_out, d_in/2] (even column in the low nibble); else [d_out, d_in].
    ``sym`` takes the symmetric quantizer (rtn_quantize_ex).
    """
    _require_cuda(W, "W")
    d_out, d_in = W.shape
    dev = W.device
    if out is None:
        ng = d_in // group_size if group_size > 0 and d_in % group_size == 0 else 1
        packed = torch.empty(d_out, d_in // 2 if bits == 4 else d_in, dtype=torch.uint8, device=dev)
        out = (packed, torch.empty(d_out, ng, dtype=torch.float16, device=dev),
               torch.empty(d_out, ng, dtype=torch.float16, device=dev))
    packed, scales, zeros = out
    st = lib().rtn_quantize_ex(W.data_ptr(), _dtype_code(W), d_out, d_in, bits, group_size,
                               int(bool(sym)), packed.data_ptr(), scales.data_ptr(),
                               zeros.data_ptr(), _stream())
    _check(st, "rtn_quantize_ex")
    return packed, scales, zeros


def rtn_clip_search(W: torch.Tensor, bits: int = 4, group_size: int = 128,
                    H: torch.Tensor | None = None, sym: bool = False, min_ratio: float = 0.5,
                    step: float = 0.05):
    """Group RTN with a clip search per group (criterion d·H_gg·d, or d·d without H) ->
    (packed uint8, scales fp16, zeros fp16, ratio index uint8 [d_out, d_in/g])."""
    _require_cuda(W, "W")
    d_out, d_in = W.shape
    dev = W.device
    ng = d_in // group_size if group_size > 0 and d_in % group_size == 0 else 1
    packed = torch.empty(d_out, d_in // 2 if bits == 4 else d_in, dtype=torch.uint8, device=dev)
    scales = torch.empty(d_out, ng, dtype=torch.float16, device=dev)
    zeros = torch.empty(d_out, ng, dtype=torch.float16, device=dev)
    ridx = torch.empty(d_out, ng, dtype=torch.uint8, device=dev)
    if H is not None:
        _require_cuda(H, "H")
        if H.dtype != torch.float32 or H.shape != (d_in, d_in):
            raise ValueError("H must be fp32 [d_in, d_in]")
    st = lib().rtn_clip_search(W.data_ptr(), _dtype_code(W), d_out, d_in, bits, group_size,
                               int(bool(sym)), _ptr(H), float(min_ratio), float(step),
                               packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
                               ridx.data_ptr(), _stream())
    _check(st, "rtn_clip_search")
    return packed, scales, zeros, ridx


def rtn_range_clip(W: torch.Tensor, bits: int = 4, group_size: int = 128,
                   percentile: float = 99.99, abs_range: float = 0.0, sym: bool = False):
    """Group RTN of the weights clipped to each group's (100 - percentile)/percentile
    quantiles, limited to [-abs_range, abs_range] when abs_range > 0 ->
    (packed uint8, scales fp16, zeros fp16)."""
    _require_cuda(W, "W")
    d_out, d_in = W.shape
    dev = W.device
    ng = d_in // group_size if group_size > 0 and d_in % group_size == 0 else 1
    packed = torch.empty(d_out, d_in // 2 if bits == 4 else d_in, dtype=torch.uint8, device=dev)
    scales = torch.empty(d_out, ng, dtype=torch.float16, device=dev)
    zeros = torch.empty(d_out, ng, dtype=torch.float16, device=dev)
    st = lib().rtn_range_clip(W.data_ptr(), _dtype_code(W), d_out, d_in, bits, group_size,
                              int(bool(sym)), float(percentile), float(abs_range),
                              packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(), _stream())
    _check(st, "rtn_range_clip")
    return packed, scales, zeros


# ------------------------------------------------------------------------------------------
# W4A16 layer
# ------------------------------------------------------------------------------------------
def w4a16_pack(codes: torch.Tensor, perm: torch.Tensor | None = None) -> torch.Tensor:
    """INT4 codes [d_out, d_in] (original order) -> packed [d_out, d_in/2] in perm's order."""
    _require_cuda(codes, "codes")
    d_out, d_in = codes.shape
    packed = torch.empty(d_out, d_in // 2, dtype=torch.uint8, device=codes.device)
    _check(lib().w4a16_pack(codes.data_ptr(), d_out, d_in, _ptr(perm), packed.data_ptr(),
                            _stream()), "w4a16_pack")
    return packed


def w4a16_linear(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                 zeros: torch.Tensor, group_size: int = 128, perm: torch.Tensor | None = None,
                 R: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None,
                 status: torch.Tensor | None = None) -> torch.Tensor:
    """Y = fp16(X·Ŵᵀ + R) for fp16 X [n, d_in] and packed INT4 weights [d_out, d_in/2]."""
    _require_cuda(X, "X")
    n, d_in = X.shape
    d_out = packed.shape[0]
    if out is None:
        out = torch.empty(n, d_out, dtype=torch.float16, device=X.device)
    nb = int(lib().w4a16_linear_workspace(n, d_in, int(perm is not None)))
    if perm is not None and (workspace is None or workspace.numel() < nb):
        workspace = torch.empty(nb, dtype=torch.uint8, device=X.device)
    st = lib().w4a16_linear(X.data_ptr(), n, d_in, packed.data_ptr(), scales.data_ptr(),
                            zeros.data_ptr(), group_size, d_out, _ptr(perm), _ptr(R),
                            out.data_ptr(), _ptr(workspace),
                            0 if workspace is None else workspace.numel(), _ptr(status),
                            _stream())
    _check(st, "w4a16_linear")
    return out


def channel_abs_sum(X: torch.Tensor, sums: torch.Tensor | None = None) -> torch.Tensor:
    """sums[c] += Σ_t |X[t, c]| (fp64 [d]); a new zeroed buffer when `sums` is None."""
    _require_cuda(X, "X")
    n, d = X.shape
    if sums is None:
        sums = torch.zeros(d, dtype=torch.float64, device=X.device)
    _check(lib().gptq_channel_abs_sum(X.data_ptr(), _dtype_code(X), n, d, sums.data_ptr(),
                                      _stream()), "gptq_channel_abs_sum")
    return sums


def awq_lite_search(W: torch.Tensor, x_abs_sum: torch.Tensor, n_tokens: int, H: torch.Tensor,
                    bits: int = 4, group_size: int = 128, sym: bool = False,
                    alpha_step: float = 0.1) -> dict:
    """AWQ-lite grid search (H full symmetric). Returns dict(packed, scales, zeros, s (fp16
    [d_in]), losses (list), best (index), alpha)."""
    _require_cuda(W, "W")
    _require_cuda(H, "H")
    d_out, d_in = W.shape
    dev = W.device
    ng = d_in // group_size
    n_alpha = int(round(1.0 / alpha_step)) + 1
    packed = torch.empty(d_out, d_in // 2 if bits == 4 else d_in, dtype=torch.uint8, device=dev)
    scales = torch.empty(d_out, ng, dtype=torch.float16, device=dev)
    zeros = torch.empty(d_out, ng, dtype=torch.float16, device=dev)
    s_out = torch.empty(d_in, dtype=torch.float16, device=dev)
    ws = torch.empty(max(1, int(lib().awq_lite_workspace(d_out, d_in, float(alpha_step)))),
                     dtype=torch.uint8, device=dev)
    losses = (ctypes.c_double * n_alpha)()
    best = ctypes.c_int(-1)
    st = lib().awq_lite_search(W.data_ptr(), _dtype_code(W), d_out, d_in, x_abs_sum.data_ptr(),
                               int(n_tokens), H.data_ptr(), bits, group_size, int(bool(sym)),
                               float(alpha_step), packed.data_ptr(), scales.data_ptr(),
                               zeros.data_ptr(), s_out.data_ptr(), losses, ctypes.byref(best),
                               ws.data_ptr(), ws.numel(), _stream())
    _check(st, "awq_lite_search")
    return dict(packed=packed, scales=scales, zeros=zeros, s=s_out, losses=list(losses),
                best=int(best.value), alpha=int(best.value) * alpha_step)


def rms_norm(X: torch.Tensor, eps: float = 1e-6, out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = fp16(x / sqrt(mean(x²) + eps)) per row of fp16 X [n, d] (unit-weight RMS norm)."""
    _require_cuda(X, "X")
    n, d = X.shape
    if out is None:
        out = torch.empty_like(X)
    _check(lib().gptq_rms_norm(X.data_ptr(), n, d, float(eps), out.data_ptr(), _stream()),
           "gptq_rms_norm")
    return out


def silu_mul(GU: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """A = fp16(silu(gate)·up) for GU fp16 [n, 2·d_ff] (gate outputs, then up outputs)."""
    _require_cuda(GU, "GU")
    n, two = GU.shape
    if out is None:
        out = torch.empty(n, two // 2, dtype=torch.float16, device=GU.device)
    _check(lib().gptq_silu_mul(GU.data_ptr(), n, two // 2, out.data_ptr(), _stream()),
           "gptq_silu_mul")
    return out


# ------------------------------------------------------------------------------------------
# stage timing
# ------------------------------------------------------------------------------------------
def profile_enable(on: bool = True) -> None:
    lib().gptq_profile_enable(int(bool(on)))


def profile_read() -> dict:
    buf = (ctypes.c_float * len(STAGES))()
    n = lib().gptq_profile_read(buf, len(STAGES))
    return {STAGES[i]: float(buf[i]) for i in range(n)}


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().gptq_launch_count())


def test_stall_factor(on: bool) -> None:
    """Test hook: make the factorisation's bounded wait run out (see include/gptq.h)."""
    _check(lib().gptq_test_stall_factor(int(bool(on))), "gptq_test_stall_factor")


def status_string(status: int) -> str:
    return lib().gptq_status_string(status).decode()

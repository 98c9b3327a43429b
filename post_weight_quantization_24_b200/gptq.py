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
                   out: dict | None = None) -> dict:
    """GPTQ-quantize W [d_out, d_in] (fp16/fp32) with Hessian H [d_in, d_in] (upper read).

    Returns dict(codes uint8 [d_out, d_in] original order, scales/zeros fp16 [d_out, d_in/g],
    g_idx int32 [d_in], perm int32 [d_in], loss float | None).
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
    st = lib().gptq_quantize_layer(
        W.data_ptr(), _dtype_code(W), d_out, d_in, H.data_ptr(), bits, group_size, block_size,
        float(percdamp), int(bool(act_order)), out["codes"].data_ptr(), out["scales"].data_ptr(),
        out["zeros"].data_ptr(), out["g_idx"].data_ptr(), _ptr(out.get("perm")),
        ctypes.byref(loss) if compute_loss else None, workspace.data_ptr(),
        workspace.numel(), _stream())
    _check(st, "gptq_quantize_layer")
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
                        out: tuple | None = None):
    """Group min-max RTN of W [d_out, d_in] -> (packed uint8, scales fp16, zeros fp16).

    bits == 4: packed is [d_out, d_in/2] (even column in the low nibble); else [d_out, d_in].
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
    st = lib().rtn_minmax_quantize(W.data_ptr(), _dtype_code(W), d_out, d_in, bits, group_size,
                                   packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
                                   _stream())
    _check(st, "rtn_minmax_quantize")
    return packed, scales, zeros


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

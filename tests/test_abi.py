"""The C-ABI library loads and exports every entry point its header declares; host-side
argument checks reject bad calls before anything is launched (no GPU needed)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")


@pytest.fixture(scope="module")
def L():
    from post_weight_quantization_24_b200 import build, gptq
    build.build()
    return gptq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b((?:gptq|rtn)_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("gptq_hessian_accumulate", "gptq_quantize_layer", "rtn_minmax_quantize",
                     "gptq_hessian_create", "gptq_hessian_destroy", "gptq_inverse_factor"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings(L):
    from post_weight_quantization_24_b200 import gptq
    for code, name in gptq.STATUS.items():
        assert gptq.status_string(code).startswith(name)


def test_argument_errors_are_reported_before_any_launch(L):
    from post_weight_quantization_24_b200 import gptq
    ERR_ARG = -1
    fake = 256  # never dereferenced: every case fails a host-side check first
    # quantize_layer: null W, bad bits, group not dividing d_in, block not multiple of group
    args = dict(W=fake, dt=0, d_out=4, d_in=128, H=fake, bits=4, g=32, B=128, pd=0.01, ao=0,
                codes=fake, sc=fake, zr=fake, gidx=fake, perm=None, loss=None, ws=fake,
                wsb=1 << 40, s=None)

    def q(**kw):
        a = dict(args, **kw)
        return L.gptq_quantize_layer(a["W"], a["dt"], a["d_out"], a["d_in"], a["H"], a["bits"],
                                     a["g"], a["B"], a["pd"], a["ao"], a["codes"], a["sc"],
                                     a["zr"], a["gidx"], a["perm"], a["loss"], a["ws"], a["wsb"],
                                     a["s"])
    assert q(W=None) == ERR_ARG
    assert q(bits=1) == ERR_ARG and q(bits=9) == ERR_ARG
    assert q(g=48) == ERR_ARG                    # 128 % 48 != 0
    assert q(g=32, B=48) == ERR_ARG              # block not a multiple of 8 * ...
    assert q(g=64, B=96) == ERR_ARG              # block not a multiple of group
    assert q(B=256) == ERR_ARG                   # wider than one launch handles
    assert q(pd=-1.0) == ERR_ARG
    assert q(d_in=100) == ERR_ARG                # not a multiple of 8
    assert q(dt=7) == ERR_ARG
    assert q(ws=fake + 8) == ERR_ARG             # workspace not 256-byte aligned
    # workspace too small
    assert q(wsb=16) == -7
    # rtn
    assert L.rtn_minmax_quantize(None, 0, 4, 128, 4, 128, fake, fake, fake, None) == ERR_ARG
    assert L.rtn_minmax_quantize(fake, 0, 4, 128, 4, 96, fake, fake, fake, None) == ERR_ARG
    assert L.rtn_minmax_quantize(fake, 0, 4, 128, 9, 128, fake, fake, fake, None) == ERR_ARG
    # hessian
    h = ctypes.c_void_p()
    assert L.gptq_hessian_create(100, ctypes.byref(h)) == ERR_ARG
    assert L.gptq_hessian_accumulate_into(fake, 64, fake, -1, 0, None, None) == ERR_ARG
    assert L.gptq_hessian_accumulate_into(fake, 64, fake + 8, 10, 0, None, None) == ERR_ARG
    assert L.gptq_hessian_accumulate_into(fake, 64, fake, 10, 100, None, None) == ERR_ARG
    assert L.gptq_hessian_destroy(None) == 0
    assert gptq.STATUS[ERR_ARG] == "GPTQ_ERR_ARG"


def test_workspace_sizes(L):
    def r256(b):
        return (b + 255) // 256 * 256
    for d_out, d_in in ((512, 512), (11008, 4096), (4096, 11008), (3, 8)):
        nbl = (d_in + 127) // 128
        panel = 512 if d_in >= 9216 else 128      # the factorisation's split-panel width
        expect = (r256(40) + 2 * r256(d_in * d_in * 4) + r256(d_out * d_in * 4)
                  + 4 * r256(d_out * 512 * 4) + r256(d_out * d_in) + r256(d_in * 128 * 4)
                  + r256(nbl * 128 * 128 * 4) + r256(4 * d_in * panel * 4) + 2 * r256(d_in * 4))
        assert L.gptq_quantize_layer_workspace(d_out, d_in, 128) == expect
    assert L.gptq_quantize_layer_workspace(0, 512, 128) == 0


def test_missing_library_fails_loudly(monkeypatch):
    """No silent fallback: without the built library every entry point raises."""
    from post_weight_quantization_24_b200 import gptq
    monkeypatch.setattr(gptq, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libgptq_b200.so"))
    monkeypatch.setattr(gptq, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        gptq.lib()
    with pytest.raises(RuntimeError, match="not built"):
        gptq.quantize_layer_workspace(16, 128)


def test_host_tensors_are_refused():
    """The binding only marshals device tensors; host tensors raise instead of running on the CPU."""
    import torch
    from post_weight_quantization_24_b200 import gptq
    W = torch.zeros(4, 128, dtype=torch.float16)
    H = torch.eye(128)
    with pytest.raises(ValueError, match="CUDA"):
        gptq.rtn_minmax_quantize(W, 4, 32)
    with pytest.raises(ValueError, match="CUDA"):
        gptq.quantize_layer(W, H, bits=4, group_size=32)
    with pytest.raises(ValueError, match="CUDA"):
        gptq.quantize_layer_noalloc(W, H, bits=4, group_size=32)

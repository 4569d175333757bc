"""The C-ABI library: it loads on a machine without a GPU, exports exactly
the entry points include/sage.h declares, and its host-side validation
rejects bad arguments before touching the device (the refusal convention of
the FlyDSL pa_decode page: bad arguments and unsupported shapes are refused
with distinct errors)."""
import ctypes
import os
import re
import subprocess

import pytest

import quantized_attention_smoothing_b200 as sage
from quantized_attention_smoothing_b200 import build as sage_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage.h")


@pytest.fixture(scope="module")
def L():
    sage_build.build()
    return sage.lib()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:sage_status|size_t|const char\s*\*)\s+(sage_\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_documented_entry_points():
    names = _declared()
    for n in ("sage_hadamard_init", "sage_quant_qk", "sage_quant_v", "sage_attn_fwd",
              "sage_attn_decode"):
        assert n in names
    assert sorted(names) == sorted(sage.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for n in _declared():
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", sage.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(set(re.findall(r"\bT (sage_\w+)$", out, flags=re.M)))
    assert exported == _declared()


def test_status_strings(L):
    assert sage.status_string(0) == "SAGE_OK"
    assert sage.status_string(6) == "SAGE_ERR_TIMEOUT"
    assert sage.status_string(99) == "SAGE_ERR_UNKNOWN"


def test_workspace_sizes_are_host_only(L):
    # one fp32 statistic per (b, kv head, d): the K mean, the V multiplier 448 / a
    assert L.sage_quant_qk_workspace(1, 24, 24, 4096, 4096, 128) == 1 * 24 * 128 * 4
    assert L.sage_quant_v_workspace(1, 40, 32760, 128) == 1 * 40 * 128 * 4
    assert L.sage_quant_qkv_workspace(2, 32, 8, 4096, 4096, 64) == 2 * (2 * 8 * 64 * 4)
    assert L.sage_quant_qkv_workspace(1, 1, 0, 1, 1, 64) == 0
    assert L.sage_attn_fwd_workspace(1, 24, 24, 4096, 4096, 128) == 0
    assert L.sage_quant_qk_workspace(0, 1, 1, 1, 1, 64) == 0


def _cview(ptr=0x1000, size=(1, 2, 256, 64), stride=None):
    v = sage.CView4()
    v.ptr = ptr
    if stride is None:
        stride = (size[1] * size[2] * size[3], size[2] * size[3], size[3], 1)
    for i in range(4):
        v.size[i] = size[i]
        v.stride[i] = stride[i]
    return v


def _view(ptr=0x1000, size=(1, 2, 256, 64)):
    v = sage.View4()
    c = _cview(ptr, size)
    v.ptr = c.ptr
    for i in range(4):
        v.size[i] = c.size[i]
        v.stride[i] = c.stride[i]
    return v


def test_attn_fwd_validation_without_gpu(L):
    p = ctypes.c_void_p(0x10000)
    ok_out = _view(0x20000, (1, 2, 256, 64))
    # null pointer
    assert L.sage_attn_fwd(None, p, p, p, p, p, 1, 2, 2, 256, 256, 64, 64, 64, 0.125, 0,
                           ok_out, None, 0, None) == sage.SAGE_ERR_INVALID_ARG
    # output shape mismatch
    bad_out = _view(0x20000, (1, 2, 255, 64))
    assert L.sage_attn_fwd(p, p, p, p, p, p, 1, 2, 2, 256, 256, 64, 64, 64, 0.125, 0,
                           bad_out, None, 0, None) == sage.SAGE_ERR_INVALID_ARG
    # unsupported head dim / block size / GQA ratio
    out96 = _view(0x20000, (1, 2, 256, 96))
    assert L.sage_attn_fwd(p, p, p, p, p, p, 1, 2, 2, 256, 256, 96, 64, 64, 0.125, 0,
                           out96, None, 0, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_attn_fwd(p, p, p, p, p, p, 1, 2, 2, 256, 256, 64, 48, 64, 0.125, 0,
                           ok_out, None, 0, None) == sage.SAGE_ERR_UNSUPPORTED
    out3 = _view(0x20000, (1, 3, 256, 64))
    assert L.sage_attn_fwd(p, p, p, p, p, p, 1, 3, 2, 256, 256, 64, 64, 64, 0.125, 0,
                           out3, None, 0, None) == sage.SAGE_ERR_UNSUPPORTED
    # misaligned quantised operand
    q = ctypes.c_void_p(0x10008)
    assert L.sage_attn_fwd(q, p, p, p, p, p, 1, 2, 2, 256, 256, 64, 64, 64, 0.125, 0,
                           ok_out, None, 0, None) == sage.SAGE_ERR_ALIGNMENT
    # non-finite scale
    assert L.sage_attn_fwd(p, p, p, p, p, p, 1, 2, 2, 256, 256, 64, 64, 64, float("nan"), 0,
                           ok_out, None, 0, None) == sage.SAGE_ERR_INVALID_ARG


def test_quant_validation_without_gpu(L):
    p = ctypes.c_void_p(0x10000)
    # null handle
    assert L.sage_quant_qk(None, _cview(), _cview(), 64, 64, p, p, p, p, None, p, 1 << 20,
                           None) == sage.SAGE_ERR_INVALID_ARG
    # V: negative stride, unsupported D, missing workspace
    assert L.sage_quant_v(_cview(stride=(1, 1, -1, 1)), p, p, p, 1 << 20, None) == \
        sage.SAGE_ERR_INVALID_ARG
    assert L.sage_quant_v(_cview(size=(1, 2, 256, 96)), p, p, p, 1 << 20, None) == \
        sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_quant_v(_cview(), p, p, None, 0, None) == sage.SAGE_ERR_WORKSPACE
    assert L.sage_quant_v(_cview(), p, p, p, 16, None) == sage.SAGE_ERR_WORKSPACE
    assert L.sage_quant_v(_cview(), ctypes.c_void_p(0x10001), p, p, 1 << 20, None) == \
        sage.SAGE_ERR_ALIGNMENT
    # Q, K and V in one call: null handle, null V
    assert L.sage_quant_qkv(None, _cview(), _cview(), _cview(), 64, 64, p, p, p, p, None, p, p, p,
                            1 << 20, None) == sage.SAGE_ERR_INVALID_ARG
    assert L.sage_quant_qkv(p, _cview(), _cview(), _cview(ptr=0), 64, 64, p, p, p, p, None, p, p,
                            p, 1 << 20, None) == sage.SAGE_ERR_INVALID_ARG


def test_hadamard_init_argument_checks(L):
    h = ctypes.c_void_p()
    assert L.sage_hadamard_init(128, 0, None) == sage.SAGE_ERR_INVALID_ARG
    assert L.sage_hadamard_init(128, -1, ctypes.byref(h)) == sage.SAGE_ERR_INVALID_ARG
    assert L.sage_hadamard_init(96, 0, ctypes.byref(h)) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_hadamard_destroy(None) == sage.SAGE_OK


def test_decode_validation_without_gpu(L):
    """Argument marshalling of the decode entry point and its refusals."""
    p = ctypes.c_void_p(0x10000)
    q = _cview(size=(2, 4, 16, 128))
    out = _view(0x20000, (2, 4, 16, 128))
    args = [q, p, p, p, p, p, p, 2, 4, 16, 1, 128, 128, 64, 100, 4096, 0.088, 0, out, None, None, p,
            1 << 30, None]
    # null handle
    assert L.sage_attn_decode(None, *args) == sage.SAGE_ERR_INVALID_ARG
    # the Python wrapper passes the same argument count as the C declaration
    class FakeHandle:
        handle = None
    qt = __import__("torch").zeros((2, 4, 16, 128), dtype=__import__("torch").bfloat16)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_decode(FakeHandle(), qt, qt, qt, qt, qt, qt, qt, 128, 100, 4096, 0.088, qt,
                              None, stream=0)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG


def test_decode_mxfp4_marshalling_without_gpu(L):
    """The MXFP4-cache decode entry point: argument count of the binding and
    the null-handle refusal (nothing else is reachable without a device)."""
    p = ctypes.c_void_p(0x10000)
    q = _cview(size=(2, 1, 16, 128))
    out = _view(0x20000, (2, 1, 16, 128))
    args = [q, p, p, p, p, p, p, 2, 1, 16, 1, 128, 128, 64, 100, 4096, 0.088, out, None, None, p,
            1 << 30, None]
    assert L.sage_attn_decode_mxfp4(None, *args) == sage.SAGE_ERR_INVALID_ARG
    torch = __import__("torch")

    class FakeHandle:
        handle = None
    qt = torch.zeros((2, 1, 16, 128), dtype=torch.bfloat16)
    u8 = torch.zeros((4, 1, 128, 64), dtype=torch.uint8)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_decode_mxfp4(FakeHandle(), qt, u8, u8, u8, u8, torch.zeros((2, 4), dtype=torch.int32),
                                    torch.zeros(2, dtype=torch.int32), 128, 4, 4096, 0.088, qt,
                                    ws=u8, stream=0)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG

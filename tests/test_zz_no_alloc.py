"""sage_quant_qk_noalloc: the quantisation entry point for callers that
cannot allocate device memory when they call it (a serving loop whose device
memory is budgeted once at start-up, or code that must not risk the implicit
device synchronisation of cudaMalloc / cudaFree). It keeps its scratch in a
fixed array inside the library instead of a caller workspace.

Checked through the C ABI: two calls in a row (different shapes, so the
second call sees the first call's leftovers in the shared scratch) give
exactly the outputs of sage_quant_qk with a caller workspace, and a call
whose scratch need exceeds the fixed 8 MiB is refused before any launch.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

import quantized_attention_smoothing_b200 as sage
import workloads

pytestmark = pytest.mark.gpu


def _quant_with_workspace(h, q, k, blk_q, blk_k):
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    bufs = sage.QuantBuffers(B, H, Hk, Lq, Lk, D, blk_q, blk_k)
    sage.sage_quant_qk(h, q, k, blk_q, blk_k, bufs.q8, bufs.q_scale, bufs.k8, bufs.k_scale,
                       bufs.k_mean, bufs.ws)
    return bufs


def _quant_no_alloc(h, q, k, blk_q, blk_k):
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    bufs = sage.QuantBuffers(B, H, Hk, Lq, Lk, D, blk_q, blk_k)
    st = sage.lib().sage_quant_qk_noalloc(
        h.handle, sage._view(q, sage.CView4), sage._view(k, sage.CView4), blk_q, blk_k,
        sage._ptr(bufs.q8), sage._ptr(bufs.q_scale), sage._ptr(bufs.k8), sage._ptr(bufs.k_scale),
        sage._ptr(bufs.k_mean), sage._stream(None))
    assert st == sage.SAGE_OK, sage.status_string(st)
    return bufs


def _same(a, b):
    for name in ("q8", "q_scale", "k8", "k_scale", "k_mean"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_no_alloc_matches_workspace_entry_point_twice():
    from quantized_attention_smoothing_b200 import build
    build.build()
    h = sage.Hadamard(128)
    shapes = [
        dict(B=1, H=24, Hk=24, L=4096, D=128, kbias_std=2.0, outlier_channels=4, seed=31),
        dict(B=2, H=4, Hk=2, L=777, D=128, kbias_std=3.0, heavy_frac=0.02, seed=32),
    ]
    for sh in shapes:                     # two calls in a row, different sizes
        q, k, v = workloads.make_prefill(**sh)
        q, k = q.cuda(), k.cuda()
        ref = _quant_with_workspace(h, q, k, 128, 64)
        got = _quant_no_alloc(h, q, k, 128, 64)
        torch.cuda.synchronize()
        assert sage.sage_device_error() == sage.SAGE_OK
        _same(ref, got)


def test_no_alloc_rejects_sizes_beyond_its_scratch():
    h = sage.Hadamard(128)
    # 32768 kv heads of D = 128 need 32768 * 128 * 4 B = 16 MiB of K means
    big = sage.CView4()
    big.ptr = 0x10000
    sizes = (1, 32768, 1, 128)
    strides = (32768 * 128, 128, 128, 1)
    for i in range(4):
        big.size[i] = sizes[i]
        big.stride[i] = strides[i]
    p = ctypes.c_void_p(0x10000)
    st = sage.lib().sage_quant_qk_noalloc(h.handle, big, big, 128, 64, p, p, p, p, None, None)
    assert st == sage.SAGE_ERR_WORKSPACE

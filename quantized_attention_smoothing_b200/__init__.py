"""Python binding of libsage, the sm_100a quantized-attention library.

Argument marshalling only: every step of the path runs in the CUDA kernels
behind the C ABI declared in ``include/sage.h``; there is no CPU or PyTorch
fallback, and a missing or unloadable ``libsage.so`` raises at once.

The functions keep the C names. Tensors are torch tensors on the current
CUDA device; views are passed with their own strides (no ``.contiguous()``).
``stream`` defaults to torch's current stream.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage.so")

SAGE_OK = 0
SAGE_ERR_INVALID_ARG = 1
SAGE_ERR_UNSUPPORTED = 2
SAGE_ERR_ALIGNMENT = 3
SAGE_ERR_WORKSPACE = 4
SAGE_ERR_CUDA = 5
SAGE_ERR_TIMEOUT = 6

EXPORTS = (
    "sage_hadamard_init", "sage_hadamard_destroy", "sage_hadamard_matrix",
    "sage_quant_qk_workspace", "sage_quant_qk", "sage_quant_qk_noalloc",
    "sage_quant_v_workspace", "sage_quant_v", "sage_quant_k", "sage_quant_qkv_workspace",
    "sage_quant_qkv",
    "sage_attn_fwd_workspace", "sage_attn_fwd", "sage_attn_fwd_q16", "sage_attn_decode_workspace",
    "sage_attn_decode", "sage_status_string", "sage_device_error", "sage_device_error_where",
    "sage_wait_probe", "sage_quant_qk_mx", "sage_attn_fwd_mx", "sage_attn_decode_mxfp4",
)

SAGE_KERNEL_ATTN = 1
SAGE_KERNEL_DECODE = 2
SAGE_KERNEL_PROBE = 3
SAGE_KERNEL_ATTN_MX = 4
SAGE_KV_PER_TENSOR_SCALES = 1
SAGE_KV_V_TRANSPOSED = 2


class SageError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s failed: %s" % (where, status_string(status)))


class CView4(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("size", ctypes.c_int64 * 4),
                ("stride", ctypes.c_int64 * 4)]


class View4(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("size", ctypes.c_int64 * 4),
                ("stride", ctypes.c_int64 * 4)]


_lib = None


def lib():
    """Load libsage.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OSError("libsage.so not built: run `python -m quantized_attention_smoothing_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.sage_status_string.restype = ctypes.c_char_p
    L.sage_status_string.argtypes = [i32]
    L.sage_hadamard_init.restype = i32
    L.sage_hadamard_init.argtypes = [i32, i32, ctypes.POINTER(vp)]
    L.sage_hadamard_destroy.restype = i32
    L.sage_hadamard_destroy.argtypes = [vp]
    L.sage_hadamard_matrix.restype = i32
    L.sage_hadamard_matrix.argtypes = [vp, vp, ctypes.POINTER(i32)]
    L.sage_quant_qk_workspace.restype = sz
    L.sage_quant_qk_workspace.argtypes = [i32] * 6
    L.sage_quant_qk.restype = i32
    L.sage_quant_qk.argtypes = [vp, CView4, CView4, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.sage_quant_qk_noalloc.restype = i32
    L.sage_quant_qk_noalloc.argtypes = [vp, CView4, CView4, i32, i32, vp, vp, vp, vp, vp, vp]
    L.sage_quant_v_workspace.restype = sz
    L.sage_quant_v_workspace.argtypes = [i32] * 4
    L.sage_quant_v.restype = i32
    L.sage_quant_v.argtypes = [CView4, vp, vp, vp, sz, vp]
    L.sage_quant_k.restype = i32
    L.sage_quant_k.argtypes = [vp, CView4, i32, vp, vp, vp, vp, sz, vp]
    L.sage_quant_qkv_workspace.restype = sz
    L.sage_quant_qkv_workspace.argtypes = [i32] * 6
    L.sage_quant_qkv.restype = i32
    L.sage_quant_qkv.argtypes = [vp, CView4, CView4, CView4, i32, i32] + [vp] * 8 + [sz, vp]
    L.sage_attn_fwd_workspace.restype = sz
    L.sage_attn_fwd_workspace.argtypes = [i32] * 6
    L.sage_attn_fwd.restype = i32
    L.sage_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp] + [i32] * 8 + [f32, i32, View4, vp, sz, vp]
    L.sage_attn_fwd_q16.restype = i32
    L.sage_attn_fwd_q16.argtypes = [vp, CView4, i32, vp, vp, vp, vp, i32, i32, i32, f32, i32, View4,
                                    vp, sz, vp]
    L.sage_attn_decode_workspace.restype = sz
    L.sage_attn_decode_workspace.argtypes = [i32] * 6
    L.sage_attn_decode.restype = i32
    L.sage_attn_decode.argtypes = [vp, CView4, vp, vp, vp, vp, vp, vp] + [i32] * 9 + \
        [f32, i32, View4, vp, vp, vp, sz, vp]
    L.sage_attn_decode_mxfp4.restype = i32
    L.sage_attn_decode_mxfp4.argtypes = [vp, CView4, vp, vp, vp, vp, vp, vp] + [i32] * 9 + \
        [f32, View4, vp, vp, vp, sz, vp]
    L.sage_device_error.restype = i32
    L.sage_device_error.argtypes = [vp]
    L.sage_device_error_where.restype = i32
    L.sage_device_error_where.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.sage_quant_qk_mx.restype = i32
    L.sage_quant_qk_mx.argtypes = [vp, CView4, CView4, vp, vp, vp, vp, vp, vp, sz, vp]
    L.sage_attn_fwd_mx.restype = i32
    L.sage_attn_fwd_mx.argtypes = [vp] * 6 + [i32] * 6 + [f32, i32, View4, vp, sz, vp]
    L.sage_wait_probe.restype = i32
    L.sage_wait_probe.argtypes = [ctypes.c_uint64, vp]
    _lib = L
    return L


def status_string(status):
    return lib().sage_status_string(int(status)).decode()


def _check(status, where):
    if status != SAGE_OK:
        raise SageError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _view(t, cls):
    if t.dim() != 4:
        raise ValueError("expected a 4-d tensor view, got shape %s" % (tuple(t.shape),))
    v = cls()
    v.ptr = t.data_ptr()
    for i in range(4):
        v.size[i] = t.shape[i]
        v.stride[i] = t.stride(i)
    return v


class Hadamard:
    """Owns a sage_hadamard handle (built once per head dim and device)."""

    def __init__(self, head_dim, device=None):
        if device is None:
            device = torch.cuda.current_device()
        h = ctypes.c_void_p()
        _check(lib().sage_hadamard_init(int(head_dim), int(device), ctypes.byref(h)),
               "sage_hadamard_init")
        self.handle = h
        self.head_dim = int(head_dim)
        self.device = int(device)

    def matrix(self):
        import numpy as np
        out = np.zeros((self.head_dim, self.head_dim), dtype=np.int8)
        d = ctypes.c_int()
        _check(lib().sage_hadamard_matrix(self.handle, out.ctypes.data_as(ctypes.c_void_p),
                                          ctypes.byref(d)), "sage_hadamard_matrix")
        return out

    def close(self):
        if self.handle is not None and _lib is not None:
            _lib.sage_hadamard_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sage_hadamard_init(head_dim, device=None):
    return Hadamard(head_dim, device)


def sage_quant_qk_workspace(B, H, Hk, Lq, Lk, D):
    return int(lib().sage_quant_qk_workspace(B, H, Hk, Lq, Lk, D))


def sage_quant_v_workspace(B, Hk, L, D):
    return int(lib().sage_quant_v_workspace(B, Hk, L, D))


def sage_attn_fwd_workspace(B, H, Hk, Lq, Lk, D):
    return int(lib().sage_attn_fwd_workspace(B, H, Hk, Lq, Lk, D))


def sage_attn_decode_workspace(B, T, H, Hk, D, window):
    return int(lib().sage_attn_decode_workspace(B, T, H, Hk, D, window))


def sage_quant_qk(h, q, k, blk_q, blk_k, q8, q_scale, k8, k_scale, k_mean=None, ws=None,
                  stream=None):
    _check(lib().sage_quant_qk(h.handle, _view(q, CView4), _view(k, CView4), int(blk_q),
                               int(blk_k), _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale),
                               _ptr(k_mean), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream)), "sage_quant_qk")


def sage_quant_qk_noalloc(h, q, k, blk_q, blk_k, q8, q_scale, k8, k_scale, k_mean=None,
                          stream=None):
    """sage_quant_qk without a caller workspace: for callers that cannot
    allocate device memory at the call (scratch comes from a fixed array in
    the library; see include/sage.h for its limit and the sharing rules)."""
    _check(lib().sage_quant_qk_noalloc(h.handle, _view(q, CView4), _view(k, CView4), int(blk_q),
                                       int(blk_k), _ptr(q8), _ptr(q_scale), _ptr(k8),
                                       _ptr(k_scale), _ptr(k_mean), _stream(stream)),
           "sage_quant_qk_noalloc")


def sage_quant_k(h, k, blk_k, k8, k_scale, k_mean=None, ws=None, stream=None):
    _check(lib().sage_quant_k(h.handle, _view(k, CView4), int(blk_k), _ptr(k8), _ptr(k_scale),
                              _ptr(k_mean), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                              _stream(stream)), "sage_quant_k")


def sage_attn_fwd_q16(h, q, blk_q, k8, k_scale, v8_t, v_scale, Hk, Lk, blk_k, softmax_scale,
                      causal, out, ws=None, stream=None):
    _check(lib().sage_attn_fwd_q16(h.handle, _view(q, CView4), int(blk_q), _ptr(k8), _ptr(k_scale),
                                   _ptr(v8_t), _ptr(v_scale), int(Hk), int(Lk), int(blk_k),
                                   float(softmax_scale), 1 if causal else 0, _view(out, View4),
                                   _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                   _stream(stream)), "sage_attn_fwd_q16")


def sage_quant_qkv_workspace(B, H, Hk, Lq, Lk, D):
    return int(lib().sage_quant_qkv_workspace(B, H, Hk, Lq, Lk, D))


def sage_quant_qkv(h, q, k, v, blk_q, blk_k, q8, q_scale, k8, k_scale, v8_t, v_scale, k_mean=None,
                   ws=None, stream=None):
    _check(lib().sage_quant_qkv(h.handle, _view(q, CView4), _view(k, CView4), _view(v, CView4),
                                int(blk_q), int(blk_k), _ptr(q8), _ptr(q_scale), _ptr(k8),
                                _ptr(k_scale), _ptr(k_mean), _ptr(v8_t), _ptr(v_scale), _ptr(ws),
                                0 if ws is None else ws.numel() * ws.element_size(),
                                _stream(stream)), "sage_quant_qkv")


def sage_quant_v(v, v8_t, v_scale, ws=None, stream=None):
    _check(lib().sage_quant_v(_view(v, CView4), _ptr(v8_t), _ptr(v_scale), _ptr(ws),
                              0 if ws is None else ws.numel() * ws.element_size(),
                              _stream(stream)), "sage_quant_v")


def sage_attn_fwd(q8, q_scale, k8, k_scale, v8_t, v_scale, B, H, Hk, Lq, Lk, D, blk_q, blk_k,
                  softmax_scale, causal, out, ws=None, stream=None):
    _check(lib().sage_attn_fwd(_ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(v8_t),
                               _ptr(v_scale), B, H, Hk, Lq, Lk, D, blk_q, blk_k,
                               float(softmax_scale), int(bool(causal)), _view(out, View4),
                               _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream)), "sage_attn_fwd")


def sage_attn_decode(h, q, k_cache, v_cache, k_scale, v_scale, page_table, ctx_lens, page_size,
                     num_pages, window, softmax_scale, out, ws=None, stream=None, q8_out=None,
                     q_scale_out=None, kv_flags=0):
    B, T, H, D = q.shape
    Hk = k_cache.shape[1]
    max_pages = page_table.shape[1]
    if ws is None:
        # the split-KV partials (none when every (sequence, kv head) runs in
        # one CTA)
        n = sage_attn_decode_workspace(B, T, H, Hk, D, window)
        if n > 0:
            ws = torch.empty((n,), dtype=torch.uint8, device=q.device)
    _check(lib().sage_attn_decode(h.handle, _view(q, CView4), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(k_scale), _ptr(v_scale), _ptr(page_table), _ptr(ctx_lens),
                                  B, T, H, Hk, D, int(page_size), int(max_pages), int(num_pages),
                                  int(window), float(softmax_scale), int(kv_flags), _view(out, View4),
                                  _ptr(q8_out), _ptr(q_scale_out), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream)), "sage_attn_decode")


def sage_attn_decode_mxfp4(h, q, k_cache, v_cache, k_sf, v_sf, page_table, ctx_lens, page_size,
                           num_pages, window, softmax_scale, out, ws=None, stream=None, q8_out=None,
                           q_scale_out=None):
    """Paged decode over an MXFP4 cache: k_cache / v_cache uint8 [num_pages,
    Hk, page, D / 2] (two E2M1 codes a byte), k_sf / v_sf uint8 e8m0
    [num_pages, Hk, page, D / 32]."""
    B, T, H, D = q.shape
    Hk = k_cache.shape[1]
    max_pages = page_table.shape[1]
    if ws is None:
        n = sage_attn_decode_workspace(B, T, H, Hk, D, window)
        if n > 0:
            ws = torch.empty((n,), dtype=torch.uint8, device=q.device)
    _check(lib().sage_attn_decode_mxfp4(h.handle, _view(q, CView4), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(k_sf), _ptr(v_sf), _ptr(page_table), _ptr(ctx_lens),
                                        B, T, H, Hk, D, int(page_size), int(max_pages), int(num_pages),
                                        int(window), float(softmax_scale), _view(out, View4),
                                        _ptr(q8_out), _ptr(q_scale_out), _ptr(ws),
                                        0 if ws is None else ws.numel() * ws.element_size(),
                                        _stream(stream)), "sage_attn_decode_mxfp4")


def sage_quant_qk_mx(h, q, k, q4, q_sf, k4, k_sf, k_mean=None, ws=None, stream=None):
    _check(lib().sage_quant_qk_mx(h.handle, _view(q, CView4), _view(k, CView4), _ptr(q4), _ptr(q_sf),
                                  _ptr(k4), _ptr(k_sf), _ptr(k_mean), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "sage_quant_qk_mx")


def sage_attn_fwd_mx(q4, q_sf, k4, k_sf, v8_t, v_scale, B, H, Hk, Lq, Lk, D, softmax_scale, causal,
                     out, ws=None, stream=None):
    _check(lib().sage_attn_fwd_mx(_ptr(q4), _ptr(q_sf), _ptr(k4), _ptr(k_sf), _ptr(v8_t), _ptr(v_scale),
                                  B, H, Hk, Lq, Lk, D, float(softmax_scale), int(bool(causal)),
                                  _view(out, View4), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "sage_attn_fwd_mx")


def sage_device_error(stream=None):
    return int(lib().sage_device_error(_stream(stream)))


def sage_device_error_where(stream=None):
    """(status, kernel id, site) of the error words; reads and clears them."""
    k = ctypes.c_int()
    s = ctypes.c_int()
    st = int(lib().sage_device_error_where(_stream(stream), ctypes.byref(k), ctypes.byref(s)))
    return st, k.value, s.value


def sage_wait_probe(limit_ns, stream=None):
    _check(lib().sage_wait_probe(int(limit_ns), _stream(stream)), "sage_wait_probe")


# ---------------------------------------------------------------- convenience

def round_up(x, m):
    return (x + m - 1) // m * m


class QuantBuffers:
    """Device buffers of the quantised operands for one [B, H(k), L, D] shape."""

    def __init__(self, B, H, Hk, Lq, Lk, D, blk_q, blk_k, device=None):
        dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.shape = (B, H, Hk, Lq, Lk, D, blk_q, blk_k)
        self.q8 = torch.empty((B, H, round_up(Lq, 128), D), dtype=torch.int8, device=dev)
        self.q_scale = torch.empty((B, H, math.ceil(Lq / blk_q)), dtype=torch.float32, device=dev)
        self.k8 = torch.empty((B, Hk, round_up(Lk, 128), D), dtype=torch.int8, device=dev)
        self.k_scale = torch.empty((B, Hk, math.ceil(Lk / blk_k)), dtype=torch.float32, device=dev)
        self.k_mean = torch.empty((B, Hk, D), dtype=torch.float32, device=dev)
        self.v8_t = torch.empty((B, Hk, D, round_up(Lk, 128)), dtype=torch.uint8, device=dev)
        self.v_scale = torch.empty((B, Hk, D), dtype=torch.float32, device=dev)
        ws = max(sage_quant_qkv_workspace(B, H, Hk, Lq, Lk, D), sage_quant_qk_workspace(B, H, Hk, Lq, Lk, D),
                 sage_attn_fwd_workspace(B, H, Hk, Lq, Lk, D), 16)
        self.ws = torch.empty((ws,), dtype=torch.uint8, device=dev)
        # for K and V without Q: the V quantisation has its own workspace so
        # it can run on a second stream beside the K quantisation
        self.ws_v = torch.empty((max(sage_quant_v_workspace(B, Hk, Lk, D), 16),), dtype=torch.uint8,
                                device=dev)
        self.side = torch.cuda.Stream(device=dev)


def sage_attention(h, q, k, v, blk_q, blk_k, softmax_scale, causal=False, out=None, bufs=None,
                   stream=None):
    """Quantise Q/K/V and run the quantised attention; q, k, v are [B, H(k),
    L, D] bf16 views. Returns (out, bufs); out defaults to a [B, H, L, D]
    view of a [B, L, H, D] tensor (the video-DiT layout)."""
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    if bufs is None:
        bufs = QuantBuffers(B, H, Hk, Lq, Lk, D, blk_q, blk_k, q.device.index)
    if out is None:
        out = torch.empty((B, Lq, H, D), dtype=torch.bfloat16, device=q.device).permute(0, 2, 1, 3)
    quantise(h, q, k, v, blk_q, blk_k, bufs, stream)
    sage_attn_fwd(bufs.q8, bufs.q_scale, bufs.k8, bufs.k_scale, bufs.v8_t, bufs.v_scale, B, H, Hk,
                  Lq, Lk, D, blk_q, blk_k, softmax_scale, causal, out, None, stream)
    return out, bufs


def sage_attention_q16(h, q, k, v, blk_q, blk_k, softmax_scale, causal=False, out=None, bufs=None,
                       stream=None):
    """sage_attention with Q rotated and quantised inside the attention
    kernel (sage_quant_k + sage_quant_v beside it + sage_attn_fwd_q16): the
    same output bits, no q8 / q_scale round trip."""
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    if bufs is None:
        bufs = QuantBuffers(B, H, Hk, Lq, Lk, D, blk_q, blk_k, q.device.index)
    if out is None:
        out = torch.empty((B, Lq, H, D), dtype=torch.bfloat16, device=q.device).permute(0, 2, 1, 3)
    quantise(h, None, k, v, blk_q, blk_k, bufs, stream)
    sage_attn_fwd_q16(h, q, blk_q, bufs.k8, bufs.k_scale, bufs.v8_t, bufs.v_scale, Hk, Lk, blk_k,
                      softmax_scale, causal, out, None, stream)
    return out, bufs


def quantise(h, q, k, v, blk_q, blk_k, bufs, stream=None):
    """sage_quant_qkv on `stream`; when q is None, sage_quant_k on `stream`
    and, beside it, sage_quant_v on the buffers' second stream (the two read
    and write disjoint buffers), work issued to `stream` afterwards waiting
    for both."""
    s = torch.cuda.current_stream() if stream is None else stream
    if q is not None:
        sage_quant_qkv(h, q, k, v, blk_q, blk_k, bufs.q8, bufs.q_scale, bufs.k8, bufs.k_scale,
                       bufs.v8_t, bufs.v_scale, bufs.k_mean, bufs.ws, s)
        return
    fork = torch.cuda.Event()
    fork.record(s)
    bufs.side.wait_event(fork)
    sage_quant_k(h, k, blk_k, bufs.k8, bufs.k_scale, bufs.k_mean, bufs.ws, s)
    sage_quant_v(v, bufs.v8_t, bufs.v_scale, bufs.ws_v, bufs.side)
    join = torch.cuda.Event()
    join.record(bufs.side)
    s.wait_event(join)


class MxBuffers:
    """Device buffers of the MXFP4 Q / K and FP8 V operands for one shape."""

    def __init__(self, B, H, Hk, Lq, Lk, D, device=None):
        dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        LpQ, LpK = round_up(Lq, 128), round_up(Lk, 128)
        self.q4 = torch.empty((B, H, LpQ, D // 2), dtype=torch.uint8, device=dev)
        self.q_sf = torch.empty((B, H, LpQ // 128, 512), dtype=torch.uint8, device=dev)
        self.k4 = torch.empty((B, Hk, LpK, D // 2), dtype=torch.uint8, device=dev)
        self.k_sf = torch.empty((B, Hk, LpK // 128, 512), dtype=torch.uint8, device=dev)
        self.k_mean = torch.empty((B, Hk, D), dtype=torch.float32, device=dev)
        self.v8_t = torch.empty((B, Hk, D, LpK), dtype=torch.uint8, device=dev)
        self.v_scale = torch.empty((B, Hk, D), dtype=torch.float32, device=dev)
        self.ws = torch.empty((max(sage_quant_qk_workspace(B, H, Hk, Lq, Lk, D), 16),),
                              dtype=torch.uint8, device=dev)
        self.ws_v = torch.empty((max(sage_quant_v_workspace(B, Hk, Lk, D), 16),), dtype=torch.uint8,
                                device=dev)


def sage_attention_mx(h, q, k, v, softmax_scale, causal=False, out=None, bufs=None, stream=None):
    """MXFP4 Q / K + FP8 V path: sage_quant_qk_mx + sage_quant_v +
    sage_attn_fwd_mx on [B, H(k), L, D] bf16 views. Returns (out, bufs)."""
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    if bufs is None:
        bufs = MxBuffers(B, H, Hk, Lq, Lk, D, q.device.index)
    if out is None:
        out = torch.empty((B, Lq, H, D), dtype=torch.bfloat16, device=q.device).permute(0, 2, 1, 3)
    s = torch.cuda.current_stream() if stream is None else stream
    sage_quant_qk_mx(h, q, k, bufs.q4, bufs.q_sf, bufs.k4, bufs.k_sf, bufs.k_mean, bufs.ws, s)
    sage_quant_v(v, bufs.v8_t, bufs.v_scale, bufs.ws_v, s)
    sage_attn_fwd_mx(bufs.q4, bufs.q_sf, bufs.k4, bufs.k_sf, bufs.v8_t, bufs.v_scale, B, H, Hk, Lq, Lk,
                     D, softmax_scale, causal, out, None, s)
    return out, bufs

"""CPU oracle for SageAttention-style quantized attention.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's
CPU-baseline leg may import this module; the product path never does.  The
arithmetic lives in ``sage_oracle.c`` (plain C, fp64 where the method fixes no
precision); this file only marshals numpy arrays to it, one (batch, head)
slice per call, optionally over a thread pool (ctypes releases the GIL).

bf16 tensors are passed as ``numpy.uint16`` bit patterns, e4m3 codes as
``numpy.uint8``. Logical layouts follow the pages: prefill inputs are
[B, H, L, D] views of any stride ("sage_attn3" API page; "Sage v2
improvements": no forced contiguous copies).
"""
import ctypes
import os
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

KEY_TILE = 128          # softmax key-tile width of the oracle's online softmax
E4M3_MAX = 448.0        # OCP e4m3 largest finite value
INT8_MAX = 127.0

_lib = None
_i8p = ctypes.POINTER(ctypes.c_int8)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)


_lib_lock = threading.Lock()


def lib():
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:                     # worker threads may ask for it at once
        return _load()


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.or_bf16_to_f32.restype = ctypes.c_float
        L.or_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.or_f64_to_bf16.restype = ctypes.c_uint16
        L.or_f64_to_bf16.argtypes = [ctypes.c_double]
        L.or_e4m3_decode.restype = ctypes.c_double
        L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.or_e4m3_encode.restype = ctypes.c_uint8
        L.or_e4m3_encode.argtypes = [ctypes.c_double]
        L.or_hadamard.restype = ctypes.c_int
        L.or_hadamard.argtypes = [ctypes.c_int, _i32p]
        L.or_fwht_rows_f32.restype = None
        L.or_fwht_rows_f32.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int]
        L.or_k_mean.restype = None
        L.or_k_mean.argtypes = [_u16p, ctypes.c_int, ctypes.c_int, _f32p]
        L.or_quant_i8_head.restype = None
        L.or_quant_i8_head.argtypes = [_u16p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, _i8p, _f32p]
        L.or_quant_v_head.restype = None
        L.or_quant_v_head.argtypes = [_u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8p, _f32p]
        L.or_attn_head.restype = None
        L.or_attn_head.argtypes = [_i8p, _f32p, _i8p, _f32p, _u8p, ctypes.c_int64, _f32p,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                   _i32p, ctypes.c_int, _u16p, _f64p, _f64p]
        L.or_p_fp32_delta.restype = ctypes.c_double
        L.or_p_fp32_delta.argtypes = [ctypes.c_double, ctypes.c_double]
        L.or_e4m3_flip_step.restype = ctypes.c_double
        L.or_e4m3_flip_step.argtypes = [ctypes.c_double, ctypes.c_double]
        L.or_attn_exact_head.restype = None
        L.or_attn_exact_head.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_double, ctypes.c_int, _i32p,
                                         ctypes.c_int, _f64p]
        L.or_e2m1_decode.restype = ctypes.c_double
        L.or_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.or_e2m1_encode.restype = ctypes.c_uint8
        L.or_e2m1_encode.argtypes = [ctypes.c_double]
        L.or_quant_mxfp4_head.restype = None
        L.or_quant_mxfp4_head.argtypes = [_u16p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _u8p, _u8p]
        L.or_attn_mxfp4_head.restype = None
        L.or_attn_mxfp4_head.argtypes = [_u8p, _u8p, _u8p, _u8p, _u8p, ctypes.c_int64, _f32p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                         ctypes.c_int, ctypes.c_int, _i32p, ctypes.c_int, _u16p,
                                         _f64p, _f64p]
        L.or_decode_quant_q_row.restype = None
        L.or_decode_quant_q_row.argtypes = [_u16p, ctypes.c_int, _u8p, _f32p]
        L.or_decode_seq_flags.restype = None
        L.or_decode_seq_flags.argtypes = [_u16p, _u8p, _u8p, _f32p, _f32p, _i32p, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                          _u16p, _f64p, _f64p]
        L.or_decode_seq.restype = None
        L.or_decode_seq.argtypes = [_u16p, _u8p, _u8p, _f32p, _f32p, _i32p, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_double, _u16p, _f64p]
        L.or_decode_seq_mxkv.restype = None
        L.or_decode_seq_mxkv.argtypes = [_u16p, _u8p, _u8p, _u8p, _u8p, _i32p, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_double, _u16p, _f64p, _f64p]
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def _pool_map(fn, items, threads):
    items = list(items)
    if threads is None:
        threads = os.cpu_count() or 1
    if threads <= 1 or len(items) <= 1:
        return [fn(x) for x in items]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


def round_up(x, m):
    return (x + m - 1) // m * m


# ---------------------------------------------------------------- formats

def bf16_to_f32(u16):
    """Exact widening of bf16 bit patterns to float32."""
    u16 = np.asarray(u16, dtype=np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16(x):
    """Round-to-nearest-even of doubles to bf16 bit patterns (one rounding)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    f = lib().or_f64_to_bf16
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def e4m3_decode(codes):
    L = lib()
    table = np.array([L.or_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x):
    x = np.asarray(x, dtype=np.float64)
    f = lib().or_e4m3_encode
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


# ---------------------------------------------------------------- Hadamard

def hadamard(D):
    """Sylvester Hadamard matrix H_D (int32 +-1), built once per D
    ("Sage v2 improvements": the matrix is created once and reused)."""
    h = np.zeros((D, D), dtype=np.int32)
    if lib().or_hadamard(D, _p(h, _i32p)) != 0:
        raise ValueError("D must be a power of two")
    return h


def fwht_f32(x):
    """fp32 butterfly rotation x -> x * H along the last axis."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    D = x.shape[-1]
    lib().or_fwht_rows_f32(_p(x, _f32p), x.size // D, D)
    return x


# ---------------------------------------------------------------- quantisation

def k_mean(k):
    """Per-(b, h) mean of K over the sequence. k: uint16 [B, Hk, L, D]."""
    B, Hk, L, D = k.shape
    out = np.zeros((B, Hk, D), dtype=np.float32)
    for b in range(B):
        for h in range(Hk):
            kk = np.ascontiguousarray(k[b, h])
            lib().or_k_mean(_p(kk, _u16p), L, D, _p(out[b, h], _f32p))
    return out


def _quant_i8(x, mean, blk, threads):
    B, H, L, D = x.shape
    Lpad = round_up(L, 128)
    nb = (L + blk - 1) // blk
    codes = np.zeros((B, H, Lpad, D), dtype=np.int8)
    scales = np.zeros((B, H, nb), dtype=np.float32)

    def one(bh):
        b, h = bh
        xx = np.ascontiguousarray(x[b, h])
        mp = None
        if mean is not None:
            mm = np.ascontiguousarray(mean[b, h], dtype=np.float32)
            mp = _p(mm, _f32p)
        cc = np.zeros((Lpad, D), dtype=np.int8)
        ss = np.zeros((nb,), dtype=np.float32)
        lib().or_quant_i8_head(_p(xx, _u16p), mp, L, D, blk, Lpad, _p(cc, _i8p), _p(ss, _f32p))
        codes[b, h] = cc
        scales[b, h] = ss

    _pool_map(one, [(b, h) for b in range(B) for h in range(H)], threads)
    return codes, scales


def quant_qk(q, k, blk_q, blk_k, threads=None):
    """Smooth K, rotate Q and K, quantise both to INT8 per token block.
    q: uint16 [B, H, Lq, D]; k: uint16 [B, Hk, Lk, D]."""
    kmean = k_mean(k)
    q8, qs = _quant_i8(q, None, blk_q, threads)
    k8, ks = _quant_i8(k, kmean, blk_k, threads)
    return {"q8": q8, "qs": qs, "k8": k8, "ks": ks, "kmean": kmean}


def quant_v(v, threads=None):
    """FP8 e4m3 per-channel quantisation of V, written transposed.
    v: uint16 [B, Hk, L, D] -> v8t uint8 [B, Hk, D, Lpad], vs float32 [B, Hk, D]."""
    B, H, L, D = v.shape
    Lpad = round_up(L, 128)
    v8t = np.zeros((B, H, D, Lpad), dtype=np.uint8)
    vs = np.zeros((B, H, D), dtype=np.float32)

    def one(bh):
        b, h = bh
        vv = np.ascontiguousarray(v[b, h])
        cc = np.zeros((D, Lpad), dtype=np.uint8)
        ss = np.zeros((D,), dtype=np.float32)
        lib().or_quant_v_head(_p(vv, _u16p), L, D, Lpad, _p(cc, _u8p), _p(ss, _f32p))
        v8t[b, h] = cc
        vs[b, h] = ss

    _pool_map(one, [(b, h) for b in range(B) for h in range(H)], threads)
    return v8t, vs


# ---------------------------------------------------------------- attention

def attn(q8, qs, k8, ks, v8t, vs, Lq, Lk, blk_q, blk_k, softmax_scale, causal, rows=None,
         quantize_p=True, threads=None, want_f64=False, want_flip=False):
    """Quantised attention over the quantised operands.
    Returns bf16 bits [B, H, nrows, D] (and the fp64 values if want_f64, and
    then also the per-element fp32 P-rounding margin if want_flip)."""
    B, H, _, D = q8.shape
    Hk = k8.shape[1]
    group = H // Hk
    want_f64 = want_f64 or want_flip
    if rows is None:
        rows = np.arange(Lq, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    n = rows.size
    out = np.zeros((B, H, n, D), dtype=np.uint16)
    o64 = np.zeros((B, H, n, D), dtype=np.float64) if want_f64 else None
    flip = np.zeros((B, H, n, D), dtype=np.float64) if want_flip else None

    def one(bh):
        b, h = bh
        hk = h // group
        a_q8 = np.ascontiguousarray(q8[b, h])
        a_qs = np.ascontiguousarray(qs[b, h])
        a_k8 = np.ascontiguousarray(k8[b, hk])
        a_ks = np.ascontiguousarray(ks[b, hk])
        a_v8 = np.ascontiguousarray(v8t[b, hk])
        a_vs = np.ascontiguousarray(vs[b, hk])
        oo = np.zeros((n, D), dtype=np.uint16)
        of = np.zeros((n, D), dtype=np.float64) if want_f64 else None
        ff = np.zeros((n, D), dtype=np.float64) if want_flip else None
        lib().or_attn_head(_p(a_q8, _i8p), _p(a_qs, _f32p), _p(a_k8, _i8p), _p(a_ks, _f32p),
                           _p(a_v8, _u8p), a_v8.shape[1], _p(a_vs, _f32p), Lq, Lk, D, blk_q,
                           blk_k, float(softmax_scale), int(bool(causal)), int(bool(quantize_p)),
                           _p(rows, _i32p), n, _p(oo, _u16p),
                           _p(of, _f64p) if want_f64 else None,
                           _p(ff, _f64p) if want_flip else None)
        out[b, h] = oo
        if want_f64:
            o64[b, h] = of
        if want_flip:
            flip[b, h] = ff

    _pool_map(one, [(b, h) for b in range(B) for h in range(H)], threads)
    if want_flip:
        return out, o64, flip
    return (out, o64) if want_f64 else out


def attn_exact(q, k, v, softmax_scale, causal, rows=None, threads=None):
    """fp64 softmax(q k^T * scale) v of the unquantised bf16 inputs."""
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    group = H // Hk
    if rows is None:
        rows = np.arange(Lq, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    n = rows.size
    out = np.zeros((B, H, n, D), dtype=np.float64)

    def one(bh):
        b, h = bh
        qq = np.ascontiguousarray(q[b, h])
        kk = np.ascontiguousarray(k[b, h // group])
        vv = np.ascontiguousarray(v[b, h // group])
        oo = np.zeros((n, D), dtype=np.float64)
        lib().or_attn_exact_head(_p(qq, _u16p), _p(kk, _u16p), _p(vv, _u16p), Lq, Lk, D,
                                 float(softmax_scale), int(bool(causal)), _p(rows, _i32p), n,
                                 _p(oo, _f64p))
        out[b, h] = oo

    _pool_map(one, [(b, h) for b in range(B) for h in range(H)], threads)
    return out


def sage_attention(q, k, v, blk_q, blk_k, softmax_scale, causal, rows=None, threads=None):
    """The whole path: quantise Q/K/V, then quantised attention."""
    qk = quant_qk(q, k, blk_q, blk_k, threads)
    v8t, vs = quant_v(v, threads)
    out = attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, q.shape[2], k.shape[2], blk_q,
               blk_k, softmax_scale, causal, rows=rows, threads=threads)
    return out, qk, v8t, vs


# ---------------------------------------------------------------- decode

KV_PER_TENSOR = 1       # ksc / vsc hold one scale each
KV_V_TRANSPOSED = 2     # vc is [num_pages, Hk, D, page]


def decode(q, kc, vc, ksc, vsc, ptab, ctx, window, softmax_scale, threads=None, want_f64=False,
           kv_flags=0, want_flip=False):
    """Paged FP8 decode. q: uint16 [B, T, H, D]; kc: uint8 [num_pages, Hk,
    page, D]; vc: the same, or [num_pages, Hk, D, page] with KV_V_TRANSPOSED;
    ksc, vsc: float32 [num_pages, Hk, page], or one value each with
    KV_PER_TENSOR; ptab: int32 [B, max_pages]; ctx: int32 [B]. Returns bf16
    bits [B, T, H, D] (and the fp64 values, and with want_flip the margin of
    the PV weights an fp32 evaluation may round to the neighbouring bf16)."""
    B, T, H, D = q.shape
    Hk, page = kc.shape[1], kc.shape[2]
    want_f64 = want_f64 or want_flip
    kc = np.ascontiguousarray(kc)
    vc = np.ascontiguousarray(vc)
    ksc = np.ascontiguousarray(ksc, dtype=np.float32)
    vsc = np.ascontiguousarray(vsc, dtype=np.float32)
    out = np.zeros((B, T, H, D), dtype=np.uint16)
    o64 = np.zeros((B, T, H, D), dtype=np.float64) if want_f64 else None
    flip = np.zeros((B, T, H, D), dtype=np.float64) if want_flip else None

    def one(b):
        qq = np.ascontiguousarray(q[b])
        pt = np.ascontiguousarray(ptab[b], dtype=np.int32)
        oo = np.zeros((T, H, D), dtype=np.uint16)
        of = np.zeros((T, H, D), dtype=np.float64) if want_f64 else None
        ff = np.zeros((T, H, D), dtype=np.float64) if want_flip else None
        lib().or_decode_seq_flags(_p(qq, _u16p), _p(kc, _u8p), _p(vc, _u8p), _p(ksc, _f32p),
                                  _p(vsc, _f32p), _p(pt, _i32p), int(ctx[b]), T, H, Hk, D, page,
                                  int(window), float(softmax_scale), int(kv_flags), _p(oo, _u16p),
                                  _p(of, _f64p) if want_f64 else None,
                                  _p(ff, _f64p) if want_flip else None)
        out[b] = oo
        if want_f64:
            o64[b] = of
        if want_flip:
            flip[b] = ff

    _pool_map(one, list(range(B)), threads)
    if want_flip:
        return out, o64, flip
    return (out, o64) if want_f64 else out


def decode_mxfp4(q, kc, vc, ksf, vsf, ptab, ctx, window, softmax_scale, threads=None, want_f64=False,
                 want_flip=False):
    """Paged decode over an MXFP4 cache. q: uint16 [B, T, H, D]; kc, vc:
    uint8 [num_pages, Hk, page, D / 2] packed E2M1 (element 2i in the low
    nibble of byte i); ksf, vsf: uint8 e8m0 [num_pages, Hk, page, D / 32];
    ptab: int32 [B, max_pages]; ctx: int32 [B]. Returns bf16 bits (and the
    fp64 values, and with want_flip the bf16-weight margin) like decode()."""
    B, T, H, D = q.shape
    Hk, page = kc.shape[1], kc.shape[2]
    want_f64 = want_f64 or want_flip
    kc, vc = np.ascontiguousarray(kc, dtype=np.uint8), np.ascontiguousarray(vc, dtype=np.uint8)
    ksf, vsf = np.ascontiguousarray(ksf, dtype=np.uint8), np.ascontiguousarray(vsf, dtype=np.uint8)
    out = np.zeros((B, T, H, D), dtype=np.uint16)
    o64 = np.zeros((B, T, H, D), dtype=np.float64) if want_f64 else None
    flip = np.zeros((B, T, H, D), dtype=np.float64) if want_flip else None

    def one(b):
        qq = np.ascontiguousarray(q[b])
        pt = np.ascontiguousarray(ptab[b], dtype=np.int32)
        oo = np.zeros((T, H, D), dtype=np.uint16)
        of = np.zeros((T, H, D), dtype=np.float64) if want_f64 else None
        ff = np.zeros((T, H, D), dtype=np.float64) if want_flip else None
        lib().or_decode_seq_mxkv(_p(qq, _u16p), _p(kc, _u8p), _p(vc, _u8p), _p(ksf, _u8p), _p(vsf, _u8p),
                                 _p(pt, _i32p), int(ctx[b]), T, H, Hk, D, page, int(window),
                                 float(softmax_scale), _p(oo, _u16p), _p(of, _f64p) if want_f64 else None,
                                 _p(ff, _f64p) if want_flip else None)
        out[b] = oo
        if want_f64:
            o64[b] = of
        if want_flip:
            flip[b] = ff

    _pool_map(one, list(range(B)), threads)
    if want_flip:
        return out, o64, flip
    return (out, o64) if want_f64 else out


def decode_quant_q(q):
    """The decode's query quantisation: every (b, t, h) row rotated and cast
    to e4m3 with scale max|q_hat| / 448. q: uint16 [B, T, H, D] ->
    (codes uint8 [B, T, H, D], scales float32 [B, T, H])."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    B, T, H, D = q.shape
    rows = q.reshape(-1, D)
    codes = np.zeros(rows.shape, dtype=np.uint8)
    scales = np.zeros((rows.shape[0],), dtype=np.float32)
    f = lib().or_decode_quant_q_row
    for i in range(rows.shape[0]):
        f(_p(rows[i], _u16p), D, _p(codes[i], _u8p), _p(scales[i:i + 1], _f32p))
    return codes.reshape(B, T, H, D), scales.reshape(B, T, H)


# ---------------------------------------------------------------- MXFP4 variant

def e2m1_decode(codes):
    L = lib()
    table = np.array([L.or_e2m1_decode(c) for c in range(16)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8) & 15]


def e2m1_encode(x):
    x = np.asarray(x, dtype=np.float64)
    f = lib().or_e2m1_encode
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


def _quant_mxfp4(x, mean, threads):
    B, H, L, D = x.shape
    Lpad = round_up(L, 128)
    codes = np.zeros((B, H, Lpad, D // 2), dtype=np.uint8)
    sf = np.zeros((B, H, Lpad, D // 32), dtype=np.uint8)

    def one(bh):
        b, h = bh
        xx = np.ascontiguousarray(x[b, h])
        mp = None
        if mean is not None:
            mm = np.ascontiguousarray(mean[b, h], dtype=np.float32)
            mp = _p(mm, _f32p)
        cc = np.zeros((Lpad, D // 2), dtype=np.uint8)
        ss = np.zeros((Lpad, D // 32), dtype=np.uint8)
        lib().or_quant_mxfp4_head(_p(xx, _u16p), mp, L, D, Lpad, _p(cc, _u8p), _p(ss, _u8p))
        codes[b, h] = cc
        sf[b, h] = ss

    _pool_map(one, [(b, h) for b in range(B) for h in range(H)], threads)
    return codes, sf


def quant_qk_mxfp4(q, k, threads=None):
    """Smooth K, rotate Q and K, quantise both to MXFP4 (E2M1 codes, one e8m0
    scale per 32 elements of a row). q: uint16 [B, H, Lq, D]; k: uint16
    [B, Hk, Lk, D]. Codes [B, H, Lpad, D/2] (element 2i in the low nibble),
    scales [B, H, Lpad, D/32] in plain row-major order."""
    kmean = k_mean(k)
    q4, qsf = _quant_mxfp4(q, None, threads)
    k4, ksf = _quant_mxfp4(k, kmean, threads)
    return {"q4": q4, "qsf": qsf, "k4": k4, "ksf": ksf, "kmean": kmean}


def attn_mxfp4(q4, qsf, k4, ksf, v8t, vs, Lq, Lk, softmax_scale, causal, rows=None,
               quantize_p=True, threads=None, want_f64=False, want_flip=False):
    """Quantised attention with MXFP4 Q / K and FP8 P / V. Returns bf16 bits
    [B, H, nrows, D] (and the fp64 values, and the P-rounding margin)."""
    B, H, _, D2 = q4.shape
    D = 2 * D2
    Hk = k4.shape[1]
    group = H // Hk
    want_f64 = want_f64 or want_flip
    if rows is None:
        rows = np.arange(Lq, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    n = rows.size
    out = np.zeros((B, H, n, D), dtype=np.uint16)
    o64 = np.zeros((B, H, n, D), dtype=np.float64) if want_f64 else None
    flip = np.zeros((B, H, n, D), dtype=np.float64) if want_flip else None

    def one(bh):
        b, h = bh
        hk = h // group
        a = [np.ascontiguousarray(t) for t in (q4[b, h], qsf[b, h], k4[b, hk], ksf[b, hk])]
        a_v8 = np.ascontiguousarray(v8t[b, hk])
        a_vs = np.ascontiguousarray(vs[b, hk])
        oo = np.zeros((n, D), dtype=np.uint16)
        of = np.zeros((n, D), dtype=np.float64) if want_f64 else None
        ff = np.zeros((n, D), dtype=np.float64) if want_flip else None
        lib().or_attn_mxfp4_head(_p(a[0], _u8p), _p(a[1], _u8p), _p(a[2], _u8p), _p(a[3], _u8p),
                                 _p(a_v8, _u8p), a_v8.shape[1], _p(a_vs, _f32p), Lq, Lk, D,
                                 float(softmax_scale), int(bool(causal)), int(bool(quantize_p)),
                                 _p(rows, _i32p), n, _p(oo, _u16p),
                                 _p(of, _f64p) if want_f64 else None,
                                 _p(ff, _f64p) if want_flip else None)
        out[b, h] = oo
        if want_f64:
            o64[b, h] = of
        if want_flip:
            flip[b, h] = ff

    _pool_map(one, [(b, h) for b in range(B) for h in range(H)], threads)
    if want_flip:
        return out, o64, flip
    return (out, o64) if want_f64 else out

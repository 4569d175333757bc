"""Shared helpers of the GPU parity tests: run the CUDA path through the
C-ABI binding on seeded inputs, run the oracle on the same inputs, compare.

Tolerance of the bf16 attention output: the GPU's fp32 result may differ
from the oracle's fp64 value y by at most 2e-3 before its final bf16
rounding, so element-wise |gpu - y| <= 2e-3 + ulp_bf16(y)/2, plus, where the
oracle reports one, the margin of the P codes that an fp32 evaluation of
448 p may round the other way (the scores are fp32 before the FP8 cast, and
a code whose exact value lies within fp32 error of an e4m3 rounding midpoint
can land on either side; the oracle gives the effect of moving each such
code by one step) -- for the decode, the bound on the bf16 PV weights
p * v_scale, which a kernel with running maxima rounds at other scales than
the oracle's window maximum. The cosine against the oracle must be >= 0.9999 and
against unquantised fp64 attention >= 0.998. Every comparison reports how
many elements needed the margin.
"""
import math

import numpy as np
import torch

import oracle
import quantized_attention_smoothing_b200 as sage
import workloads

MAX_ABS = 2e-3
COS_ORACLE = 0.9999
COS_EXACT = 0.998


def bits(t):
    return workloads.bits_u16(t.cpu() if t.is_cuda else t)


def to_gpu(t):
    """Copy to the GPU keeping the strides (views stay views)."""
    return t.to("cuda")


def gpu_quant(h, q, k, v, blk_q, blk_k, fused=False):
    """sage_quant_qk + sage_quant_v, or (fused) sage_quant_qkv."""
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    bufs = sage.QuantBuffers(B, H, Hk, Lq, Lk, D, blk_q, blk_k)
    if fused:
        sage.sage_quant_qkv(h, q, k, v, blk_q, blk_k, bufs.q8, bufs.q_scale, bufs.k8, bufs.k_scale,
                            bufs.v8_t, bufs.v_scale, bufs.k_mean, bufs.ws)
    else:
        sage.sage_quant_qk(h, q, k, blk_q, blk_k, bufs.q8, bufs.q_scale, bufs.k8, bufs.k_scale,
                           bufs.k_mean, bufs.ws)
        sage.sage_quant_v(v, bufs.v8_t, bufs.v_scale, bufs.ws_v)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    return bufs


def assert_quant_bitexact(bufs, ref_qk, ref_v8t, ref_vs, Lq, Lk):
    got = {
        "q8": bufs.q8.cpu().numpy(), "qs": bufs.q_scale.cpu().numpy(),
        "k8": bufs.k8.cpu().numpy(), "ks": bufs.k_scale.cpu().numpy(),
        "kmean": bufs.k_mean.cpu().numpy(),
    }
    for name in ("q8", "k8"):
        a, b = got[name], ref_qk[name]
        assert a.shape == b.shape, name
        bad = np.argwhere(a != b)
        assert bad.size == 0, "%s differs at %d places, first %s: gpu %d oracle %d" % (
            name, len(bad), tuple(bad[0]), a[tuple(bad[0])], b[tuple(bad[0])])
    for name in ("qs", "ks", "kmean"):
        a, b = got[name], ref_qk[name]
        assert a.shape == b.shape, name
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), name
    v8t = bufs.v8_t.cpu().numpy()
    vs = bufs.v_scale.cpu().numpy()
    assert v8t.shape == ref_v8t.shape
    bad = np.argwhere(v8t != ref_v8t)
    assert bad.size == 0, "v8t differs at %d places, first %s" % (len(bad), tuple(bad[0]))
    assert np.array_equal(vs.view(np.uint32), ref_vs.view(np.uint32))


def bf16_ulp(x):
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 2.0 ** -126)))
    e = np.maximum(e, -126)
    return 2.0 ** (e - 7)


def compare_output(gpu_bf16_bits, oracle_f64, exact_f64=None, label="", margin=None):
    g = workloads_f32(gpu_bf16_bits).astype(np.float64)
    y = oracle_f64
    if isinstance(y, tuple):                 # (oracle value, P-rounding margin)
        y, margin = y
    ulp = bf16_ulp(np.maximum(np.abs(g), np.abs(y)))
    plain = np.abs(g - y) - ulp / 2
    excess = plain if margin is None else plain - margin
    worst = float(excess.max())
    cos = cosine(g, y)
    stats = {"max_excess": worst, "max_abs": float(np.abs(g - y).max()), "cos_oracle": cos,
             "beyond_plain_bar": int((plain > MAX_ABS).sum()), "elements": int(plain.size)}
    if stats["beyond_plain_bar"]:
        print("%s: %d of %d elements beyond 2e-3 + ulp/2 (largest %.3g)%s"
              % (label, stats["beyond_plain_bar"], plain.size, float(plain.max()),
                 "" if margin is None else "; the oracle's rounding margin covers %s"
                 % ("each" if worst <= MAX_ABS else "not all")))
    assert worst <= MAX_ABS, "%s: |gpu - oracle| exceeds 2e-3 + ulp/2 (+ margin) by %g" % (label, worst)
    assert cos >= COS_ORACLE, "%s: cosine vs oracle %.6f" % (label, cos)
    if exact_f64 is not None:
        ce = cosine(g, exact_f64)
        stats["cos_exact"] = ce
        assert ce >= COS_EXACT, "%s: cosine vs exact %.6f" % (label, ce)
    return stats


def workloads_f32(u16):
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def cosine(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb))


def sample_rows(L, n, seed=0):
    """Rows spread over the sequence, always including tile edges and the tail."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 127, 128, 255, 256, L - 129, L - 128, L - 2, L - 1}
    rows = set(r for r in fixed if 0 <= r < L)
    rows.update(rng.choice(L, size=min(n, L), replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int32)

"""Pins of the oracle's MXFP4 variant (MXFP4 Q and K, FP8 P and V):

* the E2M1 codec against the format's definition (1 sign, 2 exponent bits
  with bias 1, 1 mantissa bit, a subnormal step of 0.5), by brute force over
  the grid it defines: every code, every rounding midpoint (ties to the even
  code), saturation at 6 and the sign of zero;
* the block quantisation: every block's scale 2^E puts the block maximum in
  [4, 8), every code is the nearest grid value of x * 2^-E (independent brute
  force over the rotation computed with scipy's Hadamard matrix), and the
  round trip is within half a grid step (or the saturation error);
* the attention: with the e4m3 rounding of P switched off it equals fp64
  softmax over the dequantised operands (numpy), and the method stays close
  to unquantised attention on a small video-DiT-like workload.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import workloads


def _grid():
    """E2M1 from its definition: (-1)^s * 2^(e-1) * (1 + m/2) for e > 0,
    (-1)^s * 0.5 * m for e = 0; code = s << 3 | e << 1 | m."""
    vals = {}
    for s in (0, 1):
        for e in range(4):
            for m in range(2):
                mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
                vals[(s << 3) | (e << 1) | m] = -mag if s else mag
    return vals


def _nearest_code(x):
    """Brute force: the non-negative code nearest |x| (ties to the even
    code), |x| >= 6 saturating, with x's sign."""
    g = _grid()
    ax = min(abs(x), 6.0)
    best = min(range(8), key=lambda c: (abs(g[c] - ax), c & 1))
    return best | (8 if math.copysign(1.0, x) < 0 else 0)


def test_e2m1_decode_every_code(oracle_mod):
    g = _grid()
    for c in range(16):
        assert oracle_mod.lib().or_e2m1_decode(c) == g[c]
        assert math.copysign(1.0, oracle_mod.lib().or_e2m1_decode(c)) == math.copysign(1.0, g[c])


def test_e2m1_encode_midpoints_saturation_and_sign(oracle_mod):
    L = oracle_mod.lib()
    mags = sorted(set(abs(v) for v in _grid().values()))
    probes = list(mags)
    for a, b in zip(mags, mags[1:]):
        mid = 0.5 * (a + b)
        probes += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, 10.0)]
    probes += [6.0, 6.5, 7.999, 1e30, 1e-30, 0.0]
    rng = np.random.default_rng(3)
    probes += list(rng.uniform(0, 7, 2000))
    for v in probes:
        for x in (v, -v):
            assert L.or_e2m1_encode(x) == _nearest_code(x), x
    assert L.or_e2m1_encode(-0.0) == 8 and L.or_e2m1_encode(0.0) == 0


def test_block_quantisation_against_brute_force(oracle_mod):
    g = torch.Generator().manual_seed(12)
    D, L = 128, 70
    x = (torch.randn((1, 2, L, D), generator=g) * 3).to(torch.bfloat16)
    x[0, 1, 5] = 0.0                          # an all-zero row: scale 2^-127, zero codes
    x[0, 1, 6, :32] = 1e-6                    # tiny values in one block
    codes, sf = oracle_mod._quant_mxfp4(workloads.bits_u16(x), None, None)
    Hm = scipy.linalg.hadamard(D).astype(np.float64)
    xf = x.float().numpy()
    for h in range(2):
        for l in range(L):
            rot = oracle_mod.fwht_f32(xf[0, h, l][None, :])[0]
            assert np.abs(rot - xf[0, h, l] @ Hm).max() <= 1e-4 * max(1e-30, np.abs(xf[0, h, l]).sum())
            for b in range(D // 32):
                blk = rot[32 * b:32 * b + 32].astype(np.float64)
                E = int(sf[0, h, l, b]) - 127
                a = np.abs(blk).max()
                if a == 0:
                    assert E == -127
                else:
                    assert 4.0 <= a * 2.0 ** -E < 8.0 or E == -127
                for e in range(32):
                    d = 32 * b + e
                    byte = codes[0, h, l, d // 2]
                    c = (byte >> 4) if d & 1 else (byte & 15)
                    if a == 0:
                        assert c == 0
                        continue
                    assert c == _nearest_code(blk[e] * 2.0 ** -E), (h, l, d)
                    y = _grid()[c] * 2.0 ** E
                    sc = abs(blk[e]) * 2.0 ** -E
                    half_step = 0.25 if sc < 2 else (0.5 if sc < 4 else 1.0)
                    bound = half_step if sc <= 6 else sc - 6.0
                    assert abs(y - blk[e]) <= bound * 2.0 ** E * (1 + 1e-12)
    assert (codes[:, :, L:] == 0).all() and (sf[:, :, L:] == 0).all()


def _dequant(oracle_mod, codes, sf):
    lo = oracle_mod.e2m1_decode(codes & 15)
    hi = oracle_mod.e2m1_decode(codes >> 4)
    vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (2 * codes.shape[-1],))
    scale = np.repeat(2.0 ** (sf.astype(np.float64) - 127), 32, axis=-1)
    return vals * scale


@pytest.mark.parametrize("Lq,Lk,causal,H,Hk", [
    (200, 330, False, 2, 2),
    (300, 300, True, 2, 1),
    (150, 90, True, 1, 1),
])
def test_mxfp4_attention_without_p_rounding_equals_exact_softmax(oracle_mod, Lq, Lk, causal, H, Hk):
    D = 128
    g = torch.Generator().manual_seed(Lq + Lk)
    q = (torch.randn((1, H, Lq, D), generator=g) * 2).to(torch.bfloat16)
    k = (torch.randn((1, Hk, Lk, D), generator=g) + 1).to(torch.bfloat16)
    v = torch.randn((1, Hk, Lk, D), generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    b = workloads.bits_u16
    qk = oracle_mod.quant_qk_mxfp4(b(q), b(k))
    v8t, vs = oracle_mod.quant_v(b(v))
    _, got = oracle_mod.attn_mxfp4(qk["q4"], qk["qsf"], qk["k4"], qk["ksf"], v8t, vs, Lq, Lk, scale,
                                   causal, quantize_p=False, want_f64=True)
    qd = _dequant(oracle_mod, qk["q4"], qk["qsf"])
    kd = _dequant(oracle_mod, qk["k4"], qk["ksf"])
    for h in range(H):
        hk = h // (H // Hk)
        s = qd[0, h, :Lq] @ kd[0, hk, :Lk].T * (scale / D)
        if causal:
            vis = np.arange(Lk)[None, :] <= np.arange(Lq)[:, None] + (Lk - Lq)
            s = np.where(vis, s, -np.inf)
        vdq = oracle_mod.e4m3_decode(v8t[0, hk, :, :Lk]).T * vs[0, hk][None, :].astype(np.float64)
        ref = np.zeros((Lq, D))
        for i in range(Lq):
            if np.isfinite(s[i]).any():
                w = np.exp(s[i] - s[i].max())
                ref[i] = (w / w.sum()) @ vdq
        assert np.abs(got[0, h] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_mxfp4_method_stays_close_to_exact_attention(oracle_mod):
    """The MXFP4 variant against unquantised fp64 attention with a large
    per-channel K bias (N(0, 16)): with the K smoothing and the rotation the
    FP4 Q / K keep the output within cosine 0.98 of exact attention; without
    the smoothing the bias dominates every block's scale and it drops below
    0.95. (FP4 keeps less than INT8: the INT8 path stays above 0.999 here.)"""
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=512, D=128, seed=33, kbias_std=4.0)
    scale = 1.0 / math.sqrt(128)
    b = workloads.bits_u16
    rows = np.arange(0, 512, 5, dtype=np.int32)
    qk = oracle_mod.quant_qk_mxfp4(b(q), b(k))
    v8t, vs = oracle_mod.quant_v(b(v))
    exact = oracle_mod.attn_exact(b(q), b(k), b(v), scale, False, rows=rows).ravel()

    def cosine(bits):
        g = oracle_mod.bf16_to_f32(bits).astype(np.float64).ravel()
        return float(g @ exact / (np.linalg.norm(g) * np.linalg.norm(exact)))

    good = cosine(oracle_mod.attn_mxfp4(qk["q4"], qk["qsf"], qk["k4"], qk["ksf"], v8t, vs, 512, 512,
                                        scale, False, rows=rows))
    k4n, ksfn = oracle_mod._quant_mxfp4(b(k), None, None)
    bad = cosine(oracle_mod.attn_mxfp4(qk["q4"], qk["qsf"], k4n, ksfn, v8t, vs, 512, 512, scale, False,
                                       rows=rows))
    assert good >= 0.98 and bad < 0.95, (good, bad)

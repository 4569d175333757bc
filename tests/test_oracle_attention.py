"""Pins of the oracle's quantised attention.

* With the e4m3 rounding of P switched off, the tiled online softmax (the
  QK -> update_mdo -> accumulate_d -> RS_32_to_8 -> PV sequence of "Sage2
  SM89 Temporal Pair Experiment", Candidate) must equal plain fp64 softmax
  over the dequantised operands, for many tiles, ragged tails, causal masks
  and GQA.
* With one key tile the running max is the row max, so P8 has a closed form;
  it is checked with torch's own float8 conversion.
* Special cases: L = 1 (softmax = 1), identical keys (mean of V rows), rows
  with no visible key.
* The whole method stays within the accuracy gate against unquantised fp64
  attention (cosine >= 0.998) on the small workloads, and a planted mistake
  (dropping K smoothing) is caught by that gate on an outlier workload.
"""
import math

import numpy as np
import pytest
import torch

import workloads


def _bits(t):
    return workloads.bits_u16(t)


def _dequant_reference(oracle_mod, qk, v8t, vs, Lq, Lk, blk_q, blk_k, scale, causal, D, H, Hk):
    """fp64 softmax(Sq Sk^T * scale / D) (V8 * vs) from the quantised operands."""
    B = qk["q8"].shape[0]
    out = np.zeros((B, H, Lq, D))
    for b in range(B):
        for h in range(H):
            hk = h // (H // Hk)
            qd = qk["q8"][b, h, :Lq].astype(np.float64) * np.repeat(qk["qs"][b, h], blk_q)[:Lq, None]
            kd = qk["k8"][b, hk, :Lk].astype(np.float64) * np.repeat(qk["ks"][b, hk], blk_k)[:Lk, None]
            vd = oracle_mod.e4m3_decode(v8t[b, hk, :, :Lk]).T * vs[b, hk][None, :].astype(np.float64)
            s = (qd @ kd.T) * (scale / D)
            if causal:
                i = np.arange(Lq)[:, None]
                j = np.arange(Lk)[None, :]
                s = np.where(j <= i + (Lk - Lq), s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            ok = np.isfinite(mx)
            e = np.where(ok, np.exp(s - np.where(ok, mx, 0)), 0.0)
            den = e.sum(axis=1, keepdims=True)
            out[b, h] = np.where(den > 0, (e @ vd) / np.where(den > 0, den, 1), 0.0)
    return out


@pytest.mark.parametrize("Lq,Lk,causal,H,Hk,D,blk_q,blk_k", [
    (256, 256, False, 2, 2, 64, 64, 64),
    (300, 555, False, 2, 1, 64, 128, 64),
    (383, 383, True, 2, 2, 128, 128, 64),
    (129, 400, True, 4, 2, 64, 64, 128),
    (500, 130, True, 1, 1, 64, 64, 64),      # Lq > Lk: leading rows see no key
])
def test_online_softmax_equals_exact_without_p_rounding(oracle_mod, Lq, Lk, causal, H, Hk, D,
                                                         blk_q, blk_k):
    g = torch.Generator().manual_seed(Lq * 7 + Lk)
    q = (torch.randn((1, H, Lq, D), generator=g) * 2).to(torch.bfloat16)
    k = (torch.randn((1, Hk, Lk, D), generator=g) * 2 + 1).to(torch.bfloat16)
    v = torch.randn((1, Hk, Lk, D), generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    qk = oracle_mod.quant_qk(_bits(q), _bits(k), blk_q, blk_k)
    v8t, vs = oracle_mod.quant_v(_bits(v))
    _, got = oracle_mod.attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, Lq, Lk, blk_q, blk_k,
                             scale, causal, quantize_p=False, want_f64=True)
    ref = _dequant_reference(oracle_mod, qk, v8t, vs, Lq, Lk, blk_q, blk_k, scale, causal, D, H, Hk)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    if causal and Lq > Lk:
        assert (got[:, :, :Lq - Lk] == 0).all()


def test_single_tile_p8_closed_form(oracle_mod):
    """Lk <= 128: P8 = e4m3(448 * exp(x - rowmax)), d = sum exp(x - rowmax)."""
    Lq, Lk, D, H = 64, 100, 64, 2
    g = torch.Generator().manual_seed(99)
    q = torch.randn((1, H, Lq, D), generator=g).to(torch.bfloat16)
    k = (torch.randn((1, H, Lk, D), generator=g) + 2).to(torch.bfloat16)
    v = torch.randn((1, H, Lk, D), generator=g).to(torch.bfloat16)
    scale = 0.125
    qk = oracle_mod.quant_qk(_bits(q), _bits(k), 64, 64)
    v8t, vs = oracle_mod.quant_v(_bits(v))
    _, got = oracle_mod.attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, Lq, Lk, 64, 64,
                             scale, False, want_f64=True)
    for h in range(H):
        acc = qk["q8"][0, h, :Lq].astype(np.int64) @ qk["k8"][0, h, :Lk].astype(np.int64).T
        x = acc * qk["qs"][0, h, 0].astype(np.float64) * np.repeat(qk["ks"][0, h], 64)[None, :Lk] \
            * (scale / D)
        p = np.exp(x - x.max(axis=1, keepdims=True))
        p8 = torch.from_numpy(p * 448.0).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        vdec = oracle_mod.e4m3_decode(v8t[0, h, :, :Lk]).T
        ref = (p8 @ vdec) * vs[0, h][None, :] / (448.0 * p.sum(axis=1, keepdims=True))
        assert np.abs(got[0, h] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_length_one_returns_dequantised_v(oracle_mod):
    D = 64
    g = torch.Generator().manual_seed(1)
    q = torch.randn((1, 1, 1, D), generator=g).to(torch.bfloat16)
    k = torch.randn((1, 1, 1, D), generator=g).to(torch.bfloat16)
    v = torch.randn((1, 1, 1, D), generator=g).to(torch.bfloat16)
    out, _, v8t, vs = oracle_mod.sage_attention(_bits(q), _bits(k), _bits(v), 64, 64, 0.125, False)
    ref = oracle_mod.e4m3_decode(v8t[0, 0, :, 0]) * vs[0, 0].astype(np.float64)
    assert np.array_equal(out[0, 0, 0], oracle_mod.f64_to_bf16(ref))
    # and the dequantised V row is the V row itself within e4m3 precision
    vf = oracle_mod.bf16_to_f32(_bits(v))[0, 0, 0]
    assert np.abs(ref - vf).max() <= 2.0 ** -4 * np.abs(vf).max()


def test_identical_keys_give_mean_of_v(oracle_mod):
    L, D = 300, 64
    g = torch.Generator().manual_seed(2)
    q = torch.randn((1, 1, L, D), generator=g).to(torch.bfloat16)
    k = torch.randn((1, 1, 1, D), generator=g).expand(1, 1, L, D).to(torch.bfloat16).contiguous()
    v = torch.randn((1, 1, L, D), generator=g).to(torch.bfloat16)
    out, _, v8t, vs = oracle_mod.sage_attention(_bits(q), _bits(k), _bits(v), 64, 64, 0.125, False)
    vdec = oracle_mod.e4m3_decode(v8t[0, 0, :, :L]) * vs[0, 0][:, None].astype(np.float64)
    ref = oracle_mod.f64_to_bf16(vdec.mean(axis=1))
    # smoothed identical keys are all zero -> every logit is 0 -> p = 1
    for i in range(L):
        assert np.array_equal(out[0, 0, i], ref)


def _cosine(a, b):
    a = a.ravel().astype(np.float64)
    b = b.ravel().astype(np.float64)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def test_method_accuracy_gate_c1(oracle_mod):
    cfg, q, k, v = workloads.make_prefill_config("c1")
    out, _, _, _ = oracle_mod.sage_attention(_bits(q), _bits(k), _bits(v), cfg["blk_q"],
                                             cfg["blk_k"], cfg["softmax_scale"], cfg["causal"])
    exact = oracle_mod.attn_exact(_bits(q), _bits(k), _bits(v), cfg["softmax_scale"], cfg["causal"])
    assert _cosine(oracle_mod.bf16_to_f32(out), exact) >= 0.998


def test_method_accuracy_gate_outliers_and_planted_mistake(oracle_mod):
    """A C2-like workload (outlier K channels, large K bias) on fewer tokens:
    the method passes the gate; without K smoothing it does not."""
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=512, D=128, seed=21, kbias_std=30.0,
                                     outlier_channels=4, outlier_mult=20.0)
    scale = 1.0 / math.sqrt(128)
    rows = np.arange(0, 512, 7, dtype=np.int32)
    out, qk, v8t, vs = oracle_mod.sage_attention(_bits(q), _bits(k), _bits(v), 128, 64, scale,
                                                 False, rows=rows)
    exact = oracle_mod.attn_exact(_bits(q), _bits(k), _bits(v), scale, False, rows=rows)
    good = _cosine(oracle_mod.bf16_to_f32(out), exact)
    assert good >= 0.998
    # planted mistake: quantise K without subtracting its mean
    k8n, ksn = oracle_mod._quant_i8(_bits(k), None, 64, None)
    bad_out = oracle_mod.attn(qk["q8"], qk["qs"], k8n, ksn, v8t, vs, 512, 512, 128, 64, scale,
                              False, rows=rows)
    bad = _cosine(oracle_mod.bf16_to_f32(bad_out), exact)
    assert bad < good and bad < 0.998


def _numpy_softmax_attention(q, k, v, scale, causal, rows):
    """Plain fp64 softmax(q k^T * scale) v with numpy, written independently
    of the oracle: the reference every accuracy gate is taken against. The
    causal mask is the bottom-right aligned one (key j visible to query i iff
    j <= i + Lk - Lq); a row that sees no key is zero."""
    B, H, Lq, D = q.shape
    Hk, Lk = k.shape[1], k.shape[2]
    qf = q.astype(np.float64)
    kf = k.astype(np.float64)
    vf = v.astype(np.float64)
    out = np.zeros((B, H, len(rows), D))
    for b in range(B):
        for h in range(H):
            hk = h // (H // Hk)
            s = qf[b, h, rows] @ kf[b, hk].T * scale          # [n, Lk]
            if causal:
                vis = np.arange(Lk)[None, :] <= rows[:, None] + (Lk - Lq)
                s = np.where(vis, s, -np.inf)
            for n in range(len(rows)):
                if not np.isfinite(s[n]).any():
                    continue
                w = np.exp(s[n] - s[n].max())
                out[b, h, n] = (w / w.sum()) @ vf[b, hk]
    return out


@pytest.mark.parametrize("B,H,Hk,Lq,Lk,D,causal,rows", [
    (1, 2, 2, 37, 37, 64, False, None),          # non-causal
    (1, 2, 2, 45, 45, 64, True, None),           # causal, Lq == Lk
    (2, 2, 1, 19, 60, 128, True, None),          # causal, Lq < Lk (bottom-right), GQA
    (1, 4, 2, 70, 23, 64, True, None),           # causal, Lq > Lk: leading rows see nothing
    (1, 6, 2, 50, 50, 64, False, None),          # GQA, group 3
    (1, 2, 2, 200, 180, 64, True, [0, 1, 19, 20, 21, 150, 199]),   # rows= subset
])
def test_exact_reference_equals_numpy_softmax(oracle_mod, B, H, Hk, Lq, Lk, D, causal, rows):
    """or_attn_exact_head (the unquantised fp64 reference behind every
    cosine >= 0.998 gate) against numpy: a wrong mask offset, a scale applied
    twice or a wrong GQA head map would each fail here."""
    g = torch.Generator().manual_seed(B * 1000 + Lq * 7 + Lk + H)
    q = (torch.randn((B, H, Lq, D), generator=g) * 1.5).to(torch.bfloat16)
    k = (torch.randn((B, Hk, Lk, D), generator=g) + 0.5).to(torch.bfloat16)
    v = torch.randn((B, Hk, Lk, D), generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    r = np.arange(Lq, dtype=np.int32) if rows is None else np.array(rows, dtype=np.int32)
    got = oracle_mod.attn_exact(_bits(q), _bits(k), _bits(v), scale, causal, rows=r)
    ref = _numpy_softmax_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                   scale, causal, r)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    if causal and Lq > Lk:
        n_dark = Lq - Lk
        assert (got[:, :, r < n_dark] == 0).all()


def _e4m3_round(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _fp32_p_attention(oracle_mod, qk, v8t, vs, h, L, D, blk, scale, rel_noise, rng):
    """The method's per-tile sequence written with numpy, independently of the
    oracle, with 448 p formed in fp32 the way a GPU kernel forms it (fp32
    logit scales, fp32 base-2 logits, fp32 exp2), then multiplied by
    (1 + u), |u| <= rel_noise, before the e4m3 cast; O and d in fp64."""
    q8 = qk["q8"][0, h, :L].astype(np.int64)
    k8 = qk["k8"][0, h, :L].astype(np.int64)
    acc = q8 @ k8.T
    qs = np.repeat(qk["qs"][0, h], blk)[:L]
    ks = np.repeat(qk["ks"][0, h], blk)[:L]
    vdec = oracle_mod.e4m3_decode(v8t[0, h, :, :L]).T
    arow = (qs.astype(np.float32) * np.float32(scale / D * math.log2(math.e))).astype(np.float32)
    kc = (ks[None, :].astype(np.float32) * arow[:, None]).astype(np.float32)
    y = (acc.astype(np.float32) * kc).astype(np.float32)
    m = np.full(L, -np.inf, dtype=np.float32)
    d = np.zeros(L)
    O = np.zeros((L, D))
    for t0 in range(0, L, 128):
        yt = y[:, t0:t0 + 128]
        mn = np.maximum(m, yt.max(1))
        alpha = np.where(np.isfinite(m), np.exp2((m - mn).astype(np.float32)).astype(np.float64), 0.0)
        p448 = np.exp2((yt + np.float32(math.log2(448.0)) - mn[:, None]).astype(np.float32))
        p448 = p448.astype(np.float64) * (1.0 + rel_noise * rng.uniform(-1.0, 1.0, p448.shape))
        O *= alpha[:, None]
        d = d * alpha + (p448 / 448.0).sum(1)
        O += _e4m3_round(p448) @ vdec[t0:t0 + 128]
        m = mn
    return O * vs[0, h][None, :].astype(np.float64) / (448.0 * d[:, None])


def test_p_rounding_margin_bounds_an_fp32_evaluation(oracle_mod):
    """The oracle's per-element margin for P codes that an fp32 evaluation
    may round the other way ("RS_32_to_8": scores are fp32 before the FP8
    cast). An independent numpy evaluation with fp32 logits and exponentials
    (plus noise of 1e-6 relative, inside the margin's error bound) lands
    within that margin of the oracle everywhere, though it moves elements by
    more than 1e-4 through flipped codes; with noise a hundred times larger
    the margin no longer holds (it is not vacuous)."""
    H, L, D, scale = 4, 1024, 64, 0.125
    g = torch.Generator().manual_seed(5)
    q = (torch.randn((1, H, L, D), generator=g) * 2).to(torch.bfloat16)
    k = (torch.randn((1, H, L, D), generator=g) * 2 + 1).to(torch.bfloat16)
    v = torch.randn((1, H, L, D), generator=g).to(torch.bfloat16)
    qk = oracle_mod.quant_qk(_bits(q), _bits(k), 64, 64)
    v8t, vs = oracle_mod.quant_v(_bits(v))
    _, y, margin = oracle_mod.attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, L, L, 64, 64,
                                   scale, False, want_flip=True)
    assert (margin >= 0).all() and (margin > 0).any()
    rng = np.random.default_rng(0)
    moved = 0
    for h in range(H):
        got = _fp32_p_attention(oracle_mod, qk, v8t, vs, h, L, D, 64, scale, 1e-6, rng)
        dev = np.abs(got - y[0, h])
        # 1e-5: the fp32 exponentials' own effect on d and on the codes that do not flip
        assert (dev <= margin[0, h] + 1e-5).all(), float((dev - margin[0, h]).max())
        moved += int((dev > 1e-4).sum())
    assert moved > 0                       # flipped codes did move elements
    worst = 0.0
    for h in range(H):
        got = _fp32_p_attention(oracle_mod, qk, v8t, vs, h, L, D, 64, scale, 1e-4, rng)
        worst = max(worst, float((np.abs(got - y[0, h]) - margin[0, h]).max()))
    assert worst > 1e-3


def test_e4m3_flip_step_at_the_midpoints(oracle_mod):
    """or_e4m3_flip_step: zero away from the rounding midpoints, the
    neighbouring code's distance at them, with the e4m3 grid checked against
    torch's float8 decode."""
    L = oracle_mod.lib()
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(1, 126):
        lo, here, hi = grid[c - 1], grid[c], grid[c + 1]
        mid_up = 0.5 * (here + hi)
        assert L.or_e4m3_flip_step(here, 1e-6) == 0.0
        assert L.or_e4m3_flip_step(mid_up * (1 - 1e-7), 1e-6) == hi - here
        assert L.or_e4m3_flip_step(mid_up * (1 + 1e-7), 1e-6) == hi - here
        assert L.or_e4m3_flip_step(0.5 * (lo + here) * (1 + 1e-7), 1e-6) == here - lo
    assert L.or_e4m3_flip_step(448.0, 1e-3) == 0.0                 # saturates: no code above
    assert L.or_e4m3_flip_step(2.0 ** -10 * (1 - 1e-7), 1e-6) == 2.0 ** -9

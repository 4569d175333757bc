"""Pins of the oracle's paged FP8 decode.

* The sliding-window convention (each of the MTP query tokens attends to the
  `window` keys ending at its own position) reproduces the window-tile counts
  the FlyDSL pa_decode page prints (tests/golden/window_tiles.txt).
* The oracle's paged, GQA, per-token-scaled decode equals a brute-force
  computation over the un-paged cache that uses torch's float8 conversion for
  the query quantisation, scipy's Hadamard matrix for the rotation and
  torch's bfloat16 conversion for the PV weights p_j * v_scale_j.
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_tiles():
    rows = []
    for line in open(os.path.join(GOLDEN, "window_tiles.txt")):
        if line.strip() and not line.startswith("#"):
            rows.append(tuple(int(x) for x in line.split()))
    return rows


def _attended_keys(ctx, T, window):
    """Union of the keys that the T last positions attend to (our reading)."""
    keys = set()
    for t in range(T):
        p = ctx - T + t
        keys.update(range(max(0, p - window + 1), p + 1))
    return keys


@pytest.mark.parametrize("window,mtp,tile,tiles", _golden_tiles())
def test_window_convention_reproduces_page_tile_counts(window, mtp, tile, tiles):
    assert (window + mtp - 2 + tile - 1) // tile + 1 == tiles
    worst = 0
    for ctx in range(window + mtp, window + mtp + 2 * tile):
        keys = _attended_keys(ctx, mtp, window)
        assert len(keys) == window + mtp - 1
        worst = max(worst, len({j // tile for j in keys}))
    assert worst == tiles


def _brute_decode(oracle_mod, d, window, scale):
    q = d["q"].float().numpy()                          # [B, T, H, D]
    B, T, H, D = q.shape
    Hk, page = d["k_cache"].shape[1], d["k_cache"].shape[2]
    Hmat = scipy.linalg.hadamard(D).astype(np.float64)
    kdec = oracle_mod.e4m3_decode(d["k_cache"].numpy())
    vdec = oracle_mod.e4m3_decode(d["v_cache"].numpy())
    out = np.zeros((B, T, H, D))
    for b in range(B):
        ctx = int(d["ctx_lens"][b])
        pages = d["page_table"][b].numpy()
        toks = np.arange(ctx)
        phys = pages[toks // page]
        slot = toks % page
        for h in range(H):
            hk = h // (H // Hk)
            K = kdec[phys, hk, slot]                    # [ctx, D]
            V = vdec[phys, hk, slot]
            ks = d["k_scale"].numpy()[phys, hk, slot].astype(np.float64)
            vs = d["v_scale"].numpy()[phys, hk, slot].astype(np.float64)
            for t in range(T):
                qh = oracle_mod.fwht_f32(q[b, t, h][None, :])[0]
                assert np.abs(qh - q[b, t, h] @ Hmat).max() <= 1e-4 * np.abs(q[b, t, h]).sum()
                a = np.abs(qh).max()
                s = np.float32(a) / np.float32(448.0)
                r = np.float32(448.0) / np.float32(a)
                q8 = torch.from_numpy((qh * r).astype(np.float32)).to(torch.float8_e4m3fn)
                q8 = q8.to(torch.float64).numpy()
                p = ctx - T + t
                lo = max(0, p - window + 1)
                sl = slice(lo, p + 1)
                logits = (K[sl] @ q8) * float(s) * ks[sl] * (scale / D)
                w = np.exp(logits - logits.max())
                # bf16 PV operand: fp32 product rounded by torch's bf16 cast
                wv = w.astype(np.float32) * vs[sl].astype(np.float32)
                wv = torch.from_numpy(wv).to(torch.bfloat16).to(torch.float64).numpy()
                out[b, t, h] = (wv @ V[sl]) / w.sum()
    return out


@pytest.mark.parametrize("B,T,H,Hk,D,page,lo,hi,window", [
    (3, 4, 8, 2, 64, 16, 40, 90, 32),
    (2, 1, 4, 1, 128, 128, 100, 300, 512),      # window >= ctx: whole context
    (2, 4, 16, 1, 128, 128, 300, 700, 256),
])
def test_decode_matches_brute_force(oracle_mod, B, T, H, Hk, D, page, lo, hi, window):
    d = workloads.make_decode(B=B, T=T, H=H, Hk=Hk, D=D, page=page, ctx_lo=lo, ctx_hi=hi,
                              seed=B * 100 + D)
    scale = 1.0 / math.sqrt(D)
    out, o64 = oracle_mod.decode(workloads.bits_u16(d["q"]), d["k_cache"].numpy(),
                                 d["v_cache"].numpy(), d["k_scale"].numpy(), d["v_scale"].numpy(),
                                 d["page_table"].numpy(), d["ctx_lens"].numpy(), window, scale,
                                 want_f64=True)
    ref = _brute_decode(oracle_mod, d, window, scale)
    assert np.abs(o64 - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    assert np.array_equal(out, oracle_mod.f64_to_bf16(o64))


def test_decode_query_codes_match_torch_float8(oracle_mod):
    """The decode's query quantisation (rotation by the butterfly, scale
    max|q_hat| / 448, e4m3 codes) against scipy's Hadamard matrix and torch's
    float8 cast, code for code; an all-zero row gives scale 0 and +0 codes."""
    g = torch.Generator().manual_seed(11)
    for D in (64, 128):
        q = torch.randn((2, 3, 5, D), generator=g).to(torch.bfloat16)
        q[1, 2, 4] = 0.0
        codes, scales = oracle_mod.decode_quant_q(workloads.bits_u16(q))
        Hmat = scipy.linalg.hadamard(D).astype(np.float64)
        qf = q.float().numpy()
        for idx in np.ndindex(q.shape[:3]):
            qh = oracle_mod.fwht_f32(qf[idx][None, :])[0]
            assert np.abs(qh - qf[idx] @ Hmat).max() <= 1e-4 * max(1e-30, np.abs(qf[idx]).sum())
            a = np.float32(np.abs(qh).max())
            if a == 0:
                assert scales[idx] == 0 and (codes[idx] == 0).all()
                continue
            assert scales[idx] == np.float32(a / np.float32(448.0))
            r = np.float32(448.0) / a
            ref = torch.from_numpy((qh * r).astype(np.float32)).to(torch.float8_e4m3fn)
            assert np.array_equal(codes[idx], ref.view(torch.uint8).numpy())
            # the largest magnitude lands on 448 (code 0x7E, either sign)
            assert ((codes[idx] & 0x7F) == 0x7E).any()


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_decode_cache_variants_match_brute_force(oracle_mod, flags):
    """Per-tensor scales (one K and one V scale for the whole cache) and the
    transposed V cache ([num_pages, Hk, D, page]), the variants of the
    FlyDSL pa_decode page's shape list: the oracle on the variant's layout
    equals the brute force on the equivalent per-token, untransposed cache."""
    d = workloads.make_decode(B=2, T=4, H=16, Hk=2, D=128, page=64, ctx_lo=200, ctx_hi=500, seed=31)
    scale = 1.0 / math.sqrt(128)
    ksc, vsc, vc = d["k_scale"].numpy(), d["v_scale"].numpy(), d["v_cache"].numpy()
    if flags & 1:
        ks1, vs1 = np.float32(0.0123), np.float32(0.0456)
        d["k_scale"] = torch.full_like(d["k_scale"], float(ks1))
        d["v_scale"] = torch.full_like(d["v_scale"], float(vs1))
        ksc, vsc = np.array([ks1], dtype=np.float32), np.array([vs1], dtype=np.float32)
    if flags & 2:
        vc = np.ascontiguousarray(vc.transpose(0, 1, 3, 2))
    out, o64 = oracle_mod.decode(workloads.bits_u16(d["q"]), d["k_cache"].numpy(), vc, ksc, vsc,
                                 d["page_table"].numpy(), d["ctx_lens"].numpy(), 128, scale,
                                 want_f64=True, kv_flags=flags)
    ref = _brute_decode(oracle_mod, d, 128, scale)
    assert np.abs(o64 - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())


def _fp32_weight_decode(oracle_mod, d, window, scale, rel_noise, rng):
    """The decode written with numpy independently of the oracle, the way a
    kernel with a running maximum over key tiles and splits forms it: p_j in
    fp32, each weight p_j * v_scale_j rounded to bf16 at the scale of some
    earlier (smaller) maximum -- here a random factor 2^-u, u in [0, 4), per
    key -- and scaled back afterwards, times (1 + noise)."""
    q = d["q"].float().numpy()
    B, T, H, D = q.shape
    Hk, page = d["k_cache"].shape[1], d["k_cache"].shape[2]
    codes, qs = oracle_mod.decode_quant_q(workloads.bits_u16(d["q"]))
    qd = oracle_mod.e4m3_decode(codes)
    kdec = oracle_mod.e4m3_decode(d["k_cache"].numpy())
    vdec = oracle_mod.e4m3_decode(d["v_cache"].numpy())
    out = np.zeros((B, T, H, D))
    for b in range(B):
        ctx = int(d["ctx_lens"][b])
        toks = np.arange(ctx)
        phys = d["page_table"][b].numpy()[toks // page]
        for h in range(H):
            hk = h // (H // Hk)
            K = kdec[phys, hk, toks % page]
            V = vdec[phys, hk, toks % page]
            ks = d["k_scale"].numpy()[phys, hk, toks % page]
            vs = d["v_scale"].numpy()[phys, hk, toks % page]
            for t in range(T):
                p = ctx - T + t
                sl = slice(max(0, p - window + 1), p + 1)
                acc = (K[sl] @ qd[b, t, h]).astype(np.float32)
                y = (acc * ks[sl]).astype(np.float32) * np.float32(qs[b, t, h] * scale / D * math.log2(math.e))
                y = y.astype(np.float32)
                pw = np.exp2((y - y.max()).astype(np.float32)).astype(np.float64)
                shift = np.exp2(rng.uniform(0.0, 4.0, pw.shape))           # 2^u
                wv = (pw * shift).astype(np.float32) * vs[sl].astype(np.float32)
                wv = torch.from_numpy(wv.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
                wv = wv / shift * (1.0 + rel_noise * rng.uniform(-1.0, 1.0, pw.shape))
                out[b, t, h] = (wv @ V[sl]) / pw.sum()
    return out


def test_decode_weight_margin_bounds_rounding_at_another_scale(oracle_mod):
    """The oracle's decode margin, sum_j (ulp(w_j) / 2 + 2^-8 w_j) |v_j| / l:
    an independent
    numpy decode whose bf16 weights are rounded at other scales (as a kernel
    with running maxima does) stays within it everywhere, on rows peaked by
    k_scale x 20 where it moves elements by more than 1e-4; weights perturbed
    by 2^-5 (beyond a bf16 step) break it."""
    d = workloads.make_decode(B=6, T=4, H=16, Hk=1, D=128, page=64, ctx_lo=300, ctx_hi=600, seed=77)
    d["k_scale"] = d["k_scale"] * 20.0
    scale = 1.0 / math.sqrt(128)
    _, y, margin = oracle_mod.decode(workloads.bits_u16(d["q"]), d["k_cache"].numpy(),
                                     d["v_cache"].numpy(), d["k_scale"].numpy(), d["v_scale"].numpy(),
                                     d["page_table"].numpy(), d["ctx_lens"].numpy(), 256, scale,
                                     want_flip=True)
    rng = np.random.default_rng(2)
    got = _fp32_weight_decode(oracle_mod, d, 256, scale, 0.0, rng)
    dev = np.abs(got - y)
    assert (dev <= margin + 1e-6).all(), float((dev - margin).max())
    assert (dev > 1e-4).sum() > 0
    bad = _fp32_weight_decode(oracle_mod, d, 256, scale, 2.0 ** -5, rng)
    assert float((np.abs(bad - y) - margin).max()) > 1e-4


# OCP MX E2M1 magnitudes by the code's low three bits (bit 3 is the sign)
_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _mx_dequant(codes, sf, D):
    """Packed E2M1 [..., D/2] (element 2i in the low nibble of byte i) with
    e8m0 scales [..., D/32] -> float64 [..., D]."""
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[:-1] + (D,))
    val = np.where(nib & 8, -_E2M1[nib & 7], _E2M1[nib & 7])
    return val * np.repeat(np.exp2(sf.astype(np.float64) - 127.0), 32, axis=-1)


@pytest.mark.parametrize("B,T,H,Hk,D,window,page", [(2, 4, 16, 2, 128, 256, 128), (3, 1, 8, 1, 64, 1000, 128),
                                                    (2, 2, 8, 2, 128, 100, 16)])
def test_decode_mxfp4_cache_matches_brute_force(oracle_mod, B, T, H, Hk, D, window, page):
    """The MXFP4-cache decode (packed E2M1 K/V with an e8m0 scale per 32
    channels of a token) equals a brute force over the dequantised un-paged
    cache: the format's value table and 2^(E - 127), scipy's Hadamard matrix,
    torch's float8 cast of the rotated query and torch's bfloat16 cast of the
    PV weights p_j."""
    d = workloads.make_decode(B=B, T=T, H=H, Hk=Hk, D=D, page=page, ctx_lo=150, ctx_hi=600, seed=60 + D + page,
                              kv_format="mxfp4")
    scale = 1.0 / math.sqrt(D)
    out, o64 = oracle_mod.decode_mxfp4(workloads.bits_u16(d["q"]), d["k_cache"].numpy(), d["v_cache"].numpy(),
                                       d["k_scale"].numpy(), d["v_scale"].numpy(), d["page_table"].numpy(),
                                       d["ctx_lens"].numpy(), window, scale, want_f64=True)
    q = d["q"].float().numpy()
    Hmat = scipy.linalg.hadamard(D).astype(np.float64)
    kdq = _mx_dequant(d["k_cache"].numpy(), d["k_scale"].numpy(), D)
    vdq = _mx_dequant(d["v_cache"].numpy(), d["v_scale"].numpy(), D)
    ref = np.zeros((B, T, H, D))
    for b in range(B):
        ctx = int(d["ctx_lens"][b])
        toks = np.arange(ctx)
        phys = d["page_table"][b].numpy()[toks // page]
        for h in range(H):
            hk = h // (H // Hk)
            K, V = kdq[phys, hk, toks % page], vdq[phys, hk, toks % page]
            for t in range(T):
                qh = q[b, t, h] @ Hmat
                a = np.float32(np.abs(qh).max())
                s = a / np.float32(448.0)
                q8 = torch.from_numpy((qh * (np.float32(448.0) / a)).astype(np.float32)).to(torch.float8_e4m3fn)
                q8 = q8.to(torch.float64).numpy()
                p = ctx - T + t
                sl = slice(max(0, p - window + 1), p + 1)
                logits = (K[sl] @ q8) * float(s) * (scale / D)
                w = np.exp(logits - logits.max())
                wb = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
                ref[b, t, h] = (wb @ V[sl]) / w.sum()
    assert np.abs(o64 - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    assert np.array_equal(out, oracle_mod.f64_to_bf16(o64))
    # the block scales matter: with every scale taken as 1 the outputs move
    flat = _mx_dequant(d["k_cache"].numpy(), np.full_like(d["k_scale"].numpy(), 127), D)
    assert not np.allclose(flat, kdq)

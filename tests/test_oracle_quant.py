"""Pins of the oracle's smoothing and quantisation steps.

K smoothing subtracts the per-(b, h) mean of K over the sequence; that mean
is checked against math.fsum (an exactly rounded sum), and the premise that
smoothing K leaves softmax(Q K^T) unchanged is checked in fp64. INT8 and e4m3
quantisation are pinned by their round-trip error bounds, their range, the
code that the block maximum must reach, zero blocks, padding, and (for e4m3)
torch's own float8 conversion."""
import math

import numpy as np
import pytest
import torch

import workloads


def _bits(t):
    return workloads.bits_u16(t)


def test_k_mean_equals_exactly_rounded_mean(oracle_mod):
    q, k, v = workloads.make_prefill(B=2, H=3, Hk=3, L=777, D=64, seed=5, kbias_std=2.0)
    kb = _bits(k)
    got = oracle_mod.k_mean(kb)
    kf = oracle_mod.bf16_to_f32(kb).astype(np.float64)
    for b in range(2):
        for h in range(3):
            for d in range(64):
                s = math.fsum(kf[b, h, :, d].tolist())
                assert got[b, h, d] == np.float32(s / 777.0)


def test_smoothing_k_leaves_softmax_unchanged():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((50, 32))
    k = rng.standard_normal((70, 32)) + rng.standard_normal((1, 32)) * 4
    mean = k.mean(axis=0, keepdims=True)

    def softmax(s):
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        return e / e.sum(axis=1, keepdims=True)

    a = softmax(q @ k.T * 0.3)
    b = softmax(q @ (k - mean).T * 0.3)
    assert np.abs(a - b).max() < 1e-12
    # smoothing Q instead would NOT be invariant (this is why only K is smoothed)
    qm = q.mean(axis=0, keepdims=True)
    c = softmax((q - qm) @ k.T * 0.3)
    assert np.abs(a - c).max() > 1e-3


@pytest.mark.parametrize("blk", [64, 128])
def test_int8_block_quant_bounds(oracle_mod, blk):
    L, D = 300, 128
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=L, D=D, seed=9, kbias_std=2.0,
                                     outlier_channels=4)
    res = oracle_mod.quant_qk(_bits(q), _bits(k), blk, blk)
    kmean = res["kmean"]
    for name, x, mean in (("q", q, None), ("k", k, kmean)):
        codes = res[name + "8"].astype(np.int64)
        scales = res[name + "s"]
        xf = oracle_mod.bf16_to_f32(_bits(x))
        if mean is not None:
            xf = (xf - mean[:, :, None, :]).astype(np.float32)
        xh = oracle_mod.fwht_f32(xf).astype(np.float64)
        nb = (L + blk - 1) // blk
        assert scales.shape == (1, 2, nb)
        assert codes.shape[2] == 384 and (codes[:, :, L:] == 0).all()
        assert np.abs(codes).max() <= 127
        for h in range(2):
            for bi in range(nb):
                r0, r1 = bi * blk, min(L, (bi + 1) * blk)
                s = float(scales[0, h, bi])
                c = codes[0, h, r0:r1]
                xb = xh[0, h, r0:r1]
                assert s == np.float32(np.abs(xb).max()) / np.float32(127.0)
                assert np.abs(c).max() == 127
                err = np.abs(xb - c * s)
                assert (err <= s / 2 * (1 + 2.0 ** -20)).all()


def test_int8_zero_block_and_short_tail(oracle_mod):
    L, D = 130, 64
    x = torch.zeros((1, 1, L, D), dtype=torch.bfloat16)
    x[0, 0, 128:, :] = 1.0                      # only the 2-row tail is nonzero
    res = oracle_mod.quant_qk(_bits(x), _bits(x), 64, 64)
    assert res["qs"][0, 0, 0] == 0 and res["qs"][0, 0, 1] == 0
    assert (res["q8"][0, 0, :128] == 0).all()
    # tail block: rotated rows are 64 * e_0 -> amax 64, code 127 at d = 0 only
    assert res["qs"][0, 0, 2] == np.float32(64.0) / np.float32(127.0)
    assert (res["q8"][0, 0, 128:130, 0] == 127).all()
    assert (res["q8"][0, 0, 128:130, 1:] == 0).all()


def test_v_e4m3_channel_quant(oracle_mod):
    L, D = 333, 64
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=L, D=D, seed=13, heavy_frac=0.05)
    v8t, vs = oracle_mod.quant_v(_bits(v))
    assert v8t.shape == (1, 2, D, 384) and (v8t[:, :, :, L:] == 0).all()
    vf = oracle_mod.bf16_to_f32(_bits(v))                     # [1, 2, L, D]
    for h in range(2):
        a = np.abs(vf[0, h]).max(axis=0)                      # [D]
        assert np.array_equal(vs[0, h], (a / np.float32(448.0)).astype(np.float32))
        r = (np.float32(448.0) / a).astype(np.float32)
        prod = (vf[0, h] * r[None, :]).astype(np.float32)     # [L, D]
        ref = torch.from_numpy(prod).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(v8t[0, h, :, :L], ref.T)
        dec = oracle_mod.e4m3_decode(v8t[0, h, :, :L]).T * vs[0, h][None, :].astype(np.float64)
        err = np.abs(dec - vf[0, h])
        bound = np.maximum(2.0 ** -4 * np.abs(vf[0, h]), 2.0 ** -10 * vs[0, h][None, :]) * 1.001
        assert (err <= bound).all()
        # the channel maximum maps to +-448
        assert (np.abs(oracle_mod.e4m3_decode(v8t[0, h, :, :L])).max(axis=1) == 448.0).all()


def test_v_zero_channel(oracle_mod):
    v = torch.zeros((1, 1, 10, 64), dtype=torch.bfloat16)
    v[0, 0, :, 1:] = 0.5
    v8t, vs = oracle_mod.quant_v(_bits(v))
    assert vs[0, 0, 0] == 0 and (v8t[0, 0, 0] == 0).all()
    assert (v8t[0, 0, 1:, :10] == 0x7E).all()

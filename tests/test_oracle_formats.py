"""Pins of the oracle's number formats (bf16, OCP e4m3) against torch's own
conversions (library routines) and against values the pages print."""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_torch_for_all_codes(oracle_mod):
    ours = oracle_mod.e4m3_decode(np.arange(256))
    ref = _torch_e4m3_values()
    nan_ours, nan_ref = np.isnan(ours), np.isnan(ref)
    assert (nan_ours == nan_ref).all()
    assert nan_ours.sum() == 2          # 0x7F and 0xFF
    assert np.array_equal(ours[~nan_ours], ref[~nan_ref])


def test_e4m3_max_is_the_page_fp8_max(oracle_mod):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "fp8_e4m3_max.txt"))
            if l.strip() and not l.startswith("#")]
    fp8_max = {name: float(v) for name, v in rows}
    vals = oracle_mod.e4m3_decode(np.arange(256))
    assert np.nanmax(vals) == fp8_max["e4m3fn"] == oracle_mod.E4M3_MAX
    assert oracle_mod.e4m3_decode(np.array([0x7E]))[0] == 448.0
    # finfo of the torch dtype the page names agrees
    assert float(torch.finfo(torch.float8_e4m3fn).max) == fp8_max["e4m3fn"]
    assert float(torch.finfo(torch.float8_e4m3fnuz).max) == fp8_max["e4m3fnuz"]


def test_e4m3_roundtrip_every_finite_code(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle_mod.e4m3_decode(codes)
    back = oracle_mod.e4m3_encode(vals)
    assert np.array_equal(back, codes)


def test_e4m3_encode_matches_torch_rne_below_max(oracle_mod):
    g = torch.Generator().manual_seed(7)
    x = torch.cat([
        torch.randn(20000, generator=g) * 50,
        torch.randn(20000, generator=g) * 0.01,            # subnormal range (< 2^-6)
        (torch.rand(5000, generator=g) * 2 - 1) * 447.9,
    ]).to(torch.float32)
    ours = oracle_mod.e4m3_encode(x.numpy().astype(np.float64))
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_ties_go_to_even_and_saturate(oracle_mod):
    enc = lambda v: int(oracle_mod.e4m3_encode(np.array([v]))[0])
    # 1.0 = 0x38, 1.125 = 0x39, 1.25 = 0x3A: midpoint 1.0625 -> even 0x38,
    # midpoint 1.1875 -> even 0x3A
    assert enc(1.0) == 0x38 and enc(1.0625) == 0x38 and enc(1.1875) == 0x3A
    # subnormal grid 2^-9: 1.5 * 2^-9 ties between codes 1 and 2 -> 2
    assert enc(1.5 * 2.0 ** -9) == 0x02 and enc(0.5 * 2.0 ** -9) == 0x00
    # saturation to +-448, NaN code, signed zero
    for v in (448.0, 449.0, 464.0, 1e6, float("inf")):
        assert enc(v) == 0x7E and enc(-v) == 0xFE
    assert enc(float("nan")) == 0x7F
    assert enc(-1e-9) == 0x80 and enc(0.0) == 0x00


def test_bf16_rounding_matches_torch(oracle_mod):
    g = torch.Generator().manual_seed(11)
    x = torch.cat([
        torch.randn(30000, generator=g) * 3,
        torch.randn(2000, generator=g) * 1e-39,           # bf16 subnormals
        torch.tensor([3.0e38, -3.39e38, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 0.0, -0.0]),
    ]).to(torch.float32)
    ours = oracle_mod.f64_to_bf16(x.numpy().astype(np.float64))
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = oracle_mod.bf16_to_f32(ref)
    assert np.array_equal(back.view(np.uint32) >> 16, ref.astype(np.uint32))


def test_e4m3_encode_every_rounding_boundary(oracle_mod):
    """The encoder is a search over the sorted code values, so it is monotonic
    and every fp32 input is pinned once each rounding boundary is: for every
    pair of neighbouring finite codes, the midpoint (exact in fp32) and the
    fp32 values just below and above it, both signs, against torch's cast."""
    vals = np.sort(np.unique(np.abs(oracle_mod.e4m3_decode(np.arange(256))[
        np.isfinite(oracle_mod.e4m3_decode(np.arange(256)))])))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    pts = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(np.inf)),
                          vals.astype(np.float32)])
    pts = np.concatenate([pts, -pts]).astype(np.float32)
    ours = oracle_mod.e4m3_encode(pts.astype(np.float64))
    ref = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert len(mids) == 126 and np.array_equal(ours, ref)


def test_int8_magic_rounding_is_round_half_even():
    """The quantisation kernels round x_hat * r to an integer by adding
    1.5 * 2^23 in fp32 and keeping the low byte of the sum. For every fp32
    value of magnitude in [2^-2, 128) (all smaller ones round to 0 both ways)
    that equals round-half-even, as the oracle's rint does."""
    magic = np.float32(12582912.0)
    for e in range(-2, 7):
        mant = np.arange(1 << 23, dtype=np.uint32)
        bits = ((np.uint32(127 + e) << np.uint32(23)) | mant).view(np.float32)
        for x in (bits, -bits):
            s = (x + magic).astype(np.float32)
            low = (s.view(np.uint32) & np.uint32(0xFF)).astype(np.uint8).view(np.int8)
            ref = np.rint(x.astype(np.float64))
            ok = np.abs(ref) <= 127
            assert np.array_equal(low[ok].astype(np.int64), ref[ok].astype(np.int64)), e
    small = np.array([0.25, -0.25, 0.5, -0.5, 1e-30, -1e-30, 0.0, -0.0], dtype=np.float32)
    s = (small + magic).astype(np.float32)
    assert np.array_equal((s.view(np.uint32) & np.uint32(0xFF)).astype(np.uint8).view(np.int8),
                          np.rint(small).astype(np.int8))

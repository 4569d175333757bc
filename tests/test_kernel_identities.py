"""Arithmetic identities the CUDA kernels rely on, checked on the CPU over
every input they can meet (the kernels themselves are checked against the
oracle by the GPU tests):

* attention: the int32 QK accumulator is summed onto the bit pattern of
  1.5 * 2^23, so the accumulated word read as fp32 is 1.5 * 2^23 + acc,
  and subtracting 1.5 * 2^23 gives acc exactly, for every |acc| <= 127 *
  127 * 128 (D = 128 products of two codes in [-127, 127]);
* decode: an e4m3 code moved into the top byte of a bf16 lane and shifted
  right by 4 (sign kept) is a bf16 whose value times 2^120 is the code's
  value, subnormal codes included;
* attention: the FMA-pipe exp2 that takes every 8th key pair keeps its
  stated relative error bound;
* decode over an MXFP4 cache: an E2M1 code's three magnitude bits placed at
  bf16 bits 6..8 and its sign at bit 15 read as a bf16 of value x * 2^-126,
  and one bf16 product by 2^(E - 1) (E <= 128; else by 2^126 and then by
  2^(E - 127)) is exactly x * 2^(E - 127) for every block exponent E the
  kernel accepts (0 .. 252); a word of eight codes becomes the four pairs
  (element m, element m + 4), the order the bf16 query rows are given too."""
import numpy as np
import torch


def test_biased_int32_accumulator_reads_as_fp32():
    bias = np.int64(0x4B400000)
    acc = np.arange(-127 * 127 * 128, 127 * 127 * 128 + 1, dtype=np.int64)
    word = (bias + acc).astype(np.uint32)
    as_f32 = word.view(np.float32)
    back = (as_f32 - np.float32(12582912.0)).astype(np.float64)
    assert np.array_equal(back, acc.astype(np.float64))


def test_e4m3_code_to_bf16_by_shift_and_scale():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint32)
    lane = codes << np.uint32(8)                        # the code byte at bits 8..15 of a 16-bit lane
    bits = ((lane >> np.uint32(4)) & np.uint32(0x07F0)) | (lane & np.uint32(0x8000))
    as_f32 = (bits << np.uint32(16)).astype(np.uint32).view(np.float32).astype(np.float64)
    got = as_f32 * 2.0 ** 120                           # exact: a power-of-two scaling
    ref = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got, ref)
    # the scaled values are bf16-representable and the subnormal codes (exponent field 0)
    # land on bf16 subnormals, which the multiply keeps
    assert (np.abs(as_f32[np.abs(ref) > 0]) < 2.0 ** -126).any()


def _e2m1_value(n):
    """The OCP MX E2M1 value of 4-bit code n (sign, two exponent bits with
    bias 1, one mantissa bit; exponent 0 is subnormal), from the format's
    definition."""
    sign = -1.0 if n & 8 else 1.0
    e, m = (n >> 1) & 3, n & 1
    return sign * (0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m))


def _bf16_bits_value(bits):
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def _exact_in_bf16(x):
    t = torch.tensor([x], dtype=torch.float64)
    return t.to(torch.bfloat16).to(torch.float64).item() == x


def test_e2m1_code_to_bf16_by_bit_placement_and_block_scale():
    for n in range(16):
        bits = ((n & 8) << 12) | ((n & 7) << 6)
        x = _e2m1_value(n)
        placed = _bf16_bits_value(bits)
        assert placed * 2.0 ** 126 == x, n
        for E in range(0, 253):
            if E <= 128:
                c = 2.0 ** (E - 1)                   # one product
                assert _exact_in_bf16(c)
                y = placed * c
            else:
                c1, c2 = 2.0 ** 126, 2.0 ** (E - 127)
                assert _exact_in_bf16(c1) and _exact_in_bf16(c2)
                y1 = placed * c1
                assert _exact_in_bf16(y1)
                y = y1 * c2
            # each product is the exact value and a bf16 value, so the bf16
            # multiply rounds nothing (nonzero codes stay nonzero)
            assert y == x * 2.0 ** (E - 127), (n, E)
            assert _exact_in_bf16(y), (n, E)
    # the largest exponent read: 6 * 2^125 is still finite in bf16
    assert _exact_in_bf16(6.0 * 2.0 ** 125)


def test_e2m1_word_to_bf16_pairs_and_query_order():
    rng = np.random.default_rng(3)
    for w in [int(v) for v in rng.integers(0, 2 ** 32, size=200, dtype=np.uint64)] + [0xFFFFFFFF, 0x89ABCDEF]:
        nib = [(w >> (4 * i)) & 15 for i in range(8)]
        for m in range(4):
            a = (w << (6 - 4 * m)) if m < 2 else (w >> (4 * m - 6))
            sgn = (w << (12 - 4 * m)) & 0xFFFFFFFF
            bits = ((a & 0x01C001C0) | (sgn & 0x80008000)) & 0xFFFFFFFF
            lo, hi = _bf16_bits_value(bits & 0xFFFF), _bf16_bits_value(bits >> 16)
            assert lo * 2.0 ** 126 == _e2m1_value(nib[m]), (hex(w), m)
            assert hi * 2.0 ** 126 == _e2m1_value(nib[m + 4]), (hex(w), m)
    # the bf16 query rows: pair m of 8 e4m3 codes (bytes of words a, b) =
    # (code m, code m + 4), bytes m of a and b picked into bytes 1 and 3
    def byte_perm(x, y, sel):
        src = [(x >> (8 * i)) & 255 for i in range(4)] + [(y >> (8 * i)) & 255 for i in range(4)]
        return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))
    for a, b in [(0x03020100, 0x07060504), (0xF1E2D3C4, 0x8A9BACBD)]:
        for m in range(4):
            t = byte_perm(a, b, (m << 4) | ((4 + m) << 12))
            assert (t >> 8) & 255 == (a >> (8 * m)) & 255 and (t >> 24) & 255 == (b >> (8 * m)) & 255


def _poly_coefficients():
    """The degree-5 coefficients of the attention kernel's FMA-pipe exp2, read
    from the CUDA source (highest degree first)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "quantized_attention_smoothing_b200", "csrc", "sage_ptx.cuh")).read()
    body = src[src.index("void exp2_poly_x2"):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"f2_pack\((0x[0-9a-fA-F.]+p[-+]?\d+)f,", body)
    return [np.float32(float.fromhex(h)) for h in hexes]


def _fma32(a, b, c):
    # fp32 a*b + c: the product of two fp32 values is exact in fp64; the fp64
    # sum then rounds far below fp32 precision, so this differs from the
    # kernel's single rounding at most at exact fp32 halfway points (one fp32
    # ulp), which the bound below does not depend on
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def test_exp2_polynomial_error_bound():
    """The kernel's exp2 on the FMA pipe (a = n + f, n = rint(a) by the
    1.5 * 2^23 bias, 2^f by a degree-5 polynomial in fp32 Horner form, 2^n
    added into the exponent field) stays within its stated relative error
    of 2.2e-7 over a in [-125, 9], evaluated step by step as the kernel does."""
    coef = _poly_coefficients()
    assert len(coef) == 6
    g = np.random.default_rng(5)
    a = np.concatenate([
        g.uniform(-125.0, 9.0, 3_000_000),
        g.uniform(-1.0, 1.0, 1_000_000),
        np.arange(-125, 10, dtype=np.float64) + 0.5,      # f = +-0.5 ties
        np.arange(-125, 10, dtype=np.float64),
    ]).astype(np.float32)
    a = np.maximum(a, np.float32(-125.0))
    bias = np.float32(12582912.0)
    t = (a + bias).astype(np.float32)
    n = (t - bias).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), a)
    p = np.full_like(f, coef[0])
    for c in coef[1:]:
        p = _fma32(p, f, np.full_like(f, c))
    e = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    e = e.astype(np.uint32).view(np.float32).astype(np.float64)
    exact = np.exp2(a.astype(np.float64))
    rel = np.abs(e - exact) / exact
    assert rel.max() <= 2.2e-7, rel.max()

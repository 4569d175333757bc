"""Arithmetic identities the CUDA kernels rely on, checked on the CPU over
every input they can meet (the kernels themselves are checked against the
oracle by the GPU tests):

* attention: the int32 QK accumulator is summed onto the bit pattern of
  1.5 * 2^23, so the accumulated word read as fp32 is 1.5 * 2^23 + acc,
  and subtracting 1.5 * 2^23 gives acc exactly, for every |acc| <= 127 *
  127 * 128 (D = 128 products of two codes in [-127, 127]);
* decode: an e4m3 code moved into the top byte of a bf16 lane and shifted
  right by 4 (sign kept) is a bf16 whose value times 2^120 is the code's
  value, subnormal codes included."""
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

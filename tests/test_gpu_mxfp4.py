"""GPU parity of the MXFP4 variant (sage_quant_qk_mx + sage_attn_fwd_mx)
against the CPU oracle: the E2M1 codes, the e8m0 scales (in the layout the
block-scaled MMA reads) and the K mean bit for bit; the attention output
element by element (with the oracle's P-rounding margin) on shapes spanning
several key tiles, ragged tails, causal masks (bottom-right aligned), GQA
and both head dims, and on sampled rows of the full B1 H24 L4096 workload."""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_smoothing_b200 as sage
import workloads
from gpu_helpers import bits, compare_output, sample_rows, to_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def handles():
    from quantized_attention_smoothing_b200 import build
    build.build()
    return {64: sage.Hadamard(64), 128: sage.Hadamard(128)}


def sf_plain(sf_tiles, D):
    """[B, H, Lpad/128, 512] scale blocks (row r, block j at 16 (r % 32) +
    4 (r // 32) + j) -> plain [B, H, Lpad, D/32]."""
    B, H, T, _ = sf_tiles.shape
    r = np.arange(128)
    out = np.zeros((B, H, T * 128, D // 32), dtype=np.uint8)
    for j in range(D // 32):
        out[:, :, :, j] = sf_tiles[:, :, :, 16 * (r % 32) + 4 * (r // 32) + j].reshape(B, H, T * 128)
    return out


def _inputs(B, H, Hk, Lq, Lk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Lq, H, D), generator=g).to(torch.bfloat16).permute(0, 2, 1, 3)
    k = (torch.randn((B, Lk, Hk, D), generator=g) + torch.randn((B, 1, Hk, D), generator=g) * 2)
    k = k.to(torch.bfloat16).permute(0, 2, 1, 3)
    v = torch.randn((B, Lk, Hk, D), generator=g).to(torch.bfloat16).permute(0, 2, 1, 3)
    return q, k, v


def _check_quant(bufs, ref, D, label):
    for name, gpu in (("q4", bufs.q4), ("k4", bufs.k4)):
        a = gpu.cpu().numpy()
        bad = np.argwhere(a != ref[name])
        assert bad.size == 0, "%s %s differs at %d places, first %s" % (label, name, len(bad), tuple(bad[0]))
    for name, gpu in (("qsf", bufs.q_sf), ("ksf", bufs.k_sf)):
        tiles = gpu.cpu().numpy()
        assert np.array_equal(sf_plain(tiles, D), ref[name]), "%s %s" % (label, name)
        if D == 64:                                   # the unused scale slots are zero
            r = np.arange(128)
            for j in (2, 3):
                assert (tiles[:, :, :, 16 * (r % 32) + 4 * (r // 32) + j] == 0).all()
    assert np.array_equal(bufs.k_mean.cpu().numpy().view(np.uint32), ref["kmean"].view(np.uint32))


SHAPES = [
    # B, H, Hk, Lq, Lk, D, causal
    (1, 2, 2, 256, 256, 128, False),
    (1, 2, 2, 300, 300, 128, False),        # ragged tail
    (1, 2, 2, 383, 383, 128, True),         # causal, ragged
    (2, 4, 2, 257, 513, 64, False),         # GQA, Lq != Lk, D = 64
    (1, 2, 1, 129, 1000, 128, True),        # causal with Lq < Lk
    (1, 1, 1, 500, 130, 64, True),          # causal with Lq > Lk: early rows see nothing
    (1, 1, 1, 1, 1, 128, False),            # single token
    (1, 3, 3, 640, 640, 128, False),        # 5 key tiles
]


@pytest.mark.parametrize("B,H,Hk,Lq,Lk,D,causal", SHAPES)
def test_mxfp4_quant_and_attention_match_oracle(handles, B, H, Hk, Lq, Lk, D, causal):
    q, k, v = _inputs(B, H, Hk, Lq, Lk, D, Lq * 13 + Lk + D)
    scale = 1.0 / math.sqrt(D)
    out, bufs = sage.sage_attention_mx(handles[D], to_gpu(q), to_gpu(k), to_gpu(v), scale, causal)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    ref = oracle.quant_qk_mxfp4(bits(q), bits(k))
    _check_quant(bufs, ref, D, str((B, H, Hk, Lq, Lk, D)))
    v8t, vs = oracle.quant_v(bits(v))
    _, y, margin = oracle.attn_mxfp4(ref["q4"], ref["qsf"], ref["k4"], ref["ksf"], v8t, vs, Lq, Lk, scale,
                                     causal, want_flip=True)
    compare_output(bits(out), (y, margin), None, label="mxfp4 " + str((B, H, Hk, Lq, Lk, D, causal)))
    if causal and Lq > Lk:
        assert (bits(out)[:, :, :Lq - Lk] == 0).all()


def test_mxfp4_full_size_c2_sampled_rows(handles):
    """The B1 H24 L4096 D128 workload: quantised tensors bit for bit, the
    output on sampled rows of every head (tile edges and the tail included)."""
    cfg, q, k, v = workloads.make_prefill_config("c2")
    out, bufs = sage.sage_attention_mx(handles[128], to_gpu(q), to_gpu(k), to_gpu(v),
                                       cfg["softmax_scale"], cfg["causal"])
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    ref = oracle.quant_qk_mxfp4(bits(q), bits(k))
    _check_quant(bufs, ref, 128, "c2")
    v8t, vs = oracle.quant_v(bits(v))
    rows = sample_rows(cfg["L"], 16, seed=cfg["H"])
    _, y, margin = oracle.attn_mxfp4(ref["q4"], ref["qsf"], ref["k4"], ref["ksf"], v8t, vs, cfg["L"],
                                     cfg["L"], cfg["softmax_scale"], False, rows=rows, want_flip=True)
    compare_output(bits(out)[:, :, rows], (y, margin), None, label="mxfp4 c2")


def test_mxfp4_output_strides(handles):
    q, k, v = _inputs(1, 2, 2, 300, 300, 128, 5)
    h = handles[128]
    qg, kg, vg = to_gpu(q), to_gpu(k), to_gpu(v)
    o1 = torch.empty((1, 2, 300, 128), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty((1, 2, 300, 131), dtype=torch.bfloat16, device="cuda")[..., :128]
    a, _ = sage.sage_attention_mx(h, qg, kg, vg, 0.1, False, out=o1)
    b, _ = sage.sage_attention_mx(h, qg, kg, vg, 0.1, False, out=o2)
    torch.cuda.synchronize()
    assert torch.equal(a, b.contiguous())

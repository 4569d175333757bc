"""GPU parity of the quantisation kernels (smoothing, Hadamard, INT8, e4m3)
against the CPU oracle: bit-exact codes and fp32 scales, on the seeded
workloads, on 1- to 4-tile boundary lengths (the byte-parity shapes of "Sage2
SM89 Temporal Pair Experiment", Run On Spark), and for several input
layouts (strided views take another load path with identical results)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_smoothing_b200 as sage
import workloads
from gpu_helpers import assert_quant_bitexact, bits, gpu_quant, to_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H128():
    from quantized_attention_smoothing_b200 import build
    build.build()
    return sage.Hadamard(128)


@pytest.fixture(scope="module")
def H64():
    return sage.Hadamard(64)


def _check(h, q, k, v, blk_q, blk_k):
    """Both entry paths -- sage_quant_qk + sage_quant_v, and sage_quant_qkv --
    against the oracle."""
    ref = oracle.quant_qk(bits(q), bits(k), blk_q, blk_k)
    ref_v8t, ref_vs = oracle.quant_v(bits(v))
    qg, kg, vg = to_gpu(q), to_gpu(k), to_gpu(v)
    for fused in (False, True):
        bufs = gpu_quant(h, qg, kg, vg, blk_q, blk_k, fused=fused)
        assert_quant_bitexact(bufs, ref, ref_v8t, ref_vs, q.shape[2], k.shape[2])


def test_hadamard_handle_matrix(H128, H64):
    import scipy.linalg
    assert np.array_equal(H128.matrix(), scipy.linalg.hadamard(128).astype(np.int8))
    assert np.array_equal(H64.matrix(), scipy.linalg.hadamard(64).astype(np.int8))


@pytest.mark.parametrize("key", ["c1", "c2"])
def test_quant_bitexact_configs(key, H128, H64):
    cfg, q, k, v = workloads.make_prefill_config(key)
    _check(H128 if cfg["D"] == 128 else H64, q, k, v, cfg["blk_q"], cfg["blk_k"])


@pytest.mark.parametrize("L", [1, 63, 64, 65, 127, 128, 129, 255, 256, 257, 383, 384, 385, 511,
                               512, 513])
@pytest.mark.parametrize("D", [64, 128])
def test_quant_bitexact_boundary_lengths(L, D, H128, H64):
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=L, D=D, seed=1000 + L, kbias_std=2.0,
                                     outlier_channels=2, heavy_frac=0.02)
    _check(H128 if D == 128 else H64, q, k, v, 64, 32 if L % 2 else 128)


@pytest.mark.parametrize("layout", ["bhld", "blhd", "dstride2", "oddrow"])
def test_quant_bitexact_layouts(layout, H128):
    B, H, L, D = 2, 3, 300, 128
    q, k, v = workloads.make_prefill(B=B, H=H, Hk=H, L=L, D=D, seed=77, kbias_std=3.0,
                                     layout="bhld" if layout == "bhld" else "blhd")
    if layout == "dstride2":
        def widen(t):
            w = torch.zeros((B, H, L, 2 * D), dtype=torch.bfloat16)
            w[..., ::2] = t
            return w[..., ::2]
        q, k, v = widen(q), widen(k), widen(v)
        assert q.stride(3) == 2
    elif layout == "oddrow":
        def pad(t):
            w = torch.zeros((B, H, L, D + 3), dtype=torch.bfloat16)
            w[..., :D] = t
            return w[..., :D]
        q, k, v = pad(q), pad(k), pad(v)
        assert q.stride(2) == D + 3
    _check(H128, q, k, v, 128, 64)


def test_quant_gqa_and_zero_blocks(H128):
    q, k, v = workloads.make_prefill(B=1, H=4, Hk=2, L=200, D=128, seed=5, kbias_std=1.0)
    q = q.clone()
    v = v.clone()
    q[:, :, 64:128] = 0          # an all-zero Q block (blk 64) -> scale 0
    v[:, :, :, 5] = 0            # an all-zero V channel
    _check(H128, q, k, v, 64, 64)


def test_quant_deterministic(H128):
    cfg, q, k, v = workloads.make_prefill_config("c1")
    h = sage.Hadamard(64)
    a = gpu_quant(h, to_gpu(q), to_gpu(k), to_gpu(v), 64, 64)
    b = gpu_quant(h, to_gpu(q), to_gpu(k), to_gpu(v), 64, 64)
    c = gpu_quant(h, to_gpu(q), to_gpu(k), to_gpu(v), 64, 64, fused=True)
    for name in ("q8", "q_scale", "k8", "k_scale", "k_mean", "v8_t", "v_scale"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert torch.equal(getattr(a, name), getattr(c, name)), name


def test_quant_qkv_gqa_grid_parity():
    """sage_quant_qkv over many heads and odd tile counts: the K/V tiles
    alternate in the tile list and the persistent grid is made odd, so every
    CTA sees both kinds; GQA gives Q more heads than K and V."""
    h = sage.Hadamard(128)
    q, k, v = workloads.make_prefill(B=2, H=12, Hk=3, L=1000, D=128, seed=4242, kbias_std=2.0,
                                     outlier_channels=3, heavy_frac=0.02)
    _check(h, q, k, v, 128, 64)


def test_quant_qkv_rejects_mismatched_v(H128):
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=256, D=128, seed=3)
    bufs = sage.QuantBuffers(1, 2, 2, 256, 256, 128, 64, 64)
    with pytest.raises(sage.SageError) as e:
        sage.sage_quant_qkv(H128, to_gpu(q), to_gpu(k), to_gpu(v[:, :, :200]), 64, 64, bufs.q8,
                            bufs.q_scale, bufs.k8, bufs.k_scale, bufs.v8_t, bufs.v_scale,
                            bufs.k_mean, bufs.ws)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG


@pytest.mark.parametrize("key", ["c3", "c4"])
def test_quant_bitexact_full_size(key, H128):
    cfg, q, k, v = workloads.make_prefill_config(key)
    _check(H128, q, k, v, cfg["blk_q"], cfg["blk_k"])

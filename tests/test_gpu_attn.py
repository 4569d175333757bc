"""GPU parity of the quantised attention forward (tcgen05 kernel) against
the CPU oracle. Element-wise on small shapes spanning several 128-key tiles
with ragged tails, causal masks (bottom-right aligned), GQA, both head dims
and all block sizes, for both the separate-Q and the in-CTA-Q paths; at the
full workload sizes every element of the B1 H24 L4096 workload, every element
of a quarter of the causal B2 H32 L8192 workload's heads, and sampled rows of
the B1 H40 L32760 workload. The oracle quantises the original inputs itself
(nothing it uses comes from the GPU)."""
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


def _oracle(q, k, v, blk_q, blk_k, scale, causal, rows=None, exact=True):
    """The oracle's quantised output (fp64 before its bf16 rounding) with its
    P-rounding margin, and the unquantised fp64 reference, from the original
    bf16 inputs."""
    qk = oracle.quant_qk(bits(q), bits(k), blk_q, blk_k)
    v8t, vs = oracle.quant_v(bits(v))
    _, ref, margin = oracle.attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, q.shape[2],
                                 k.shape[2], blk_q, blk_k, scale, causal, rows=rows, want_flip=True)
    ex = oracle.attn_exact(bits(q), bits(k), bits(v), scale, causal, rows=rows) if exact else None
    return (ref, margin), ex


def _run(handles, q, k, v, blk_q, blk_k, scale, causal, rows=None, exact=True, fused_q=False,
         heads=None):
    """GPU output (bf16 bits) of the whole path, and the oracle's on the same
    inputs. heads: compare only these head indices (the GPU runs them all)."""
    D = q.shape[3]
    run = sage.sage_attention_q16 if fused_q else sage.sage_attention
    out, _ = run(handles[D], to_gpu(q), to_gpu(k), to_gpu(v), blk_q, blk_k, scale, causal)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    gpu = bits(out)                                     # [B, H, Lq, D]
    if heads is not None:
        gpu = gpu[:, heads]
        q, k, v = q[:, heads], k[:, heads], v[:, heads]
    ref, ex = _oracle(q, k, v, blk_q, blk_k, scale, causal, rows=rows, exact=exact)
    if rows is not None:
        gpu = gpu[:, :, rows]
    return gpu, ref, ex


def _shape_inputs(B, H, Hk, Lq, Lk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Lq, H, D), generator=g).to(torch.bfloat16).permute(0, 2, 1, 3)
    k = (torch.randn((B, Lk, Hk, D), generator=g) + torch.randn((B, 1, Hk, D), generator=g) * 2)
    k = k.to(torch.bfloat16).permute(0, 2, 1, 3)
    v = torch.randn((B, Lk, Hk, D), generator=g).to(torch.bfloat16).permute(0, 2, 1, 3)
    return q, k, v


SHAPES = [
    # B, H, Hk, Lq, Lk, D, blk_q, blk_k, causal
    (1, 2, 2, 256, 256, 64, 64, 64, False),          # the small config
    (1, 2, 2, 300, 300, 128, 128, 64, False),        # ragged tail
    (1, 2, 2, 383, 383, 128, 128, 64, True),         # causal, ragged
    (2, 4, 2, 257, 513, 64, 64, 32, False),          # GQA, Lq != Lk
    (1, 2, 1, 129, 1000, 128, 128, 128, True),       # causal with Lq < Lk
    (1, 1, 1, 500, 130, 64, 64, 64, True),           # causal with Lq > Lk: early rows see nothing
    (1, 1, 1, 1, 1, 128, 32, 32, False),             # single token
    (1, 3, 3, 640, 640, 128, 64, 128, False),        # 5 key tiles, 3 CTAs (odd q-tile count)
]


@pytest.mark.parametrize("B,H,Hk,Lq,Lk,D,blk_q,blk_k,causal", SHAPES)
def test_attn_matches_oracle_elementwise(handles, B, H, Hk, Lq, Lk, D, blk_q, blk_k, causal):
    q, k, v = _shape_inputs(B, H, Hk, Lq, Lk, D, Lq * 31 + Lk + D)
    scale = 1.0 / math.sqrt(D)
    gpu, ref, ex = _run(handles, q, k, v, blk_q, blk_k, scale, causal)
    compare_output(gpu, ref, ex, label=str((B, H, Hk, Lq, Lk, D, causal)))
    if causal and Lq > Lk:
        assert (gpu[:, :, :Lq - Lk] == 0).all()


def test_attn_c1_config(handles):
    cfg, q, k, v = workloads.make_prefill_config("c1")
    gpu, ref, ex = _run(handles, q, k, v, cfg["blk_q"], cfg["blk_k"], cfg["softmax_scale"],
                        cfg["causal"])
    compare_output(gpu, ref, ex, label="c1")


def test_attn_output_strides(handles):
    """Contiguous [B,H,L,D] output, the [B,L,H,D] view, and a scalar-path view."""
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=300, D=128, seed=8, kbias_std=2.0)
    h = handles[128]
    qg, kg, vg = to_gpu(q), to_gpu(k), to_gpu(v)
    outs = []
    o1 = torch.empty((1, 2, 300, 128), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty((1, 300, 2, 128), dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)
    o3 = torch.empty((1, 2, 300, 131), dtype=torch.bfloat16, device="cuda")[..., :128]
    for o in (o1, o2, o3):
        sage.sage_attention(h, qg, kg, vg, 128, 64, 0.1, False, out=o)
        outs.append(o.contiguous())
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_attn_deterministic(handles):
    cfg, q, k, v = workloads.make_prefill_config("c1")
    h = handles[64]
    a, _ = sage.sage_attention(h, to_gpu(q), to_gpu(k), to_gpu(v), 64, 64, 0.125, False)
    b, _ = sage.sage_attention(h, to_gpu(q), to_gpu(k), to_gpu(v), 64, 64, 0.125, False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_attn_full_size_c2_every_element(handles):
    """The B1 H24 L4096 D128 video-DiT workload compared in full: every
    output element of every head against the oracle."""
    cfg, q, k, v = workloads.make_prefill_config("c2")
    gpu, ref, ex = _run(handles, q, k, v, cfg["blk_q"], cfg["blk_k"], cfg["softmax_scale"],
                        cfg["causal"], exact=True)
    compare_output(gpu, ref, ex, label="c2 full")


def test_attn_full_size_c3_quarter_of_heads(handles):
    """The causal B2 H32 L8192 D128 workload: every output element of a
    seeded quarter of its heads (8 of 32, in both batches) against the
    oracle; the GPU computes all heads in one launch."""
    cfg, q, k, v = workloads.make_prefill_config("c3")
    heads = np.sort(np.random.default_rng(cfg["H"]).choice(cfg["H"], size=cfg["H"] // 4,
                                                            replace=False))
    gpu, ref, ex = _run(handles, q, k, v, cfg["blk_q"], cfg["blk_k"], cfg["softmax_scale"],
                        cfg["causal"], exact=True, heads=heads)
    compare_output(gpu, ref, ex, label="c3 heads %s" % heads.tolist())


def test_attn_full_size_c4_sampled_rows(handles):
    """The long B1 H40 L32760 D128 workload (a ragged last tile) on sampled
    rows of every head, tile edges and the tail included."""
    cfg, q, k, v = workloads.make_prefill_config("c4")
    rows = sample_rows(cfg["L"], 4, seed=cfg["H"])
    gpu, ref, ex = _run(handles, q, k, v, cfg["blk_q"], cfg["blk_k"], cfg["softmax_scale"],
                        cfg["causal"], rows=rows, exact=True)
    compare_output(gpu, ref, ex, label="c4")


@pytest.mark.parametrize("B,H,Hk,Lq,Lk,D,blk_q,blk_k,causal", SHAPES)
def test_attn_q16_matches_oracle_elementwise(handles, B, H, Hk, Lq, Lk, D, blk_q, blk_k, causal):
    """Q rotated and quantised inside the attention kernel, compared with the
    oracle element by element (the oracle quantises Q itself)."""
    q, k, v = _shape_inputs(B, H, Hk, Lq, Lk, D, Lq * 29 + Lk + D + 5)
    scale = 1.0 / math.sqrt(D)
    gpu, ref, ex = _run(handles, q, k, v, blk_q, blk_k, scale, causal, fused_q=True)
    compare_output(gpu, ref, ex, label="q16 " + str((B, H, Hk, Lq, Lk, D, causal)))


@pytest.mark.parametrize("B,H,Hk,Lq,Lk,D,blk_q,blk_k,causal", SHAPES)
def test_attn_q16_same_bits(handles, B, H, Hk, Lq, Lk, D, blk_q, blk_k, causal):
    """Q rotated and quantised inside the attention kernel (sage_quant_k +
    sage_attn_fwd_q16) gives the same output bits as sage_quant_qk +
    sage_attn_fwd: same codes, same block scales, same kernel after them."""
    g = torch.Generator().manual_seed(Lq * 17 + Lk + D)
    q = torch.randn((B, Lq, H, D), generator=g).to(torch.bfloat16).permute(0, 2, 1, 3)
    k = (torch.randn((B, Lk, Hk, D), generator=g) + torch.randn((B, 1, Hk, D), generator=g) * 2)
    k = k.to(torch.bfloat16).permute(0, 2, 1, 3)
    v = torch.randn((B, Lk, Hk, D), generator=g).to(torch.bfloat16).permute(0, 2, 1, 3)
    qg, kg, vg = to_gpu(q), to_gpu(k), to_gpu(v)
    a, _ = sage.sage_attention(handles[D], qg, kg, vg, blk_q, blk_k, 0.1, causal)
    b, _ = sage.sage_attention_q16(handles[D], qg, kg, vg, blk_q, blk_k, 0.1, causal)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    assert torch.equal(a, b)


def test_attn_q16_strided_query(handles):
    """The in-CTA Q path on a row-strided view (vector loads) and on a view
    whose channels are not contiguous (scalar loads)."""
    q, k, v = workloads.make_prefill(B=1, H=2, Hk=2, L=300, D=128, seed=21, kbias_std=2.0)
    kg, vg = to_gpu(k), to_gpu(v)
    ref, _ = sage.sage_attention(handles[128], to_gpu(q), kg, vg, 128, 64, 0.1, False)
    wide = torch.zeros((1, 2, 300, 136), dtype=torch.bfloat16, device="cuda")
    wide[..., :128] = to_gpu(q)
    inter = torch.zeros((1, 2, 300, 128, 2), dtype=torch.bfloat16, device="cuda")
    inter[..., 0] = to_gpu(q)
    for qv in (wide[..., :128], inter[..., 0]):
        o, _ = sage.sage_attention_q16(handles[128], qv, kg, vg, 128, 64, 0.1, False)
        torch.cuda.synchronize()
        assert torch.equal(o, ref)
    oref, ex = _oracle(q, k, v, 128, 64, 0.1, False)
    compare_output(bits(ref), oref, ex, label="q16 strided")

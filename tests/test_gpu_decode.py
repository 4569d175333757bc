"""GPU parity of the paged FP8 decode (sage_attn_decode) against the CPU
oracle, element-wise: the MTP4 / GQA16 / page-128 / window-4096 workload of
the FlyDSL pa_decode page's window family, and small shapes covering other
page sizes, short contexts, windows wider than the context, padded row
grids (T * H / Hk < 64) and strided query/output views. Every call also
returns the e4m3 query codes and scales its QK product used, which must equal
the oracle's per-token query quantisation bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_smoothing_b200 as sage
import workloads
from gpu_helpers import COS_ORACLE, MAX_ABS, bf16_ulp, bits, compare_output, cosine, workloads_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h128():
    from quantized_attention_smoothing_b200 import build
    build.build()
    return sage.Hadamard(128)


@pytest.fixture(scope="module")
def h64():
    from quantized_attention_smoothing_b200 import build
    build.build()
    return sage.Hadamard(64)


def _run(h, d, window, scale, q_layout="btHd", out_layout="btHd"):
    q = d["q"]
    B, T, H, D = q.shape
    if q_layout == "strided":           # [B, T, H, D] view of a [B, H, T, D+8] buffer
        buf = torch.zeros((B, H, T, D + 8), dtype=torch.bfloat16)
        buf[..., :D] = q.permute(0, 2, 1, 3)
        qg = buf.cuda().permute(0, 2, 1, 3)[..., :D]
    else:
        qg = q.cuda()
    if out_layout == "strided":
        og = torch.empty((B, H, T, D + 8), dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)[..., :D]
    else:
        og = torch.empty((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros((max(16, sage.sage_attn_decode_workspace(B, T, H, d["k_cache"].shape[1], D,
                                                               window)),),
                     dtype=torch.uint8, device="cuda")
    q8 = torch.full((B, T, H, D), 0x7F, dtype=torch.uint8, device="cuda")
    qsc = torch.full((B, T, H), float("nan"), dtype=torch.float32, device="cuda")
    sage.sage_attn_decode(h, qg, d["k_cache"].cuda(), d["v_cache"].cuda(), d["k_scale"].cuda(),
                          d["v_scale"].cuda(), d["page_table"].cuda(), d["ctx_lens"].cuda(),
                          d["k_cache"].shape[2], d["num_pages"], window, scale, og, ws,
                          q8_out=q8, q_scale_out=qsc)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    # the e4m3 query codes and scales the kernel's QK used, bit for bit
    ref_codes, ref_scales = oracle.decode_quant_q(workloads.bits_u16(q))
    got_codes = q8.cpu().numpy()
    bad = np.argwhere(got_codes != ref_codes)
    assert bad.size == 0, "query codes differ at %d places, first %s" % (len(bad), tuple(bad[0]))
    assert np.array_equal(qsc.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    _, ref, margin = oracle.decode(workloads.bits_u16(q), d["k_cache"].numpy(), d["v_cache"].numpy(),
                                   d["k_scale"].numpy(), d["v_scale"].numpy(), d["page_table"].numpy(),
                                   d["ctx_lens"].numpy(), window, scale, want_flip=True)
    return bits(og.contiguous()), (ref, margin)


def _row_max_share(d, window, scale):
    """max_j p_j / sum_j p_j of every (b, t, h) row, in fp64 with numpy from
    the oracle's query codes: how strongly the row's largest key dominates."""
    q = d["q"]
    B, T, H, D = q.shape
    Hk, page = d["k_cache"].shape[1], d["k_cache"].shape[2]
    codes, qs = oracle.decode_quant_q(workloads.bits_u16(q))
    qd = oracle.e4m3_decode(codes)
    kdec = oracle.e4m3_decode(d["k_cache"].numpy())
    ksc = d["k_scale"].numpy().astype(np.float64)
    out = np.zeros((B, T, H))
    for b in range(B):
        ctx = int(d["ctx_lens"][b])
        toks = np.arange(ctx)
        phys = d["page_table"][b].numpy()[toks // page]
        for h in range(H):
            hk = h // (H // Hk)
            K = kdec[phys, hk, toks % page]
            ks = ksc[phys, hk, toks % page]
            for t in range(T):
                p = ctx - T + t
                sl = slice(max(0, p - window + 1), p + 1)
                x = (K[sl] @ qd[b, t, h]) * float(qs[b, t, h]) * ks[sl] * (scale / D)
                w = np.exp(x - x.max())
                out[b, t, h] = w.max() / w.sum()
    return out


def test_decode_window_family_workload(h128):
    cfg, d = workloads.make_decode_config("c5")
    gpu, ref = _run(h128, d, cfg["window"], cfg["softmax_scale"])
    stats = compare_output(gpu, ref, None, label="c5")
    assert stats["cos_oracle"] >= 0.9999


@pytest.mark.parametrize("B,T,H,Hk,page,lo,hi,window", [
    (3, 4, 8, 2, 16, 40, 90, 32),        # page 16, window < ctx, R = 16
    (2, 1, 8, 1, 128, 100, 300, 512),    # T = 1, window >= ctx, R = 8 (padded rows)
    (2, 2, 16, 2, 64, 257, 700, 256),    # page 64, R = 16
    (4, 4, 16, 1, 32, 4, 30, 4096),      # tiny contexts
    (1, 3, 12, 3, 128, 1000, 1000, 300), # T = 3, G = 4
    (2, 4, 16, 2, 16, 5000, 6000, 8192), # page 16, long window: page ids refetched 32 at a time
    (40, 2, 8, 1, 128, 1500, 2500, 4096),# 40 clusters: more than one wave of them
    (2, 3, 16, 1, 64, 700, 1200, 1024),  # R = 48: one softmax warp per group sits out
    (3, 1, 16, 1, 128, 3000, 5000, 8192),# R = 16, T = 1: the query rows repeated four times
])
def test_decode_shapes(h128, B, T, H, Hk, page, lo, hi, window):
    d = workloads.make_decode(B=B, T=T, H=H, Hk=Hk, D=128, page=page, ctx_lo=lo, ctx_hi=hi,
                              seed=B * 1000 + page + window)
    gpu, ref = _run(h128, d, window, 1.0 / math.sqrt(128))
    compare_output(gpu, ref, None, label=str((B, T, H, Hk, page, window)))


def test_decode_strided_views(h128):
    d = workloads.make_decode(B=2, T=4, H=16, Hk=1, D=128, page=128, ctx_lo=600, ctx_hi=900,
                              seed=77)
    a, ref = _run(h128, d, 512, 0.08)
    b, _ = _run(h128, d, 512, 0.08, q_layout="strided", out_layout="strided")
    assert np.array_equal(a, b)
    compare_output(a, ref, None, label="strided")


def test_decode_dominant_keys(h128):
    """Keys whose k_scale is multiplied by 40, spread over the window, give
    logits far above the running maximum in later tiles of a split (O is
    rescaled in TMEM there) and rows dominated by one key. Both sides round
    every PV weight w_j = p_j * v_scale_j to bf16, but the kernel rounds it
    at the running maximum of its tile and split and rescales afterwards,
    the oracle at the window maximum: the oracle's margin bounds the effect
    (each weight within half a bf16 step on either side). Rows where no
    single key carries a tenth of the weight must meet the plain bar."""
    d = workloads.make_decode(B=4, T=4, H=16, Hk=1, D=128, page=128, ctx_lo=3000, ctx_hi=5000,
                              seed=4242)
    ksc = d["k_scale"].clone()
    rng = np.random.default_rng(5)
    for b in range(4):
        ctx = int(d["ctx_lens"][b])
        lo = max(0, ctx - 4 - 4096 + 1)
        for j in rng.integers(lo, ctx, size=24):
            pg = int(d["page_table"][b, j // 128])
            ksc[pg, 0, j % 128] *= 40.0
    d["k_scale"] = ksc
    scale = 1.0 / math.sqrt(128)
    gpu, (ref, margin) = _run(h128, d, 4096, scale)
    share = _row_max_share(d, 4096, scale)               # [B, T, H]
    compare_output(gpu, (ref, margin), None, label="dominant keys")
    g = workloads_f32(gpu).astype(np.float64)
    ulp = bf16_ulp(np.maximum(np.abs(g), np.abs(ref)))
    plain = np.abs(g - ref) - ulp / 2
    # rows where no single key carries a tenth of the weight meet the plain
    # bar; only rows dominated by a few keys may use the margin
    spread = np.broadcast_to((share < 0.1)[..., None], plain.shape)
    assert float(plain[spread].max()) <= MAX_ABS, float(plain[spread].max())
    n_extra = int((plain > MAX_ABS).sum())
    print("dominant keys: %d of %d rows dominated (a key >= 10%% of the weight); %d of %d "
          "elements need the bf16 weight-rounding margin" % (int((share >= 0.1).sum()), share.size,
                                                             n_extra, plain.size))


def test_decode_subnormal_v_codes(h128):
    """A V cache of e4m3 subnormal codes only (exponent field 0, values
    m * 2^-9, m = 0..7, either sign) with a large v_scale: the exact e4m3 ->
    bf16 conversion of V must keep them (flushing them would zero the
    output)."""
    d = workloads.make_decode(B=2, T=4, H=16, Hk=1, D=128, page=128, ctx_lo=500, ctx_hi=900, seed=99)
    g = torch.Generator().manual_seed(3)
    codes = torch.randint(0, 16, d["v_cache"].shape, generator=g, dtype=torch.int32)
    d["v_cache"] = ((codes & 7) | ((codes & 8) << 4)).to(torch.uint8)
    d["v_scale"] = torch.full_like(d["v_scale"], 64.0)
    gpu, ref = _run(h128, d, 4096, 1.0 / math.sqrt(128))
    assert np.abs(ref).max() > 0.05
    compare_output(gpu, ref, None, label="subnormal V")


def test_decode_reports_bad_page_ids(h128):
    """A page-table entry outside [0, num_pages) for a page inside the window
    is not dereferenced: its keys are left out, the output stays finite and
    sage_device_error reports SAGE_ERR_INVALID_ARG (then clears it)."""
    d = workloads.make_decode(B=2, T=4, H=16, Hk=1, D=128, page=128, ctx_lo=600, ctx_hi=900, seed=5)
    ptab = d["page_table"].clone()
    ptab[1, 2] = d["num_pages"] + 7
    q = d["q"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    ws = None                                   # allocated by the binding
    sage.sage_attn_decode(h128, q, d["k_cache"].cuda(), d["v_cache"].cuda(), d["k_scale"].cuda(),
                          d["v_scale"].cuda(), ptab.cuda(), d["ctx_lens"].cuda(), 128, d["num_pages"],
                          4096, 1.0 / math.sqrt(128), out, ws)
    assert sage.sage_device_error() == sage.SAGE_ERR_INVALID_ARG
    assert sage.sage_device_error() == sage.SAGE_OK
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("flags", [1, 2, 3])
@pytest.mark.parametrize("B,T,H,Hk,lo,hi,window", [
    (16, 4, 16, 1, 4096, 8192, 4096),     # the window-family workload's shape
    (3, 2, 8, 2, 100, 900, 512),           # GQA 4, short contexts, T = 2
])
def test_decode_cache_variants(h128, flags, B, T, H, Hk, lo, hi, window):
    """Per-tensor K/V scales (SAGE_KV_PER_TENSOR_SCALES: a cache quantised
    with one amax / 448 scale per tensor) and the transposed V cache
    (SAGE_KV_V_TRANSPOSED, [num_pages, Hk, D, 128]), alone and together,
    against the oracle on the same layout; and bit for bit against the
    default layout given the same data (the per-tensor scale repeated in
    every per-token slot, V untransposed)."""
    d = workloads.make_decode(B=B, T=T, H=H, Hk=Hk, D=128, page=128, ctx_lo=lo, ctx_hi=hi,
                              seed=B * 7 + flags, scale_mode="per_tensor" if flags & 1 else "per_token")
    scale = 1.0 / math.sqrt(128)
    q = d["q"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    ws = None                                   # allocated by the binding
    ksc, vsc, vc = d["k_scale"], d["v_scale"], d["v_cache"]
    kfull = ksc.expand(d["k_cache"].shape[:3]).contiguous() if flags & 1 else ksc
    vfull = vsc.expand(d["k_cache"].shape[:3]).contiguous() if flags & 1 else vsc
    if flags & 2:
        vc = vc.permute(0, 1, 3, 2).contiguous()
    tabs = [d["page_table"].cuda(), d["ctx_lens"].cuda()]
    sage.sage_attn_decode(h128, q, d["k_cache"].cuda(), vc.cuda(), ksc.cuda(), vsc.cuda(), tabs[0], tabs[1],
                          128, d["num_pages"], window, scale, out, ws, kv_flags=flags)
    ref_out = torch.empty_like(out)
    sage.sage_attn_decode(h128, q, d["k_cache"].cuda(), d["v_cache"].cuda(), kfull.cuda(), vfull.cuda(),
                          tabs[0], tabs[1], 128, d["num_pages"], window, scale, ref_out, ws)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    assert torch.equal(out, ref_out)
    _, ref, margin = oracle.decode(workloads.bits_u16(d["q"]), d["k_cache"].numpy(), vc.numpy(),
                                   ksc.numpy(), vsc.numpy(), d["page_table"].numpy(),
                                   d["ctx_lens"].numpy(), window, scale, want_flip=True, kv_flags=flags)
    compare_output(bits(out), (ref, margin), None, label="kv_flags %d %s" % (flags, (B, T, H, Hk)))


def test_decode_rejects_bad_kv_flags(h128):
    d = workloads.make_decode(B=1, T=1, H=8, Hk=1, D=128, page=64, ctx_lo=100, ctx_hi=200, seed=1)
    q = d["q"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    args = [h128, q, d["k_cache"].cuda(), d["v_cache"].cuda(), d["k_scale"].cuda(), d["v_scale"].cuda(),
            d["page_table"].cuda(), d["ctx_lens"].cuda(), 64, d["num_pages"], 128, 0.1, out]
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_decode(*args, kv_flags=2)          # transposed V needs page 128
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_decode(*args, kv_flags=4)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG


@pytest.mark.parametrize("B,T,H,Hk,page,lo,hi,window", [
    (16, 4, 16, 1, 128, 4096, 8192, 4096),  # the window-family shape at D = 64
    (3, 4, 8, 2, 16, 40, 90, 32),           # page 16, window < ctx, R = 16
    (2, 1, 8, 1, 128, 100, 300, 512),       # T = 1, window >= ctx, R = 8 (padded rows)
    (2, 2, 16, 2, 64, 257, 700, 256),       # page 64, R = 16
    (1, 3, 12, 3, 32, 1000, 1000, 300),     # page 32, T = 3, G = 4
    (2, 2, 16, 1, 128, 600, 1500, 512),     # R = 32: the query rows repeated twice
])
def test_decode_head64(h64, B, T, H, Hk, page, lo, hi, window):
    """Head size 64 ("[FlyDSL] [Misc] pa_decode ...", Performance: FP8 KV at
    D64/128/256): 64-byte e4m3 rows (64B swizzle), a 64-channel bf16 V and
    PV of N = 64; query codes bit-exact and the output within tolerance."""
    d = workloads.make_decode(B=B, T=T, H=H, Hk=Hk, D=64, page=page, ctx_lo=lo, ctx_hi=hi,
                              seed=B * 3000 + page + window)
    gpu, ref = _run(h64, d, window, 1.0 / math.sqrt(64))
    stats = compare_output(gpu, ref, None, label="D64 %s" % ((B, T, H, Hk, page, window),))
    assert stats["cos_oracle"] >= 0.9999


def test_decode_head64_strided_views(h64):
    d = workloads.make_decode(B=2, T=4, H=16, Hk=1, D=64, page=64, ctx_lo=500, ctx_hi=900, seed=23)
    gpu, ref = _run(h64, d, 1024, 0.125, q_layout="strided", out_layout="strided")
    compare_output(gpu, ref, None, label="D64 strided")


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_decode_head64_cache_variants(h64, flags):
    """Per-tensor scales and the transposed V cache ([num_pages, Hk, 64, 128])
    at D = 64, against the oracle on the same layout."""
    d = workloads.make_decode(B=4, T=4, H=16, Hk=1, D=64, page=128, ctx_lo=600, ctx_hi=2000,
                              seed=70 + flags, scale_mode="per_tensor" if flags & 1 else "per_token")
    scale, window = 0.125, 1024
    q = d["q"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    vc = d["v_cache"]
    if flags & 2:
        vc = vc.permute(0, 1, 3, 2).contiguous()
    sage.sage_attn_decode(h64, q, d["k_cache"].cuda(), vc.cuda(), d["k_scale"].cuda(), d["v_scale"].cuda(),
                          d["page_table"].cuda(), d["ctx_lens"].cuda(), 128, d["num_pages"], window, scale,
                          out, kv_flags=flags)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    _, ref, margin = oracle.decode(workloads.bits_u16(d["q"]), d["k_cache"].numpy(), vc.numpy(),
                                   d["k_scale"].numpy(), d["v_scale"].numpy(), d["page_table"].numpy(),
                                   d["ctx_lens"].numpy(), window, scale, want_flip=True, kv_flags=flags)
    compare_output(bits(out), (ref, margin), None, label="D64 kv_flags %d" % flags)


@pytest.mark.parametrize("D", [128, 64])
def test_decode_one_split_per_sequence(h128, h64, D):
    """B * Hk at or above the SM count: every (sequence, kv head) runs in one
    CTA, which normalises and writes its rows itself (no workspace, no merge
    launch)."""
    B = 160
    assert sage.sage_attn_decode_workspace(B, 2, 8, 1, D, 96) == 0
    d = workloads.make_decode(B=B, T=2, H=8, Hk=1, D=D, page=16, ctx_lo=20, ctx_hi=300, seed=400 + D)
    gpu, ref = _run(h128 if D == 128 else h64, d, 96, 1.0 / math.sqrt(D))
    compare_output(gpu, ref, None, label="one split, D %d" % D)

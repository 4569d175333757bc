"""GPU parity of the paged decode over an MXFP4 cache (sage_attn_decode_mxfp4)
against the CPU oracle, element-wise: the FlyDSL pa_decode page's MXFP4 KV
shape (GQA 16, page 128, batch 32, ctx 2k, every key in the window) and
small shapes covering the other page sizes, MTP rows, sliding windows,
split and unsplit sequences and strided views; plus the format's corners:
subnormal E2M1 codes, block exponents above 128 (two bf16 products), any
bytes in the masked cache slots, and the refusals. Every call also returns
the e4m3 query codes and scales, which must equal the oracle's bit for
bit."""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_smoothing_b200 as sage
import workloads
from gpu_helpers import bits, compare_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h128():
    from quantized_attention_smoothing_b200 import build
    build.build()
    return sage.Hadamard(128)


def _call(h, d, window, scale, q_layout="btHd", out_layout="btHd", ws="zeros"):
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
    wsb = None
    if ws == "zeros":
        wsb = torch.zeros((max(16, sage.sage_attn_decode_workspace(B, T, H, d["k_cache"].shape[1], D,
                                                                    window)),),
                          dtype=torch.uint8, device="cuda")
    q8 = torch.full((B, T, H, D), 0x7F, dtype=torch.uint8, device="cuda")
    qsc = torch.full((B, T, H), float("nan"), dtype=torch.float32, device="cuda")
    sage.sage_attn_decode_mxfp4(h, qg, d["k_cache"].cuda(), d["v_cache"].cuda(), d["k_scale"].cuda(),
                                d["v_scale"].cuda(), d["page_table"].cuda(), d["ctx_lens"].cuda(),
                                d["k_cache"].shape[2], d["num_pages"], window, scale, og, wsb,
                                q8_out=q8, q_scale_out=qsc)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    return og, q8, qsc


def _run(h, d, window, scale, **kw):
    og, q8, qsc = _call(h, d, window, scale, **kw)
    q = d["q"]
    ref_codes, ref_scales = oracle.decode_quant_q(workloads.bits_u16(q))
    bad = np.argwhere(q8.cpu().numpy() != ref_codes)
    assert bad.size == 0, "query codes differ at %d places, first %s" % (len(bad), tuple(bad[0]))
    assert np.array_equal(qsc.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    _, ref, margin = oracle.decode_mxfp4(workloads.bits_u16(q), d["k_cache"].numpy(), d["v_cache"].numpy(),
                                         d["k_scale"].numpy(), d["v_scale"].numpy(),
                                         d["page_table"].numpy(), d["ctx_lens"].numpy(), window, scale,
                                         want_flip=True)
    return bits(og.contiguous()), (ref, margin)


def _mx(B, T, H, Hk, page, lo, hi, seed):
    return workloads.make_decode(B=B, T=T, H=H, Hk=Hk, D=128, page=page, ctx_lo=lo, ctx_hi=hi, seed=seed,
                                 kv_format="mxfp4")


@pytest.mark.parametrize("B,T,H,Hk,page,lo,hi,window", [
    (32, 1, 16, 1, 128, 2048, 2048, 1 << 20),   # the page's MXFP4 KV shape: GQA 16, page 128, b32, ctx 2k
    (16, 4, 16, 1, 128, 4096, 8192, 4096),      # the window-family shape (MTP4) over an MXFP4 cache
    (3, 4, 8, 2, 16, 40, 90, 32),               # page 16, window < ctx, R = 16
    (2, 1, 8, 1, 128, 100, 300, 512),           # T = 1, window >= ctx, R = 8 (padded rows)
    (2, 2, 16, 2, 64, 257, 700, 256),           # page 64
    (1, 3, 12, 3, 32, 1000, 1000, 300),         # page 32, T = 3, G = 4
    (4, 4, 16, 1, 32, 4, 30, 4096),             # tiny contexts
    (160, 2, 8, 1, 16, 20, 300, 96),            # B * Hk >= the SM count: one CTA per sequence
    (3, 3, 8, 1, 64, 300, 900, 512),            # R = 24: the query rows repeated twice
    (2, 3, 16, 1, 128, 700, 1200, 1024),        # R = 48: one softmax warp per group sits out
])
def test_decode_mx_shapes(h128, B, T, H, Hk, page, lo, hi, window):
    d = _mx(B, T, H, Hk, page, lo, hi, seed=B * 500 + page + window % 9973)
    gpu, ref = _run(h128, d, window, 1.0 / math.sqrt(128))
    stats = compare_output(gpu, ref, None, label="mx %s" % ((B, T, H, Hk, page, window),))
    assert stats["cos_oracle"] >= 0.9999


def test_decode_mx_strided_views_and_binding_workspace(h128):
    d = _mx(2, 4, 16, 1, 128, 600, 900, seed=31)
    a, ref = _run(h128, d, 512, 0.08)
    b, _ = _run(h128, d, 512, 0.08, q_layout="strided", out_layout="strided", ws=None)
    assert np.array_equal(a, b)
    compare_output(a, ref, None, label="mx strided")


def test_decode_mx_any_bytes_in_masked_slots(h128):
    """The slots past ctx of each sequence's last page, read with its tile but
    masked, hold scale code 255 (NaN) and random codes: the output is the
    same bit for bit as with ordinary bytes there (a masked key's weight is
    an exact zero, and the kernel reads scale codes above 252 as 252)."""
    d = _mx(6, 2, 16, 1, 128, 300, 1000, seed=8)
    clean, ref = _run(h128, d, 4096, 1.0 / math.sqrt(128))
    ksf, vsf = d["k_scale"].clone(), d["v_scale"].clone()
    for b in range(6):
        ctx = int(d["ctx_lens"][b])
        if ctx % 128:
            pg = int(d["page_table"][b, (ctx - 1) // 128])
            ksf[pg, :, ctx % 128:] = 255
            vsf[pg, :, ctx % 128:] = 255
    d2 = dict(d, k_scale=ksf, v_scale=vsf)
    og, _, _ = _call(h128, d2, 4096, 1.0 / math.sqrt(128))
    assert np.array_equal(bits(og.contiguous()), clean)
    compare_output(clean, ref, None, label="mx masked slots")


def test_decode_mx_subnormal_codes(h128):
    """K and V of the codes 0, +-0.5 only (E2M1's subnormals: exponent field
    0): their bf16 form is a bf16 subnormal times 2^(E - 1), which must not
    be flushed."""
    d = _mx(2, 4, 16, 1, 128, 500, 900, seed=12)
    g = torch.Generator().manual_seed(4)
    for key in ("k_cache", "v_cache"):
        lo = torch.randint(0, 4, d[key].shape, generator=g, dtype=torch.int32)
        hi = torch.randint(0, 4, d[key].shape, generator=g, dtype=torch.int32)
        nib = torch.tensor([0, 1, 8, 9], dtype=torch.int32)
        d[key] = (nib[lo] | (nib[hi] << 4)).to(torch.uint8)
    gpu, ref = _run(h128, d, 4096, 1.0)
    assert np.abs(ref[0]).max() > 0.02
    compare_output(gpu, ref, None, label="mx subnormal codes")


def test_decode_mx_large_block_exponents(h128):
    """Block exponents 129 .. 140 (values up to 6 * 2^13) on V and on a few K
    blocks: the conversion takes its two-product path there (2^126, then
    2^(E - 127)); some keys dominate their rows."""
    d = _mx(3, 4, 16, 1, 128, 1500, 3000, seed=41)
    g = torch.Generator().manual_seed(6)
    d["v_scale"] = torch.randint(129, 141, d["v_scale"].shape, generator=g, dtype=torch.int32).to(torch.uint8)
    ksf = d["k_scale"].clone()
    sel = torch.rand(ksf.shape, generator=g) < 0.01
    ksf[sel] = 131
    d["k_scale"] = ksf
    gpu, ref = _run(h128, d, 4096, 1.0 / math.sqrt(128))
    assert np.abs(ref[0]).max() > 256.0
    compare_output(gpu, ref, None, label="mx large exponents")


def test_decode_mx_reports_bad_page_ids(h128):
    """A page-table entry outside [0, num_pages) for a page inside the window
    is not dereferenced (neither its codes nor its scale blocks): its keys are
    left out, the output stays finite and sage_device_error reports
    SAGE_ERR_INVALID_ARG (then clears it)."""
    d = _mx(2, 4, 16, 1, 128, 600, 900, seed=5)
    ptab = d["page_table"].clone()
    ptab[1, 2] = d["num_pages"] + 7
    q = d["q"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    sage.sage_attn_decode_mxfp4(h128, q, d["k_cache"].cuda(), d["v_cache"].cuda(), d["k_scale"].cuda(),
                                d["v_scale"].cuda(), ptab.cuda(), d["ctx_lens"].cuda(), 128, d["num_pages"],
                                4096, 1.0 / math.sqrt(128), out)
    assert sage.sage_device_error() == sage.SAGE_ERR_INVALID_ARG
    assert sage.sage_device_error() == sage.SAGE_OK
    assert torch.isfinite(out.float()).all()


def test_decode_mx_refusals(h128):
    d = _mx(1, 1, 8, 1, 64, 100, 200, seed=1)
    q = d["q"].cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    kc, vc = d["k_cache"].cuda(), d["v_cache"].cuda()
    ksf, vsf = d["k_scale"].cuda(), d["v_scale"].cuda()
    tabs = [d["page_table"].cuda(), d["ctx_lens"].cuda()]
    with pytest.raises(sage.SageError) as e:             # scale arrays must be 16-byte aligned
        sage.sage_attn_decode_mxfp4(h128, q, kc, vc, ksf.view(-1)[1:], vsf, *tabs, 64, d["num_pages"], 128,
                                    0.1, out)
    assert e.value.status == sage.SAGE_ERR_ALIGNMENT
    with pytest.raises(sage.SageError) as e:             # page sizes as for the FP8 cache
        sage.sage_attn_decode_mxfp4(h128, q, kc, vc, ksf, vsf, *tabs, 48, d["num_pages"], 128, 0.1, out)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    h64 = sage.Hadamard(64)
    q64 = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    o64 = torch.empty_like(q64)
    with pytest.raises(sage.SageError) as e:             # head size 128 only
        sage.sage_attn_decode_mxfp4(h64, q64, kc, vc, ksf, vsf, *tabs, 64, d["num_pages"], 128, 0.1, o64)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    assert sage.sage_device_error() == sage.SAGE_OK


@pytest.mark.parametrize("key", ["c7_mx", "c7", "c5_mx"])
def test_decode_bench_workloads_sampled(h128, key):
    """The decode workloads the bench times, at full size and in the bench's
    launch configuration (the whole batch in one call, the binding's split
    choice and workspace): the first and last sequences' rows against the
    oracle (which runs on those two sequences alone)."""
    cfg, d = workloads.make_decode_config(key)
    mx = cfg.get("kv_format") == "mxfp4"
    q = d["q"]
    B, T, H, D = q.shape
    qg = q.cuda()
    og = torch.empty((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    run = sage.sage_attn_decode_mxfp4 if mx else sage.sage_attn_decode
    run(h128, qg, d["k_cache"].cuda(), d["v_cache"].cuda(), d["k_scale"].cuda(), d["v_scale"].cuda(),
        d["page_table"].cuda(), d["ctx_lens"].cuda(), d["k_cache"].shape[2], d["num_pages"], cfg["window"],
        cfg["softmax_scale"], og)
    torch.cuda.synchronize()
    assert sage.sage_device_error() == sage.SAGE_OK
    pick = [0, B - 1]
    qb = workloads.bits_u16(q)[pick]
    fn = oracle.decode_mxfp4 if mx else oracle.decode
    _, ref, margin = fn(qb, d["k_cache"].numpy(), d["v_cache"].numpy(), d["k_scale"].numpy(),
                        d["v_scale"].numpy(), d["page_table"].numpy()[pick], d["ctx_lens"].numpy()[pick],
                        cfg["window"], cfg["softmax_scale"], want_flip=True)
    stats = compare_output(bits(og[pick].contiguous()), (ref, margin), None, label=key + " sampled")
    assert stats["cos_oracle"] >= 0.9999

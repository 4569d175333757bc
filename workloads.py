"""Seeded synthetic inputs for the quantized attention path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no smoothing, rotation or quantisation of its own), and
both the CUDA path and the CPU oracle take their inputs from it.

Workloads (shapes and value recipes) imitate the pages' workloads:
  * video-DiT prefill ("sage_attn3" API page and "Sage v2 improvements":
    [B, L, H, D] activations handed to the kernel as [B, H, L, D] views);
  * GQA paged FP8 decode with MTP4 and a sliding window (the FlyDSL pa_decode
    page, window-family results: per-token FP8 K/V, GQA16, D128, page 128,
    one KV head).

Every tensor is drawn from a CPU ``torch.Generator`` seeded per workload, so the
same seed gives the same bits on every machine. Prefill Q/K/V are returned as
[B, H, L, D] views of [B, L, H, D] storage (non-contiguous on purpose).
"""
import math

import torch

PREFILL = {
    "c1": dict(name="prefill_b1_h2_l256_d64", B=1, H=2, Hk=2, L=256, D=64, blk_q=64, blk_k=64,
               softmax_scale=1.0 / 8.0, causal=False, kbias_std=2.0, outlier_channels=0,
               outlier_mult=20.0, heavy_frac=0.0),
    "c2": dict(name="dit_prefill_b1_h24_l4096_d128", B=1, H=24, Hk=24, L=4096, D=128, blk_q=128,
               blk_k=64, softmax_scale=1.0 / math.sqrt(128.0), causal=False, kbias_std=2.0,
               outlier_channels=4, outlier_mult=20.0, heavy_frac=0.0),
    "c3": dict(name="causal_prefill_b2_h32_l8192_d128", B=2, H=32, Hk=32, L=8192, D=128,
               blk_q=128, blk_k=64, softmax_scale=1.0 / math.sqrt(128.0), causal=True,
               kbias_std=1.0, outlier_channels=0, outlier_mult=20.0, heavy_frac=0.0),
    "c4": dict(name="dit_long_b1_h40_l32760_d128", B=1, H=40, Hk=40, L=32760, D=128, blk_q=128,
               blk_k=64, softmax_scale=1.0 / math.sqrt(128.0), causal=False, kbias_std=3.0,
               outlier_channels=0, outlier_mult=20.0, heavy_frac=0.02),
}

DECODE = {
    "c5": dict(name="gqa_paged_decode_b16_t4_h16_hk1_d128_p128_w4096", B=16, T=4, H=16, Hk=1,
               D=128, page=128, ctx_lo=4096, ctx_hi=8192, window=4096,
               softmax_scale=1.0 / math.sqrt(128.0)),
    # the same window-family shape at head size 64 (the pages' decode shape
    # list runs D 64/128/256)
    "c5_d64": dict(name="gqa_paged_decode_b16_t4_h16_hk1_d64_p128_w4096", B=16, T=4, H=16, Hk=1,
                   D=64, page=128, ctx_lo=4096, ctx_hi=8192, window=4096,
                   softmax_scale=1.0 / math.sqrt(64.0)),
    # the window-family shape over an MXFP4 cache
    "c5_mx": dict(name="gqa_paged_decode_mxfp4_b16_t4_h16_hk1_d128_p128_w4096", B=16, T=4, H=16,
                  Hk=1, D=128, page=128, ctx_lo=4096, ctx_hi=8192, window=4096,
                  softmax_scale=1.0 / math.sqrt(128.0), kv_format="mxfp4"),
    # the pages' MXFP4 KV shape list (GQA 16, page 128, batch 1/32/256, ctx
    # 2k/32k) at batch 32 and ctx 32k, every key in the window, one query
    # token; and the same shape over the FP8 cache (per-token scales)
    "c7_mx": dict(name="gqa_paged_decode_mxfp4_b32_t1_h16_hk1_d128_p128_c32768", B=32, T=1, H=16,
                  Hk=1, D=128, page=128, ctx_lo=32768, ctx_hi=32768, window=32768,
                  softmax_scale=1.0 / math.sqrt(128.0), kv_format="mxfp4"),
    "c7": dict(name="gqa_paged_decode_b32_t1_h16_hk1_d128_p128_c32768", B=32, T=1, H=16, Hk=1,
               D=128, page=128, ctx_lo=32768, ctx_hi=32768, window=32768,
               softmax_scale=1.0 / math.sqrt(128.0)),
}

SEED_BASE = 20260000
CONFIG_INDEX = {"c1": 1, "c2": 2, "c3": 3, "c4": 4, "c5": 5, "c5_d64": 6, "c5_mx": 7, "c7": 8, "c7_mx": 9}


def seed_for(key):
    return SEED_BASE + CONFIG_INDEX[key]


def _student_t3(g, shape):
    """Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3)."""
    z = torch.randn(shape, generator=g)
    chi = torch.randn((3,) + tuple(shape), generator=g).pow(2).sum(0)
    return z / torch.sqrt(chi / 3.0)


def make_prefill(B, H, Hk, L, D, seed, kbias_std=0.0, outlier_channels=0, outlier_mult=20.0,
                 heavy_frac=0.0, layout="blhd", **_unused):
    """Q, K, V bf16 with logical shape [B, H(k), L, D].

    Values ~ N(0, 1). K gets a per-(b, h, d) channel bias ~ N(0, kbias_std^2).
    ``outlier_channels`` distinct channels per (b, h) of K are multiplied by
    ``outlier_mult`` before the bias. ``heavy_frac`` of the (h, d) channels of
    each of Q, K and V (ceil(frac * H * D) channels, shared over batch) are
    redrawn from Student-t(3). ``layout`` "blhd" stores [B, L, H, D] and
    returns permuted views; "bhld" returns contiguous tensors.
    """
    g = torch.Generator().manual_seed(int(seed))

    def draw(heads):
        return torch.randn((B, heads, L, D), generator=g)

    q = draw(H)
    k = draw(Hk)
    v = draw(Hk)
    if outlier_channels:
        for b in range(B):
            for h in range(Hk):
                ch = torch.randperm(D, generator=g)[:outlier_channels]
                k[b, h, :, ch] *= outlier_mult
    if kbias_std:
        k += torch.randn((B, Hk, 1, D), generator=g) * kbias_std
    if heavy_frac:
        for t, heads in ((q, H), (k, Hk), (v, Hk)):
            n = int(math.ceil(heavy_frac * heads * D))
            idx = torch.randperm(heads * D, generator=g)[:n]
            for flat in idx.tolist():
                h, d = divmod(flat, D)
                t[:, h, :, d] = _student_t3(g, (B, L))
    out = []
    for t in (q, k, v):
        tb = t.to(torch.bfloat16)
        if layout == "blhd":
            tb = tb.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        out.append(tb)
    return out[0], out[1], out[2]


def make_prefill_config(key, layout="blhd", seed=None):
    cfg = dict(PREFILL[key])
    q, k, v = make_prefill(seed=seed_for(key) if seed is None else seed, layout=layout, **cfg)
    return cfg, q, k, v


def make_decode(B, T, H, Hk, D, page, ctx_lo, ctx_hi, seed, scale_mode="per_token", kv_format="fp8",
                **_unused):
    """Paged FP8 decode inputs.

    ctx_b ~ U{ctx_lo..ctx_hi}; the pages of all sequences are one random
    permutation of the physical pages. Cached K/V values are N(0, 1) and
    stored as e4m3 codes with one fp32 scale per token (amax / 448), or with
    scale_mode="per_tensor" one scale for the whole cache (its amax / 448;
    k_scale and v_scale are then one-element tensors), the cast done by
    torch's float8_e4m3fn conversion (the cache writer itself is not part of
    the path). Queries are bf16 N(0, 1), [B, T, H, D].
    kv_format="mxfp4": an MXFP4 cache instead, drawn directly in its storage
    format: uniform random E2M1 codes packed two per byte [num_pages, Hk,
    page, D / 2] and e8m0 block scales [num_pages, Hk, page, D / 32] (uint8,
    in k_scale / v_scale) uniform in 2^-3 .. 2^1.
    Returns a dict of CPU tensors.
    """
    g = torch.Generator().manual_seed(int(seed))
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (B,), generator=g, dtype=torch.int64)
    pages_per = [(int(c) + page - 1) // page for c in ctx]
    total = sum(pages_per)
    max_pages = (ctx_hi + page - 1) // page
    perm = torch.randperm(total, generator=g)
    ptab = torch.zeros((B, max_pages), dtype=torch.int32)
    o = 0
    for b in range(B):
        ptab[b, :pages_per[b]] = perm[o:o + pages_per[b]].to(torch.int32)
        o += pages_per[b]

    def cache():
        x = torch.randn((total, Hk, page, D), generator=g)
        if scale_mode == "per_tensor":
            scale = (x.abs().amax() / 448.0).reshape(1)
            codes = (x / scale).to(torch.float8_e4m3fn).view(torch.uint8)
            return codes.contiguous(), scale.to(torch.float32).contiguous()
        amax = x.abs().amax(dim=-1)
        scale = amax / 448.0
        codes = (x / scale.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
        return codes.contiguous(), scale.to(torch.float32).contiguous()

    def cache_mx():
        codes = torch.randint(0, 256, (total, Hk, page, D // 2), generator=g, dtype=torch.int32)
        sf = 127 + torch.randint(-3, 2, (total, Hk, page, D // 32), generator=g, dtype=torch.int32)
        return codes.to(torch.uint8).contiguous(), sf.to(torch.uint8).contiguous()

    kc, ksc = cache_mx() if kv_format == "mxfp4" else cache()
    vc, vsc = cache_mx() if kv_format == "mxfp4" else cache()
    q = torch.randn((B, T, H, D), generator=g).to(torch.bfloat16)
    return dict(q=q, k_cache=kc, v_cache=vc, k_scale=ksc, v_scale=vsc, page_table=ptab,
                ctx_lens=ctx.to(torch.int32), num_pages=total, max_pages=max_pages)


def make_decode_config(key="c5", seed=None):
    cfg = dict(DECODE[key])
    d = make_decode(seed=seed_for(key) if seed is None else seed, **cfg)
    return cfg, d


def bits_u16(t):
    """bf16 torch tensor (any strides) -> numpy uint16 view of the same bits."""
    import numpy as np
    return t.view(torch.int16).numpy().view(np.uint16)

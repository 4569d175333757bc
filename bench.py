#!/usr/bin/env python
"""Throughput of the quantised attention path on B200.

One step = the whole hot path on one batch of seeded synthetic inputs that
already sit in HBM: sage_quant_qkv (K mean, smoothing, Hadamard rotation, INT8
Q/K, e4m3 V; two launches) + sage_attn_fwd (INT8 QK^T, online softmax, e4m3
PV, bf16 out). Default workload: the long non-causal video-DiT attention
B=1 H=40 L=32760 D=128 (Q blocks 128 tokens, K blocks 64), the largest of the
single-GPU workloads. Metric: TOPS = 4 B H L^2 D / step time (halved for
causal). The line also carries the B1 H24 L4096 and the causal B2 H32 L8192
workloads under "configs", each with its attention roofline and its
quantisation bandwidth, and the paged decode: the MTP4 / GQA16 / window-4096
workload over the FP8 cache ("decode", head size 128; "decode_d64") and
over an MXFP4 cache ("decode_mxfp4"), and the batch-32 / ctx-32k / T-1
workload over both ("decode_long").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sage|reference]
                    [--workload c2|c3|c4]

N > 1 runs under torchrun: the workload's kv heads (with their query heads)
are split into N contiguous ranges, one per rank (the heads are independent,
so no data crosses ranks); timing is the max over ranks and `value` counts
the whole workload ("scaling": "strong"). `--impl reference` times the CPU
oracle on the host cores on a bounded sample of the same workload (rank 0
only).
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-attn TOPS (4*B*H*L^2*D/t) and % of B200 INT8/FP8 tensor peak"
UNIT = "TOPS"
INT8_OVER_BF16 = 2.0        # nominal dense INT8/FP8 : BF16 tensor ratio (4.5 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126e6


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sage", choices=["sage", "reference"])
    ap.add_argument("--workload", default="c4", choices=["c1", "c2", "c3", "c4"])
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other prefill workloads")
    ap.add_argument("--fused-q", action="store_true",
                    help="rotate and quantise Q inside the attention kernel (sage_attn_fwd_q16)")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the paged-decode measurement and print its object")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_traffic(workload):
    """DRAM bytes per attn_fwd launch on `workload` from the committed ncu
    summary, if the kernel source is unchanged since the capture (else None)."""
    import hashlib
    import re
    prof = os.path.join(ROOT, "profiles", "attn_fwd_%s.md" % workload)
    if not os.path.exists(prof):
        return None
    text = open(prof).read()
    m_sha = re.search(r"^source_sha256: ([0-9a-f]+)", text, flags=re.M)
    m_b = re.search(r"^dram_bytes_per_launch: (\d+)", text, flags=re.M)
    if not m_sha or not m_b:
        return None
    src = b"".join(open(os.path.join(ROOT, "quantized_attention_smoothing_b200", "csrc", f), "rb").read()
                   for f in ("attn_fwd.cu", "sage_ptx.cuh"))
    if hashlib.sha256(src).hexdigest()[:len(m_sha.group(1))] != m_sha.group(1):
        return None
    return int(m_b.group(1))


def pct(sorted_vals, q):
    """q-th percentile (nearest rank) of an ascending list."""
    i = min(len(sorted_vals) - 1, max(0, int(math.ceil(q / 100.0 * len(sorted_vals))) - 1))
    return sorted_vals[i]


def rank_max(x, world, device):
    """Max of a per-rank scalar over all ranks of the default process group
    (identity for a single rank): every multi-rank time in the JSON line is
    the slowest rank's."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(ops_per_step, steps, elapsed_ms):
    """Whole-job TOPS: `ops_per_step` (the work of all ranks together) per
    step, `steps` steps in `elapsed_ms` (the slowest rank's time)."""
    return ops_per_step * steps / (elapsed_ms * 1e-3) / 1e12


def kv_head_range(Hk, world, rank):
    """The contiguous kv heads [lo, hi) of `rank` when the Hk kv heads are
    split over `world` ranks as evenly as possible (each rank also takes the
    query heads that share those kv heads)."""
    if world > Hk:
        raise ValueError("cannot split %d kv heads over %d ranks" % (Hk, world))
    return Hk * rank // world, Hk * (rank + 1) // world


def shard_heads(cfg, q, k, v, world, rank):
    """This rank's part of a prefill workload: its kv-head range and their
    query heads (views, no copy)."""
    if world == 1:
        return cfg, q, k, v
    group = cfg["H"] // cfg["Hk"]
    lo, hi = kv_head_range(cfg["Hk"], world, rank)
    return (dict(cfg, H=(hi - lo) * group, Hk=hi - lo), q[:, lo * group:hi * group], k[:, lo:hi],
            v[:, lo:hi])


def work_ops(cfg):
    ops = 4.0 * cfg["B"] * cfg["H"] * cfg["L"] * cfg["L"] * cfg["D"]
    return ops / 2 if cfg["causal"] else ops


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, enabled=True):
        self.gpu = gpu_index
        self.proc = None
        self.enabled = enabled
        self.path = None

    def __enter__(self):
        if self.enabled:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
                time.sleep(0.3)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows),
                "samples": len(rows), "reasons": reasons}


def cpu_baseline(cfg, seconds):
    """The oracle as it stands, on the host cores, on a bounded sample of the
    workload: the quantisation of every token of a set of heads (one head per
    thread) and the attention of a seeded set of query rows of each, the
    number of rows sized to about `seconds` of wall time. The two parts are
    timed apart and scaled to the whole workload (quantisation by heads,
    attention by heads and by the keys the sampled rows see), and the value
    is the workload's ops over that whole-workload time."""
    import numpy as np

    import oracle
    import workloads

    cores = os.cpu_count() or 1
    _, q, k, v = workloads.make_prefill_config(cfg["key"])
    b = workloads.bits_u16
    heads = min(cfg["H"], cores)
    qb, kb, vb = b(q)[:1, :heads], b(k)[:1, :heads], b(v)[:1, :heads]
    L = cfg["L"]
    rng = np.random.default_rng(cfg["H"] * 7 + L)

    t = time.perf_counter()
    qk = oracle.quant_qk(qb, kb, cfg["blk_q"], cfg["blk_k"], threads=cores)
    v8t, vs = oracle.quant_v(vb, threads=cores)
    t_quant = time.perf_counter() - t

    def keys_seen(rows):
        return float(np.sum(np.minimum(rows + 1, L))) if cfg["causal"] else float(len(rows)) * L

    def run(nrows):
        rows = np.sort(rng.choice(L, size=nrows, replace=False)).astype(np.int32)
        t = time.perf_counter()
        oracle.attn(qk["q8"], qk["qs"], qk["k8"], qk["ks"], v8t, vs, L, L, cfg["blk_q"],
                    cfg["blk_k"], cfg["softmax_scale"], cfg["causal"], rows=rows, threads=cores)
        return time.perf_counter() - t, rows

    nrows = min(L, 16)
    t_attn, rows = run(nrows)
    budget = max(0.0, seconds - t_quant)
    if nrows < L and t_attn < budget / 4:
        nrows = int(min(L, max(nrows, nrows * budget / max(t_attn, 1e-3))))
        t_attn, rows = run(nrows)
    all_keys = float(L) * (L + 1) / 2 if cfg["causal"] else float(L) * L
    # whole workload on the same threads: the heads in waves of `heads`, each
    # wave's quantisation as measured, its attention scaled by keys
    waves = cfg["B"] * cfg["H"] / float(heads)
    t_whole = waves * (t_quant + t_attn * all_keys / keys_seen(rows))
    value = work_ops(cfg) / t_whole / 1e12
    return {"value": value, "unit": UNIT, "cores": min(cores, heads), "kind": "oracle",
            "sample": "B=1, %d of %d heads, one per thread: quantise every token of Q/K/V "
                      "(%.1f s), attention of %d seeded query rows of %d (%.1f s); scaled to the "
                      "whole workload (%d x %d heads): %.0f s"
                      % (heads, cfg["H"], t_quant, nrows, L, t_attn, cfg["B"], cfg["H"], t_whole)}


def bench_decode(sage, torch, stream, copies=8, reps=50, key="c5"):
    """Paged decode on one of the decode workloads: the MTP4 / GQA16 /
    window-4096 one over the FP8 cache (head size 128, or 64 with key
    "c5_d64") or over an MXFP4 cache ("c5_mx"), and the batch-32 / ctx-32k /
    T 1 one over either cache ("c7", "c7_mx"). One call = the split kernel
    and the merge kernel; cache copies rotate so that the working set
    exceeds L2 (8, or 2 when one copy is larger than L2); calls are captured
    in a CUDA graph and replayed."""
    import workloads
    cfg, d = workloads.make_decode_config(key)
    mx = cfg.get("kv_format") == "mxfp4"
    B, T, H, D = d["q"].shape
    Hk, page = d["k_cache"].shape[1], d["k_cache"].shape[2]
    h = sage.Hadamard(D)
    q = d["q"].cuda()
    tabs = [d[x].cuda() for x in ("page_table", "ctx_lens")]
    copy_bytes = sum(d[x].numel() * d[x].element_size() for x in ("k_cache", "v_cache", "k_scale", "v_scale"))
    if copy_bytes > 128 << 20:
        copies = 2
    caches = [[d[x].cuda() for x in ("k_cache", "v_cache", "k_scale", "v_scale")]
              for _ in range(copies)]
    run = sage.sage_attn_decode_mxfp4 if mx else sage.sage_attn_decode
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros((max(16, sage.sage_attn_decode_workspace(B, T, H, Hk, D, cfg["window"])),),
                     dtype=torch.uint8, device="cuda")

    def call(i):
        kc, vc, ksc, vsc = caches[i % copies]
        # torch's current stream: the side stream below, or the capture stream
        run(h, q, kc, vc, ksc, vsc, tabs[0], tabs[1], page, d["num_pages"], cfg["window"],
            cfg["softmax_scale"], out, ws, None)

    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        for i in range(copies):
            call(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            call(i)
    # replay for a fifth of a second first: a GPU that was idle runs its
    # first milliseconds at a low clock
    t_end = time.time() + 0.2
    while time.time() < t_end:
        g.replay()
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(5):
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / reps)
    if sage.sage_device_error(stream) != sage.SAGE_OK:
        raise RuntimeError("device error during decode timing")
    ms = statistics.median(times)
    times.sort()
    ctx = d["ctx_lens"].tolist()
    keys = sum(min(c, cfg["window"] + T - 1) for c in ctx)
    # K and V rows of the keys read: D e4m3 codes and one fp32 scale each, or
    # (MXFP4) D / 2 code bytes and D / 32 e8m0 scale bytes each
    row = (D // 2 + D // 32) if mx else (D + 4)
    algo = keys * Hk * 2 * row + 2 * q.numel() * 2 + tabs[0].numel() * 4 + tabs[1].numel() * 4
    pk, pk_src = peaks()
    gbs = algo / (ms * 1e-3) / 1e9
    del g
    return {"workload": cfg["name"], "us_per_call": ms * 1e3,
            "us_per_call_p10_p50_p90": [pct(times, 10) * 1e3, pct(times, 50) * 1e3, pct(times, 90) * 1e3],
            "algorithmic_bytes": algo,
            "achieved": gbs, "unit": "GB/s", "peak": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"],
            "peak_source": pk_src + " copy bandwidth (burst)",
            "launches_per_call": 2 if sage.sage_attn_decode_workspace(B, T, H, Hk, D, cfg["window"]) > 0 else 1,
            "kv_format": "mxfp4" if mx else "fp8",
            "timing": "median of 5 replays of a CUDA graph of %d calls over %d rotating cache copies"
                      % (reps, copies)}


class Prefill:
    """Device-resident input sets of one prefill workload (this rank's heads)
    and the timed loops over them."""

    def __init__(self, sage, torch, cfg, q, k, v, fused_q=False):
        self.sage, self.torch, self.cfg, self.fused_q = sage, torch, cfg, fused_q
        B, H, Hk, L, D = cfg["B"], cfg["H"], cfg["Hk"], cfg["L"], cfg["D"]
        self.h = sage.Hadamard(D)
        self.q_cpu, self.k_cpu, self.v_cpu = q, k, v
        in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
        self.set_bytes = in_bytes + 2 * q.numel() * 2
        # rotate enough input sets that consecutive steps never find their
        # inputs in the 126 MB L2
        n_sets = max(2, int(math.ceil(2 * L2_BYTES / max(self.set_bytes, 1))))
        self.sets = []
        for _ in range(n_sets):
            qs, ks, vs_ = q.cuda(), k.cuda(), v.cuda()          # [B,H,L,D] views of [B,L,H,D]
            bufs = sage.QuantBuffers(B, H, Hk, L, L, D, cfg["blk_q"], cfg["blk_k"])
            out = torch.empty((B, L, H, D), dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)
            self.sets.append((qs, ks, vs_, bufs, out))

    def quantise(self, i, stream):
        qs, ks, vs_, bufs, _ = self.sets[i % len(self.sets)]
        c = self.cfg
        self.sage.quantise(self.h, None if self.fused_q else qs, ks, vs_, c["blk_q"], c["blk_k"],
                           bufs, stream)

    def attention(self, i, stream):
        qs, _, _, bufs, out = self.sets[i % len(self.sets)]
        c = self.cfg
        if self.fused_q:
            self.sage.sage_attn_fwd_q16(self.h, qs, c["blk_q"], bufs.k8, bufs.k_scale, bufs.v8_t,
                                        bufs.v_scale, c["Hk"], c["L"], c["blk_k"], c["softmax_scale"],
                                        c["causal"], out, None, stream)
        else:
            self.sage.sage_attn_fwd(bufs.q8, bufs.q_scale, bufs.k8, bufs.k_scale, bufs.v8_t,
                                    bufs.v_scale, c["B"], c["H"], c["Hk"], c["L"], c["L"], c["D"],
                                    c["blk_q"], c["blk_k"], c["softmax_scale"], c["causal"], out,
                                    None, stream)

    def timed_steps(self, steps, warmup, stream, barrier, clocks=None):
        """Whole steps (quantise + attention): total elapsed ms and the
        per-step attention launch times (ms), CUDA events on `stream`."""
        torch = self.torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(warmup):
            self.quantise(i, stream)
            self.attention(i, stream)
        torch.cuda.synchronize()
        if self.sage.sage_device_error(stream) != self.sage.SAGE_OK:
            raise RuntimeError("device error during warm-up")
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        cm = clocks if clocks is not None else _NullCtx()
        with cm:
            barrier()
            torch.cuda.synchronize()
            t0.record(stream)
            for i in range(steps):
                self.quantise(i, stream)
                ev[i][0].record(stream)
                self.attention(i, stream)
                ev[i][1].record(stream)
            t1.record(stream)
            torch.cuda.synchronize()
            barrier()
        if self.sage.sage_device_error(stream) != self.sage.SAGE_OK:
            raise RuntimeError("device error during the timed steps")
        return t0.elapsed_time(t1), sorted(a.elapsed_time(b) for a, b in ev)

    def timed_quant(self, steps, warmup, stream):
        """The quantisation call alone (its launches), microseconds per call."""
        torch = self.torch
        qev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for i in range(warmup):
            self.quantise(i, stream)
        torch.cuda.synchronize()
        for i in range(steps):
            qev[i][0].record(stream)
            self.quantise(i, stream)
            qev[i][1].record(stream)
        torch.cuda.synchronize()
        if self.sage.sage_device_error(stream) != self.sage.SAGE_OK:
            raise RuntimeError("device error while timing the quantisation")
        return sorted(a.elapsed_time(b) * 1e3 for a, b in qev)


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def quant_object(pf, q_times, pk, pk_src):
    q_us = statistics.median(q_times)
    q_bytes = 3 * ((0 if pf.fused_q else pf.q_cpu.numel()) + pf.k_cpu.numel() + pf.v_cpu.numel())
    gbs = q_bytes / (q_us * 1e-6) / 1e9
    return {"us_per_call": q_us,
            "us_p10_p50_p90": [pct(q_times, 10), pct(q_times, 50), pct(q_times, 90)],
            "algorithmic_bytes": q_bytes, "achieved": gbs, "unit": "GB/s",
            "peak": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"],
            "peak_source": pk_src + " copy bandwidth (burst)",
            "bytes_rule": "2 B read + 1 B written per element of each quantised tensor; the "
                          "statistics pass re-reads K and V (not counted)",
            "launches_per_call": 4 if pf.fused_q else 2}


def roofline_object(ops, attn_times, pk, pk_src, traffic):
    peak_tops = pk["bf16_tflops"] * INT8_OVER_BF16
    attn_ms = statistics.mean(attn_times)
    achieved = ops / (attn_ms * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": "attn_fwd", "achieved": achieved, "peak": peak_tops,
            "unit": "TFLOP/s", "frac": achieved / peak_tops, "traffic": traffic,
            "peak_source": "%s bf16 burst x %.0f (INT8/FP8 : BF16 nominal)" % (pk_src, INT8_OVER_BF16),
            "frac_of_sustained": achieved / (pk["bf16_tflops_sustained"] * INT8_OVER_BF16),
            "attn_ms": attn_ms,
            "attn_ms_p10_p50_p90": [pct(attn_times, 10), pct(attn_times, 50), pct(attn_times, 90)]}


def bench_mx(sage, torch, key, steps, warmup, stream, pk, pk_src):
    """The MXFP4 variant on one prefill workload: a step is sage_quant_qk_mx
    + sage_quant_v + sage_attn_fwd_mx on inputs resident in HBM (rotating sets
    larger than L2). The attention's roofline is the mixed peak of its work:
    QK^T in FP4 (4 x the bf16 peak, nominal ratio), PV in FP8 (2 x)."""
    import workloads
    cfg, q, k, v = workloads.make_prefill_config(key)
    B, H, Hk, L, D = cfg["B"], cfg["H"], cfg["Hk"], cfg["L"], cfg["D"]
    h = sage.Hadamard(D)
    set_bytes = sum(t.numel() * t.element_size() for t in (q, k, v)) + 2 * q.numel() * 2
    sets = []
    for _ in range(max(2, int(math.ceil(2 * L2_BYTES / set_bytes)))):
        out = torch.empty((B, L, H, D), dtype=torch.bfloat16, device="cuda").permute(0, 2, 1, 3)
        sets.append((q.cuda(), k.cuda(), v.cuda(), sage.MxBuffers(B, H, Hk, L, L, D), out))

    def quant(i):
        qs, ks, vs_, bf, _ = sets[i % len(sets)]
        sage.sage_quant_qk_mx(h, qs, ks, bf.q4, bf.q_sf, bf.k4, bf.k_sf, bf.k_mean, bf.ws, stream)
        sage.sage_quant_v(vs_, bf.v8_t, bf.v_scale, bf.ws_v, stream)

    def attn(i):
        _, _, _, bf, out = sets[i % len(sets)]
        sage.sage_attn_fwd_mx(bf.q4, bf.q_sf, bf.k4, bf.k_sf, bf.v8_t, bf.v_scale, B, H, Hk, L, L, D,
                              cfg["softmax_scale"], cfg["causal"], out, None, stream)

    for i in range(warmup):
        quant(i)
        attn(i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        quant(i)
        ev[i][1].record(stream)
        attn(i)
        ev[i][2].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if sage.sage_device_error(stream) != sage.SAGE_OK:
        raise RuntimeError("device error in the MXFP4 timing")
    ms = t0.elapsed_time(t1) / steps
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    q_us = statistics.median(e[0].elapsed_time(e[1]) for e in ev) * 1e3
    ops = work_ops(cfg)
    p8 = pk["bf16_tflops"] * INT8_OVER_BF16
    mixed = 2.0 / (1.0 / (2.0 * p8) + 1.0 / p8)       # half the ops at the FP4 rate, half at FP8
    achieved = ops / (attn_ms * 1e-3) / 1e12
    q_bytes = (q.numel() + k.numel()) * (2 + 0.5 + 1.0 / 32) + v.numel() * 3
    del sets
    torch.cuda.empty_cache()
    return {"workload": cfg["name"], "value": ops / (ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "steps": steps,
            "roofline": {"bound": "tensor", "kernel": "attn_mx", "achieved": achieved, "peak": mixed,
                         "unit": "TFLOP/s", "frac": achieved / mixed, "attn_ms": attn_ms,
                         "peak_source": "%s bf16 burst x 4 for the FP4 QK half, x 2 for the FP8 PV half "
                                        "(nominal ratios)" % pk_src},
            "quant": {"us_per_call": q_us, "algorithmic_bytes": q_bytes,
                      "achieved": q_bytes / (q_us * 1e-6) / 1e9, "unit": "GB/s", "peak": pk["hbm_gbs"],
                      "frac": q_bytes / (q_us * 1e-6) / 1e9 / pk["hbm_gbs"],
                      "bytes_rule": "Q, K: 2 B read + 0.5 B codes + 1/32 B scale per element; V: 2 + 1",
                      "launches_per_call": 3}}


def run_reference(args):
    import workloads
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = dict(workloads.PREFILL[args.workload], key=args.workload)
    vals = []
    cb = None
    for _ in range(max(1, args.steps)):
        cb = cpu_baseline(cfg, min(args.cpu_seconds, 20.0))
        vals.append(cb["value"])
        if len(vals) >= 3:
            break
    value = statistics.median(vals)
    cb["value"] = value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": len(vals), "warmup": 0,
        "ms_per_step": work_ops(dict(cfg)) / (value * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "int8+e4m3",
        "data": "synthetic", "config": {"workload": cfg["name"], "B": cfg["B"], "H": cfg["H"],
                                        "L": cfg["L"], "D": cfg["D"]},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def measure_e2e(sage, torch, pf, steps, stream, barrier, max_over_ranks, ops_all):
    """End to end through the public API: pinned host inputs -> device ->
    quantise + attention -> result back to pinned host memory, every step.
    Steps are pipelined over two device buffer pairs and three streams
    (host->device copies, compute, device->host copies): the inputs of step
    i + 1 travel while step i computes and step i - 1's result comes back."""
    c = pf.cfg
    B, H, L, D = c["B"], c["H"], c["L"], c["D"]
    q, k, v = pf.q_cpu, pf.k_cpu, pf.v_cpu
    qh = q.permute(0, 2, 1, 3).contiguous().pin_memory()      # [B, L, H, D] host buffers
    kh = k.permute(0, 2, 1, 3).contiguous().pin_memory()
    vh = v.permute(0, 2, 1, 3).contiguous().pin_memory()
    oh = [torch.empty((B, L, H, D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dev_in = [[torch.empty_like(x, device="cuda") for x in (qh, kh, vh)] for _ in range(2)]
    dev_out = [torch.empty((B, L, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ebufs = pf.sets[0][3]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    n_e2e = steps + 2
    ev_in = [torch.cuda.Event() for _ in range(n_e2e)]
    ev_comp = [torch.cuda.Event() for _ in range(n_e2e)]
    ev_out = [torch.cuda.Event() for _ in range(n_e2e)]

    def e2e_step(i):
        j = i % 2
        qd, kd, vd = dev_in[j]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[i - 2])        # step i - 2 has read these inputs
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_out[i - 2])           # step i - 2's result has left dev_out[j]
        sage.sage_attention(pf.h, qd.permute(0, 2, 1, 3), kd.permute(0, 2, 1, 3),
                            vd.permute(0, 2, 1, 3), c["blk_q"], c["blk_k"], c["softmax_scale"],
                            c["causal"], out=dev_out[j].permute(0, 2, 1, 3), bufs=ebufs,
                            stream=stream)
        ev_comp[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[i])
            oh[j].copy_(dev_out[j], non_blocking=True)
            ev_out[i].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        e2e_step(i)
    stream.wait_event(ev_out[steps - 1])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    if sage.sage_device_error(stream) != sage.SAGE_OK:
        raise RuntimeError("device error during the end-to-end steps")
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    return {"value": job_value(ops_all, steps, e2e_ms), "unit": UNIT,
            "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in (qh, kh, vh)),
            "d2h_bytes_per_step": oh[0].numel() * oh[0].element_size(),
            "ms_per_step": e2e_ms / steps,
            "pipeline": "h2d, compute and d2h on three streams over two buffer pairs"}


def run_sage(args):
    import torch
    import torch.distributed as dist

    import quantized_attention_smoothing_b200 as sage
    import workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return rank_max(x, world, "cuda")

    pk, pk_src = peaks()
    stream = torch.cuda.current_stream()
    full_cfg = dict(workloads.PREFILL[args.workload], key=args.workload)
    _, q, k, v = workloads.make_prefill_config(args.workload)
    cfg, q, k, v = shard_heads(full_cfg, q, k, v, world, rank)
    ops_all = work_ops(full_cfg)                 # the whole workload, all ranks together
    pf = Prefill(sage, torch, cfg, q, k, v, fused_q=args.fused_q)

    clk = ClockSampler(local, enabled=not args.no_clocks)
    elapsed_local, attn_times = pf.timed_steps(args.steps, args.warmup, stream, barrier, clocks=clk)
    elapsed_ms = max_over_ranks(elapsed_local)
    value = job_value(ops_all, args.steps, elapsed_ms)
    roofline = roofline_object(work_ops(cfg), attn_times, pk, pk_src,
                               attn_traffic(cfg["name"]) if world == 1 else None)
    e2e = measure_e2e(sage, torch, pf, args.e2e_steps, stream, barrier, max_over_ranks, ops_all)
    quant = quant_object(pf, pf.timed_quant(args.steps, args.warmup, stream), pk, pk_src)
    set_desc = "%d rotating input sets of %.0f MB (> 126 MB L2 between uses)" % (len(pf.sets),
                                                                                  pf.set_bytes / 1e6)
    del pf
    torch.cuda.empty_cache()

    # the other prefill workloads (one GPU only): each with its own step
    # throughput, attention roofline and quantisation bandwidth
    extra = {}
    if world == 1 and not args.no_extra:
        for key in ("c2", "c3", "c4"):
            if key == args.workload:
                continue
            ecfg = dict(workloads.PREFILL[key], key=key)
            _, eq, ek, ev_ = workloads.make_prefill_config(key)
            epf = Prefill(sage, torch, ecfg, eq, ek, ev_, fused_q=args.fused_q)
            esteps = max(args.steps, 20)
            el, at = epf.timed_steps(esteps, max(args.warmup, 3), stream, barrier)
            eops = work_ops(ecfg)
            extra[key] = {
                "workload": ecfg["name"], "causal": ecfg["causal"],
                "value": job_value(eops, esteps, el), "unit": UNIT, "ms_per_step": el / esteps,
                "steps": esteps,
                "roofline": roofline_object(eops, at, pk, pk_src, attn_traffic(ecfg["name"])),
                "quant": quant_object(epf, epf.timed_quant(esteps, 3, stream), pk, pk_src),
                "l2": "%d rotating input sets of %.0f MB" % (len(epf.sets), epf.set_bytes / 1e6)}
            del epf
            torch.cuda.empty_cache()

    mx = {}
    if world == 1 and not args.no_extra:
        for key in ("c4", "c2"):
            mx[key] = bench_mx(sage, torch, key, max(args.steps, 10) if key == "c4" else 40,
                               max(args.warmup, 3), stream, pk, pk_src)

    dec = None if args.no_decode else bench_decode(sage, torch, stream)
    dec64 = None if args.no_decode or world > 1 else bench_decode(sage, torch, stream, key="c5_d64")
    dec_mx = None if args.no_decode or world > 1 else bench_decode(sage, torch, stream, key="c5_mx")
    dec_long = None
    if not args.no_decode and world == 1:
        dec_long = {"fp8": bench_decode(sage, torch, stream, key="c7"),
                    "mxfp4": bench_decode(sage, torch, stream, key="c7_mx")}

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(full_cfg, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "int8+e4m3", "data": "synthetic",
            "config": {"workload": full_cfg["name"], "B": full_cfg["B"], "H": full_cfg["H"],
                       "L": full_cfg["L"], "D": full_cfg["D"], "blk_q": full_cfg["blk_q"],
                       "blk_k": full_cfg["blk_k"], "causal": full_cfg["causal"],
                       "parallelism": ("kv-head shards over %d ranks" % world) if world > 1 else "single",
                       "l2": set_desc},
            "roofline": roofline,
            "cpu_baseline": cb,
            "e2e": e2e,
            "quant": quant,
            "configs": extra,
            "mxfp4": mx,
            "decode": dec,
            "decode_d64": dec64,
            "decode_mxfp4": dec_mx,
            "decode_long": dec_long,
            "gpu_launches": (5 if args.fused_q else 3) * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.decode_only:
        import torch
        import quantized_attention_smoothing_b200 as sage
        s = torch.cuda.current_stream()
        print(json.dumps({k: bench_decode(sage, torch, s, key=k) for k in ("c5", "c5_d64", "c5_mx", "c7", "c7_mx")}))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_sage(args)


if __name__ == "__main__":
    main()

"""Benchmark of the attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  1. prefill forward (fa_fwd): causal, B=4, S=4096, H=32, d=64, fp16
  2. paged split-KV decode (fa_fwd_kvcache) + LSE combine: B=64, Sq=1, H=32,
     Hkv=8, d=128, bf16, cache lengths U{1K..32K}, pages of 256, random
     block_table, num_splits (default 16)
Reported: ``value`` = prefill TFLOPS (4*d*sum of allowed (i, j) pairs / time);
``decode`` = KV-cache GB/s (valid cache bytes + q/out/lse/block_table / time).
Both are also given as fractions of the measured B200 peaks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--num-splits S] [--no-cpu-baseline] [--no-e2e]
For N > 1 launch under torch.distributed.run; every rank runs an independent
replica on its own seeded data (weak scaling, no collective on the data path);
the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

PREFILL = dict(B=4, S=4096, H=32, Hkv=32, d=64, dtype="fp16", causal=True)
DECODE = dict(B=64, Sq=1, H=32, Hkv=8, d=128, dtype="bf16", lo=1024, hi=32768, page=256)
METRIC = "attn fwd TFLOPS (causal prefill) & decode KV GB/s, % of B200 roofline"


def causal_pairs(Sq: int, Sk: int) -> int:
    """Number of allowed (i, j) pairs of a bottom-right causal mask: row i sees
    keys 0 .. i + Sk - Sq."""
    off = Sk - Sq
    return sum(min(Sk, max(0, i + off + 1)) for i in range(Sq))


def prefill_flops(c=PREFILL) -> float:
    return 4.0 * c["d"] * c["B"] * c["H"] * causal_pairs(c["S"], c["S"])


def profiled_traffic(profile: str, sources) -> int | None:
    """DRAM bytes per launch from a committed ncu summary, or None when the kernel's
    sources no longer hash to the value recorded with the capture."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_t = re.search(r"^traffic_bytes_per_launch: (\d+)", text, re.M)
    m_h = re.search(r"^source_sha256_16: ([0-9a-f]+)", text, re.M)
    if not (m_t and m_h):
        return None
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "io_aware_online_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return int(m_t.group(1)) if h.hexdigest()[:16] == m_h.group(1) else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk["hbm_gbs"], pk["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"]}
        busy = [m for m in mhz if m > 0.5 * max(mhz)] or mhz
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


def dist_setup(gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        if world > 1 or gpus > 1:
            raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}: launch with torch.distributed.run")
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- workloads
def make_prefill(rank, dev):
    c = PREFILL
    dt = synth.DTYPES[c["dtype"]]
    q, k, v = synth.dense(c["B"], c["S"], c["S"], c["H"], c["Hkv"], c["d"], dt,
                          seed=1003 + 100 * rank)
    return q, k, v


def make_decode(rank, dev):
    c = DECODE
    dt = synth.DTYPES[c["dtype"]]
    lens = synth.varlen_lengths(c["B"], c["lo"], c["hi"], seed=1005 + 100 * rank)
    kp, vp, bt, cs = synth.paged_cache(lens, c["page"], c["Hkv"], c["d"], dt,
                                       seed=1005 + 100 * rank, device=dev)
    q = synth.randn((c["B"], c["Sq"], c["H"], c["d"]), dt,
                    torch.Generator().manual_seed(1006 + 100 * rank))
    return q, kp, vp, bt, cs, lens


def decode_bytes(lens, splits):
    c = DECODE
    kv = sum(lens) * c["Hkv"] * c["d"] * 2 * 2               # K and V, valid tokens only
    io = c["B"] * c["Sq"] * c["H"] * c["d"] * 2 * 2          # q in, out
    io += c["B"] * c["H"] * c["Sq"] * 4                       # lse
    bt = sum((L + c["page"] - 1) // c["page"] for L in lens) * 4 + c["B"] * 4
    return kv + io + bt


def run_ours(args, rank, world, local):
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build as fa_build
    fa_build.build()
    fa.load()
    dev = torch.device("cuda", local)
    hbm_peak, tflops_peak, peak_src = load_peaks()

    q, k, v = make_prefill(rank, dev)
    qd_, kd_, vd_ = q.to(dev), k.to(dev), v.to(dev)
    out_p = torch.empty_like(qd_)
    lse_p = torch.empty((PREFILL["B"], PREFILL["H"], PREFILL["S"]), dtype=torch.float32, device=dev)
    if args.only == "prefill":        # keep the decode pool tiny when it is not timed
        DECODE.update(B=2, lo=1024, hi=1024)
    dq, kp, vp, bt, cs, lens = make_decode(rank, dev)
    dq_d, bt_d, cs_d = dq.to(dev), bt.to(dev), cs.to(dev)
    splits = args.num_splits
    c = DECODE
    ws_bytes = fa.fa_kvcache_workspace_size(c["B"], c["Sq"], c["H"], c["Hkv"], c["d"],
                                            bt.shape[1] * c["page"], c["page"], splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    out_d = torch.empty_like(dq_d)
    lse_d = torch.empty((c["B"], c["H"], c["Sq"]), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    do_pre = args.only in ("all", "prefill")
    do_dec = args.only in ("all", "decode")

    def prefill():
        if do_pre:
            fa.fa_fwd(qd_, kd_, vd_, out=out_p, lse=lse_p, causal=True, stream=stream)

    def decode():
        if do_dec:
            fa.fa_fwd_kvcache(dq_d, kp, vp, cache_seqlens=cs_d, block_table=bt_d, causal=True,
                              num_splits=splits, out=out_d, lse=lse_d, workspace=ws,
                              stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        prefill()
        decode()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        for s in range(K):
            flush.zero_()                       # L2 flushed between steps (not timed)
            ev[s][0].record(stream)
            prefill()
            ev[s][1].record(stream)
            decode()
            ev[s][2].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    t_pre = sum(e[0].elapsed_time(e[1]) for e in ev) / K      # ms per launch
    t_dec = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    t_pre = max(t_pre, 1e-9)
    t_dec = max(t_dec, 1e-9)
    t_step = t_pre + t_dec
    t_pre_max = max_over_ranks(t_pre, world)
    t_dec_max = max_over_ranks(t_dec, world)
    t_step_max = max_over_ranks(t_step, world)
    assert fa.fa_device_status(clear=True) == 0, "device status flags raised during the bench"

    flops = prefill_flops()
    tflops = flops / (t_pre_max * 1e-3) / 1e12 * world
    dbytes = decode_bytes(lens, splits)
    gbs = dbytes / (t_dec_max * 1e-3) / 1e9 * world
    res = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(t_step_max, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16 (prefill), bf16 (decode); fp32 accumulate",
        "data": "synthetic (seeded N(0,1))",
        "config": {
            "workload": (f"causal prefill B={PREFILL['B']} S={PREFILL['S']} H={PREFILL['H']} "
                         f"d={PREFILL['d']} {PREFILL['dtype']} + paged split-KV decode "
                         f"B={DECODE['B']} H=32 Hkv=8 d=128 bf16 cache U{{1K..32K}} page 256"),
            "prefill": dict(PREFILL, ms=round(t_pre_max, 4), flop=flops),
            "decode": dict(DECODE, num_splits=splits, sum_cache_tokens=int(sum(lens)),
                           ms=round(t_dec_max, 4), bytes=dbytes),
            "l2": "flushed between steps (256 MiB write, untimed)",
            "parallelism": f"dp{world} (independent replicas)",
        },
        "decode": {
            "value": round(gbs, 1), "unit": "GB/s", "ms": round(t_dec_max, 4),
            "roofline": {"bound": "hbm", "achieved": round(dbytes / (t_dec_max * 1e-3) / 1e9, 1),
                         "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(dbytes / (t_dec_max * 1e-3) / 1e9 / hbm_peak, 4),
                         "traffic": (profiled_traffic("decode_kernel_paged_B8.md",
                                                      ["decode_kernel.cuh", "decode.cu",
                                                       "sm100.cuh", "fa_internal.h"])
                                     if (DECODE["B"] == 64 and splits == 16) else None),
                         "peak_source": peak_src},
        },
        "roofline": {"bound": "tensor", "achieved": round(flops / (t_pre * 1e-3) / 1e12, 2),
                     "peak": tflops_peak, "unit": "TFLOP/s",
                     "frac": round(flops / (t_pre * 1e-3) / 1e12 / tflops_peak, 4),
                     "traffic": (profiled_traffic("fwd_kernel_d64_causal_B4_S4096.md",
                                                  ["fwd_kernel.cuh", "fwd_launch.cuh",
                                                   "sm100.cuh", "fa_internal.h"])
                                 if (PREFILL["d"] == 64 and PREFILL["S"] == 4096) else None),
                     "kernel": f"fwd_kernel<{PREFILL['d']}, {PREFILL['dtype']}, causal>",
                     "peak_source": f"{peak_src} bf16 burst (fp16 dense rate equals bf16)"},
        "gpu_launches": K * ((1 if do_pre else 0) + ((2 if splits > 1 else 1) if do_dec else 0)),
        "clocks": clk.summary(),
    }
    if not args.no_e2e:
        res["e2e"] = e2e_prefill(fa, q, k, v, dev, stream, flops, world)
    return res


# Workloads of the cache-update rows (not part of the default step): a 2048-token
# chunk appended after 6144 cached tokens and attended causally (chunked prefill),
# and a whole 8192-token prompt written into an empty paged cache (append).
CHUNKED = dict(B=4, cached=6144, chunk=2048, H=32, Hkv=8, d=128, dtype="bf16", page=256)
APPEND = dict(B=4, S_new=8192, Hkv=8, d=128, dtype="bf16", page=256)
# 8-bit forward (fa_fwd_fp8): the d=128 prefill point, E4M3 inputs cast from N(0,1)
FP8 = dict(B=4, S=8192, H=32, Hkv=32, d=128, dtype="e4m3", causal=True)


# backward (fa_bwd): the d=128 causal prefill point
BWD = dict(B=4, S=4096, H=32, Hkv=32, d=128, dtype="bf16", causal=True)


def run_bwd(args, rank, world, local):
    """--only bwd: time fa_bwd (D pre-pass + dK/dV + dQ kernels).  Algorithmic work:
    the five products of the backward (S, dP, dV, dK, dQ), 10 d FLOPs per allowed
    (query, key) pair, i.e. 2.5x the forward's."""
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build as fa_build
    fa_build.build()
    fa.load()
    dev = torch.device("cuda", local)
    hbm_peak, tflops_peak, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    c = BWD
    dt = synth.DTYPES[c["dtype"]]
    gen = torch.Generator(device=dev).manual_seed(3200 + rank)
    shp_q = (c["B"], c["S"], c["H"], c["d"])
    shp_k = (c["B"], c["S"], c["Hkv"], c["d"])
    q = torch.randn(shp_q, generator=gen, device=dev).to(dt)
    k = torch.randn(shp_k, generator=gen, device=dev).to(dt)
    v = torch.randn(shp_k, generator=gen, device=dev).to(dt)
    do = torch.randn(shp_q, generator=gen, device=dev).to(dt)
    out, lse = fa.fa_fwd(q, k, v, causal=True, stream=stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.load().fa_bwd_workspace_size(c["B"], c["S"], c["H"]), dtype=torch.uint8,
                     device=dev)
    work = 10.0 * c["d"] * c["B"] * c["H"] * causal_pairs(c["S"], c["S"])

    def call():
        fa.fa_bwd(do, q, k, v, out, lse, causal=True, dq=dq, dk=dk, dv=dv, workspace=ws,
                  stream=stream)
    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world)
    achieved = work / (ms * 1e-3) / 1e12
    return {"metric": "attn bwd TFLOPS (causal, dQ dK dV)", "value": round(achieved * world, 2),
            "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": c["dtype"], "data": "synthetic (seeded N(0,1))",
            "config": {"workload": "bwd", **c, "l2": "flushed between steps (256 MiB write, "
                       "untimed)", "parallelism": f"dp{world} (independent replicas)"},
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": tflops_peak,
                         "unit": "TFLOP/s", "frac": round(achieved / tflops_peak, 4),
                         "traffic": None,
                         "kernel": "bwd_dot_kernel + bwd_dkdv_kernel + bwd_dq_kernel <128, bf16>",
                         "peak_source": peak_src},
            "gpu_launches": 3 * K, "clocks": clk.summary()}


# TFLOPS vs sequence length of the causal prefill (B=4, H=Hkv=32)
SWEEP = dict(B=4, H=32, d=(64, 128), S=(512, 1024, 2048, 4096, 8192, 16384),
             dtype=("fp16", "bf16"))


def run_sweep(args, rank, world, local):
    """--only sweep: the causal prefill's TFLOPS over head dims, sequence lengths
    and 16-bit types; one JSON line whose value is the largest point (d=128,
    S=16384, bf16) and whose ``curve`` holds every point."""
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build as fa_build
    fa_build.build()
    fa.load()
    dev = torch.device("cuda", local)
    _, tflops_peak, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    c = SWEEP
    K = min(args.steps, 10)
    curve = []
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        for d in c["d"]:
            for S in c["S"]:
                for dname in c["dtype"]:
                    dt = synth.DTYPES[dname]
                    gen = torch.Generator(device=dev).manual_seed(3300 + S + d + rank)
                    shp = (c["B"], S, c["H"], d)
                    q, k, v = (torch.randn(shp, generator=gen, device=dev).to(dt)
                               for _ in range(3))
                    out = torch.empty_like(q)
                    lse = torch.empty((c["B"], c["H"], S), dtype=torch.float32, device=dev)
                    for _ in range(args.warmup):
                        flush.zero_()
                        fa.fa_fwd(q, k, v, out=out, lse=lse, causal=True, stream=stream)
                    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
                          for _ in range(K)]
                    barrier(world)
                    torch.cuda.synchronize(dev)
                    for i in range(K):
                        flush.zero_()
                        ev[i][0].record(stream)
                        fa.fa_fwd(q, k, v, out=out, lse=lse, causal=True, stream=stream)
                        ev[i][1].record(stream)
                    torch.cuda.synchronize(dev)
                    barrier(world)
                    ms = max_over_ranks(statistics.median(e[0].elapsed_time(e[1]) for e in ev),
                                        world)
                    tf = 4.0 * d * c["B"] * c["H"] * causal_pairs(S, S) / (ms * 1e-3) / 1e12
                    curve.append({"d": d, "S": S, "dtype": dname, "ms": round(ms, 4),
                                  "tflops": round(tf, 1), "frac": round(tf / tflops_peak, 4)})
                    del q, k, v, out, lse
    assert fa.fa_device_status(clear=True) == 0, "device status flags raised during the sweep"
    top = curve[-1]
    return {"metric": "attn fwd TFLOPS vs seqlen (causal prefill)",
            "value": round(top["tflops"] * world, 2), "unit": "TFLOPS", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": top["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp16 / bf16; fp32 accumulate", "data": "synthetic (seeded N(0,1))",
            "config": {"workload": "causal prefill sweep B=4 H=32 over d, S and dtype; value = "
                                   "d=128 S=16384 bf16", "B": c["B"], "H": c["H"],
                       "l2": "flushed between launches (256 MiB write, untimed)",
                       "parallelism": f"dp{world} (independent replicas)"},
            "roofline": {"bound": "tensor", "achieved": top["tflops"], "peak": tflops_peak,
                         "unit": "TFLOP/s", "frac": top["frac"], "traffic": None,
                         "kernel": "fwd_kernel<128, bf16, causal>", "peak_source": peak_src},
            "curve": curve, "gpu_launches": K * len(curve), "clocks": clk.summary()}


def run_fp8(args, rank, world, local):
    """--only fp8: time fa_fwd_fp8 on the d=128 causal prefill workload."""
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build as fa_build
    fa_build.build()
    fa.load()
    dev = torch.device("cuda", local)
    hbm_peak, tflops_peak, peak_src = load_peaks()
    fp8_peak = 2.0 * tflops_peak       # dense e4m3 vs bf16: 4.5 / 2.25 PFLOP/s nominal
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    c = FP8
    gen = torch.Generator(device=dev).manual_seed(3100 + rank)
    shape_q = (c["B"], c["S"], c["H"], c["d"])
    shape_k = (c["B"], c["S"], c["Hkv"], c["d"])
    q = torch.randn(shape_q, generator=gen, device=dev).to(torch.float8_e4m3fn)
    k = torch.randn(shape_k, generator=gen, device=dev).to(torch.float8_e4m3fn)
    v = torch.randn(shape_k, generator=gen, device=dev).to(torch.float8_e4m3fn)
    out = torch.empty(shape_q, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((c["B"], c["H"], c["S"]), dtype=torch.float32, device=dev)
    work = 4.0 * c["d"] * c["B"] * c["H"] * causal_pairs(c["S"], c["S"])

    def call():
        fa.fa_fwd_fp8(q, k, v, out=out, lse=lse, causal=True, stream=stream)
    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world)
    achieved = work / (ms * 1e-3) / 1e12
    return {"metric": "attn fwd TFLOPS, E4M3 inputs (causal prefill)", "value": round(achieved * world, 2),
            "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 (bf16 out)", "data": "synthetic (seeded N(0,1))",
            "config": {"workload": "fp8", **c, "l2": "flushed between steps (256 MiB write, "
                       "untimed)", "parallelism": f"dp{world} (independent replicas)"},
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4),
                         "traffic": None,
                         "kernel": "fwd_kernel<128, 2 tiles, e4m3, causal> (kind::f8f6f4)",
                         "peak_source": f"{peak_src} bf16 burst x 2 (nominal e4m3/bf16 ratio)"},
            "gpu_launches": K, "clocks": clk.summary()}


def run_cache_rows(args, rank, world, local):
    """--only chunked | append: time one cache-update row on its own workload."""
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build as fa_build
    fa_build.build()
    fa.load()
    dev = torch.device("cuda", local)
    hbm_peak, tflops_peak, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    c = CHUNKED if args.only == "chunked" else APPEND
    dt = synth.DTYPES[c["dtype"]]
    B, Hkv, d, page = c["B"], c["Hkv"], c["d"], c["page"]
    s_new = c["chunk"] if args.only == "chunked" else c["S_new"]
    cached = c.get("cached", 0)
    total = cached + s_new
    nblk = (total + page - 1) // page
    gen = torch.Generator(device=dev).manual_seed(3000 + rank)
    kp = torch.randn(B * nblk, page, Hkv, d, generator=gen, device=dev).to(dt)
    vp = torch.randn(B * nblk, page, Hkv, d, generator=gen, device=dev).to(dt)
    perm = torch.randperm(B * nblk, generator=torch.Generator().manual_seed(3001 + rank))
    bt = perm.to(torch.int32).reshape(B, nblk).to(dev)
    cs = torch.full((B,), cached, dtype=torch.int32, device=dev)
    kn = torch.randn(B, s_new, Hkv, d, generator=gen, device=dev).to(dt)
    vn = torch.randn(B, s_new, Hkv, d, generator=gen, device=dev).to(dt)
    if args.only == "chunked":
        H = c["H"]
        q = torch.randn(B, s_new, H, d, generator=gen, device=dev).to(dt)
        out = torch.empty_like(q)
        lse = torch.empty((B, H, s_new), dtype=torch.float32, device=dev)
        ws = torch.empty(256, dtype=torch.uint8, device=dev)
        pairs = sum(cached + i + 1 for i in range(s_new))
        work = 4.0 * d * H * B * pairs                      # algorithmic FLOPs

        def call():
            fa.fa_fwd_kvcache(q, kp, vp, kn, vn, cache_seqlens=cs, block_table=bt, causal=True,
                              out=out, lse=lse, workspace=ws, stream=stream)
    else:
        work = 2.0 * B * s_new * Hkv * d * 2 * 2            # bytes: K and V, read and written

        def call():
            fa.fa_kvcache_append(kp, vp, kn, vn, cs, block_table=bt, stream=stream)
    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world)
    if args.only == "chunked":
        achieved = work / (ms * 1e-3) / 1e12
        metric, unit, peak, punit, bound = ("chunked prefill TFLOPS (append + attend, paged KV "
                                            "cache)", "TFLOPS", tflops_peak, "TFLOP/s", "tensor")
        kernel = "kv_append_kernel + fwd_kernel<128, bf16, causal> in KV-cache mode"
    else:
        achieved = work / (ms * 1e-3) / 1e9
        metric, unit, peak, punit, bound = ("KV-cache append GB/s (paged)", "GB/s", hbm_peak,
                                            "GB/s", "hbm")
        kernel = "kv_append_kernel"
    value = achieved * world
    return {"metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": c["dtype"], "data": "synthetic (seeded N(0,1))",
            "config": {"workload": args.only, **c, "l2": "flushed between steps (256 MiB write, "
                       "untimed)", "parallelism": f"dp{world} (independent replicas)"},
            "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": peak,
                         "unit": punit, "frac": round(achieved / peak, 4), "traffic": None,
                         "kernel": kernel, "peak_source": peak_src},
            "gpu_launches": K * (2 if args.only == "chunked" else 1),
            "clocks": clk.summary()}


def e2e_prefill(fa, q, k, v, dev, stream, flops, world, steps=5):
    """Prefill TFLOPS through the public call with pinned host buffers: the H2D copy
    of q, k, v, the kernel and the D2H copy of O are all inside the timed region."""
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    hout = torch.empty_like(hq).pin_memory()
    dq_, dk_, dv_ = torch.empty_like(hq, device=dev), torch.empty_like(hk, device=dev), \
        torch.empty_like(hv, device=dev)
    dout = torch.empty_like(dq_)
    for _ in range(2):
        dq_.copy_(hq, non_blocking=True)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        dq_.copy_(hq, non_blocking=True)
        dk_.copy_(hk, non_blocking=True)
        dv_.copy_(hv, non_blocking=True)
        fa.fa_fwd(dq_, dk_, dv_, out=dout, causal=True, return_lse=False, stream=stream)
        hout.copy_(dout, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    ms = max_over_ranks(ms, world)
    h2d = 3 * hq.numel() * hq.element_size()
    d2h = hout.numel() * hout.element_size()
    return {"value": round(flops / (ms * 1e-3) / 1e12 * world, 2), "unit": "TFLOPS",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "what": "prefill via fa_fwd with pinned host inputs/outputs copied every step"}


# ---------------------------------------------------------------- CPU oracle
def oracle_prefill_sample(heads: int, threads: int):
    """Time the fp64 oracle on `heads` full (b, h) problems of the prefill workload."""
    import oracle
    c = PREFILL
    q, k, v = synth.dense(1, c["S"], c["S"], heads, heads, c["d"], synth.DTYPES[c["dtype"]],
                          seed=1003)
    t0 = time.perf_counter()
    oracle.attention_dense(q, k, v, causal=True, threads=threads)
    dt = time.perf_counter() - t0
    flops = 4.0 * c["d"] * heads * causal_pairs(c["S"], c["S"])
    return flops / dt / 1e12, dt


def cpu_baseline(args):
    # up to all 128 (b, h) problems of the workload, eight per host core (about 10 s on
    # a 16-core host); the problems are independent, so the rate is the workload's
    cores = max(1, os.cpu_count() or 1)
    problems = min(PREFILL["B"] * PREFILL["H"], 8 * cores)
    tf, dt = oracle_prefill_sample(problems, cores)
    return {"value": round(tf, 6), "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "sample": f"prefill workload, {problems} of its {PREFILL['B'] * PREFILL['H']} "
                      f"(b, h) problems, full S={PREFILL['S']} causal (fp64 C oracle, "
                      f"OpenMP over problems), {dt:.1f} s"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle on bounded samples of the prefill workload."""
    heads = max(1, min(8, os.cpu_count() or 1))        # one OpenMP thread per head
    cores = heads
    times = []
    for i in range(args.warmup + args.steps):
        tf, dt = oracle_prefill_sample(heads, heads)
        if i >= args.warmup:
            times.append((tf, dt))
    tf = statistics.median(t for t, _ in times)
    ms = statistics.median(d for _, d in times) * 1e3
    return {"metric": METRIC, "impl": "reference", "value": round(tf, 6), "unit": "TFLOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
            "config": {"workload": "causal prefill B=4 S=4096 H=32 d=64 (bounded sample: "
                                   f"batch 0, {heads} heads per step)"},
            "cpu_baseline": {"value": round(tf, 6), "unit": "TFLOPS", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{heads} heads x full S=4096 causal per step"},
            "e2e": {"value": round(tf, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--num-splits", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "chunked", "append", "fp8",
                                       "bwd", "sweep"],
                    default="all",
                    help="time one part of the step (profiling / sweeps), or one of the "
                         "cache-update rows on its own workload (chunked, append)")
    ap.add_argument("--prefill-seq", type=int, default=PREFILL["S"])
    ap.add_argument("--prefill-d", type=int, default=PREFILL["d"])
    ap.add_argument("--prefill-dtype", choices=["fp16", "bf16"], default=PREFILL["dtype"])
    ap.add_argument("--decode-batch", type=int, default=DECODE["B"])
    args = ap.parse_args()
    PREFILL.update(S=args.prefill_seq, d=args.prefill_d, dtype=args.prefill_dtype)
    DECODE.update(B=args.decode_batch)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_reference(args, rank, world)), flush=True)
            return
        if args.only in ("chunked", "append", "fp8", "bwd", "sweep"):
            fn = {"fp8": run_fp8, "bwd": run_bwd, "sweep": run_sweep}.get(args.only,
                                                                          run_cache_rows)
            res = fn(args, rank, world, local)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res = run_ours(args, rank, world, local)
        if rank == 0:
            if not args.no_cpu_baseline and world == 1:
                res["cpu_baseline"] = cpu_baseline(args)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

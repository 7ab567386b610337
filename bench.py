"""Benchmark of the attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  1. prefill forward (fa_fwd): causal, B=4, S=4096, H=32, d=64, fp16
  2. paged split-KV decode (fa_fwd_kvcache) + LSE combine: B=64, Sq=1, H=32,
     Hkv=8, d=128, bf16, cache lengths U{1K..32K}, pages of 256, random
     block_table, at num_splits 4 (headline), 16 and 1 (the unsplit control)
Each kernel runs R times back to back per step (its inputs exceed the L2); the
L2 is flushed between steps.  Per kernel the median and the minimum launch time
over the steps are reported; ``value`` uses the median.
Reported: ``value`` = prefill TFLOPS (4*d*sum of allowed (i, j) pairs / time);
``decode`` = KV-cache GB/s (valid cache bytes + q/out/lse/block_table / time).
Both are also given as fractions of the measured B200 peaks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--num-splits S] [--repeat R] [--no-cpu-baseline] [--no-e2e]
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


def sustained_tflops():
    """The measured bf16 GEMM rate under the power cap (seconds-long loop), or None."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f).get("bf16_tflops_sustained")
    return None


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


def decode_bytes(lens):
    c = DECODE
    kv = sum(lens) * c["Hkv"] * c["d"] * 2 * 2               # K and V, valid tokens only
    io = c["B"] * c["Sq"] * c["H"] * c["d"] * 2 * 2          # q in, out
    io += c["B"] * c["H"] * c["Sq"] * 4                       # lse
    bt = sum((L + c["page"] - 1) // c["page"] for L in lens) * 4 + c["B"] * 4
    return kv + io + bt


def _stats(ms_list):
    """Per-launch times (ms) of one kernel over the timed steps."""
    return {"median_ms": round(statistics.median(ms_list), 5), "min_ms": round(min(ms_list), 5),
            "mean_ms": round(sum(ms_list) / len(ms_list), 5), "launch_samples": len(ms_list)}


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
    # the headline split count first, then the others of the workload; 1 is the
    # unsplit control (one CTA per (sequence, KV head): imbalanced by design)
    split_list = [args.num_splits] + [x for x in (16, 4, 1) if x != args.num_splits]
    c = DECODE
    ws_bytes = max(fa.fa_kvcache_workspace_size(c["B"], c["Sq"], c["H"], c["Hkv"], c["d"],
                                                bt.shape[1] * c["page"], c["page"], x)
                   for x in split_list)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    out_d = torch.empty_like(dq_d)
    lse_d = torch.empty((c["B"], c["H"], c["Sq"]), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    do_pre = args.only in ("all", "prefill")
    do_dec = args.only in ("all", "decode")
    R = max(1, args.repeat)

    def prefill():
        fa.fa_fwd(qd_, kd_, vd_, out=out_p, lse=lse_p, causal=True, stream=stream)

    def decode(splits, o=None, l=None):
        fa.fa_fwd_kvcache(dq_d, kp, vp, cache_seqlens=cs_d, block_table=bt_d, causal=True,
                          num_splits=splits, out=out_d if o is None else o,
                          lse=lse_d if l is None else l, workspace=ws, stream=stream)

    groups = ([("prefill", prefill)] if do_pre else []) + (
        [(f"decode_s{x}", (lambda x=x: decode(x))) for x in split_list] if do_dec else [])
    for _ in range(args.warmup):
        flush.zero_()
        for _, fn in groups:
            fn()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(groups) + 1)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        for s in range(K):
            flush.zero_()                       # L2 flushed between steps (not timed)
            ev[s][0].record(stream)
            for g, (_, fn) in enumerate(groups):
                for _ in range(R):              # inputs exceed L2: back-to-back launches
                    fn()
                ev[s][g + 1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    per = {name: [ev[s][g].elapsed_time(ev[s][g + 1]) / R for s in range(K)]
           for g, (name, _) in enumerate(groups)}
    st = {name: _stats(v) for name, v in per.items()}
    t_step = statistics.median(ev[s][0].elapsed_time(ev[s][-1]) for s in range(K))
    t_step_max = max_over_ranks(t_step, world)
    assert fa.fa_device_status(clear=True) == 0, "device status flags raised during the bench"

    flops = prefill_flops()
    dbytes = decode_bytes(lens)
    res = {
        "metric": METRIC, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(t_step_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16 (prefill), bf16 (decode); fp32 accumulate",
        "data": "synthetic (seeded N(0,1))",
        "config": {
            "workload": (f"causal prefill B={PREFILL['B']} S={PREFILL['S']} H={PREFILL['H']} "
                         f"d={PREFILL['d']} {PREFILL['dtype']} + paged split-KV decode "
                         f"B={DECODE['B']} H=32 Hkv=8 d=128 bf16 cache U{{1K..32K}} page 256 "
                         f"at num_splits {split_list}"),
            "prefill": dict(PREFILL, flop=flops),
            "decode": dict(DECODE, num_splits=split_list, sum_cache_tokens=int(sum(lens)),
                           bytes=dbytes),
            "launches_per_kernel_per_step": R,
            "l2": ("flushed between steps (256 MiB write, untimed); within a step each kernel "
                   "runs back to back on inputs larger than L2 (prefill q/k/v "
                   f"{3 * q.numel() * q.element_size() >> 20} MiB, decode KV cache "
                   f"{(kp.numel() + vp.numel()) * kp.element_size() >> 20} MiB)"),
            "parallelism": f"dp{world} (independent replicas)",
        },
        # per decode call: the prep kernel (counter, longest-first order), the split
        # kernel and, above one split, the combine kernel
        "gpu_launches": K * R * ((1 if do_pre else 0) +
                                 (sum(3 if x > 1 else 2 for x in split_list) if do_dec else 0)),
        "clocks": clk.summary(),
    }
    if do_pre:
        t_pre = max_over_ranks(st["prefill"]["median_ms"], world)
        achieved = flops / (st["prefill"]["median_ms"] * 1e-3) / 1e12
        res["value"] = round(flops / (t_pre * 1e-3) / 1e12 * world, 2)
        res["prefill"] = dict(st["prefill"], tflops_median=round(achieved, 2),
                              tflops_best=round(flops / (st["prefill"]["min_ms"] * 1e-3) / 1e12, 2))
        res["roofline"] = {
            "bound": "tensor", "achieved": round(achieved, 2), "peak": tflops_peak,
            "unit": "TFLOP/s", "frac": round(achieved / tflops_peak, 4),
            "traffic": (profiled_traffic("fwd_kernel_d64_causal_B4_S4096.md",
                                         ["fwd_kernel.cuh", "fwd_launch.cuh", "sm100.cuh",
                                          "fa_internal.h"])
                        if (PREFILL["d"] == 64 and PREFILL["S"] == 4096) else None),
            "kernel": f"fwd_kernel<{PREFILL['d']}, {PREFILL['dtype']}, causal>",
            "peak_source": f"{peak_src} bf16 burst (fp16 dense rate equals bf16)"}
        sus = sustained_tflops()
        if sus:
            # the step repeats each kernel back to back for about a second, which can bring
            # the power cap in (see clocks); the GEMM rate measured under it, for context
            res["roofline"]["frac_vs_sustained_peak"] = round(achieved / sus, 4)
            res["roofline"]["sustained_peak"] = sus
    if do_dec:
        by = {}
        for x in split_list:
            sx = st[f"decode_s{x}"]
            gbs = dbytes / (sx["median_ms"] * 1e-3) / 1e9
            by[str(x)] = dict(sx, gbs_median=round(gbs, 1),
                              gbs_best=round(dbytes / (sx["min_ms"] * 1e-3) / 1e9, 1),
                              frac=round(gbs / hbm_peak, 4),
                              role=("headline" if x == args.num_splits else
                                    "unsplit control" if x == 1 else "reported"))
        main = by[str(args.num_splits)]
        t_dec = max_over_ranks(main["median_ms"], world)
        res["decode"] = {
            "value": round(dbytes / (t_dec * 1e-3) / 1e9 * world, 1), "unit": "GB/s",
            "num_splits": args.num_splits, "ms": round(t_dec, 5),
            "roofline": {"bound": "hbm", "achieved": main["gbs_median"], "peak": hbm_peak,
                         "unit": "GB/s", "frac": main["frac"],
                         "traffic": (profiled_traffic(f"decode_kernel_paged_B64_s{args.num_splits}.md",
                                                      ["decode_kernel.cuh", "decode.cu",
                                                       "sm100.cuh", "fa_internal.h"])
                                     if DECODE["B"] == 64 else None),
                         "kernel": "decode_kernel<128, bf16> + combine_kernel",
                         "peak_source": peak_src},
            "by_num_splits": by}
        if not do_pre:
            res.update(value=res["decode"]["value"], unit="GB/s")
    if not args.no_e2e and do_pre:
        res["e2e"] = e2e_prefill(fa, q, k, v, dev, stream, flops, world, steps=K)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(args, gpu=dict(
            q=q, k=k, v=v, out=out_p if do_pre else None, lse=lse_p if do_pre else None,
            dq=dq, kp=kp, vp=vp, bt=bt, cs=cs, lens=lens,
            decode=(lambda x, o, l: decode(x, o, l)) if do_dec else None, splits=split_list,
            dev=dev, stream=stream))
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
    """--only bwd: time fa_bwd (D pre-pass + one launch of dK/dV and dQ CTAs).  Algorithmic work:
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
                         # DRAM bytes of a whole step (both launches), like `achieved`
                         "traffic": (profiled_traffic("bwd_kernels_causal_B4_S4096_d128.md",
                                                      ["bwd_kernel.cuh", "bwd.cu", "sm100.cuh",
                                                       "fa_internal.h"])
                                     if (c["B"], c["S"], c["H"], c["Hkv"], c["d"]) ==
                                     (4, 4096, 32, 32, 128) and c["dtype"] == "bf16"
                                     and c["causal"] else None),
                         "kernel": "bwd_dot_kernel + bwd_tiles_kernel (dK/dV and dQ CTAs) <128, bf16>",
                         "peak_source": peak_src},
            "gpu_launches": 2 * K, "clocks": clk.summary()}  # D pre-pass + tile launch


# TFLOPS vs sequence length of the causal prefill (B=4, H=Hkv=32)
SWEEP = dict(B=4, H=32, d=(64, 128), S=(512, 1024, 2048, 4096, 8192, 16384),
             dtype=("fp16", "bf16"))


def run_sweep(args, rank, world, local):
    """--only sweep: the causal prefill's TFLOPS over head dims, sequence lengths
    and 16-bit types; one JSON line whose value is the largest point (d=128,
    S=16384, bf16) and whose ``curve`` holds every point with its own clock record
    (each point launches for at least ~0.3 s, L2 flushed between launches, so the
    100 ms sampler sees it)."""
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build as fa_build
    fa_build.build()
    fa.load()
    dev = torch.device("cuda", local)
    _, tflops_peak, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    c = SWEEP
    curve = []
    launches = 0
    all_reasons = set()
    for d in c["d"]:
        for S in c["S"]:
            for dname in c["dtype"]:
                dt = synth.DTYPES[dname]
                gen = torch.Generator(device=dev).manual_seed(3300 + S + d + rank)
                shp = (c["B"], S, c["H"], d)
                q, k, v = (torch.randn(shp, generator=gen, device=dev).to(dt) for _ in range(3))
                out = torch.empty_like(q)
                lse = torch.empty((c["B"], c["H"], S), dtype=torch.float32, device=dev)

                def call():
                    fa.fa_fwd(q, k, v, out=out, lse=lse, causal=True, stream=stream)
                for _ in range(args.warmup):
                    flush.zero_()
                    call()
                torch.cuda.synchronize(dev)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                call()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                est = max(e0.elapsed_time(e1), 1e-3)
                K = max(min(args.steps, 10), int(300.0 / (est + 0.05)) + 1)
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
                launches += K
                ms = max_over_ranks(statistics.median(e[0].elapsed_time(e[1]) for e in ev),
                                    world)
                ms_min = min(e[0].elapsed_time(e[1]) for e in ev)
                flop = 4.0 * d * c["B"] * c["H"] * causal_pairs(S, S)
                tf = flop / (ms * 1e-3) / 1e12
                ck = clk.summary()
                all_reasons.update(ck.get("reasons", []))
                curve.append({"d": d, "S": S, "dtype": dname, "ms": round(ms, 4),
                              "tflops": round(tf, 1),
                              "tflops_best": round(flop / (ms_min * 1e-3) / 1e12, 1),
                              "frac": round(tf / tflops_peak, 4), "launches": K, "clocks": ck})
                del q, k, v, out, lse
    assert fa.fa_device_status(clear=True) == 0, "device status flags raised during the sweep"
    top = curve[-1]
    return {"metric": "attn fwd TFLOPS vs seqlen (causal prefill)",
            "value": round(top["tflops"] * world, 2), "unit": "TFLOPS", "n_gpus": world,
            "steps": top["launches"], "warmup": args.warmup, "ms_per_step": top["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp16 / bf16; fp32 accumulate", "data": "synthetic (seeded N(0,1))",
            "config": {"workload": "causal prefill sweep B=4 H=32 over d, S and dtype; value = "
                                   "d=128 S=16384 bf16", "B": c["B"], "H": c["H"],
                       "l2": "flushed between launches (256 MiB write, untimed)",
                       "parallelism": f"dp{world} (independent replicas)"},
            "roofline": {"bound": "tensor", "achieved": top["tflops"], "peak": tflops_peak,
                         "unit": "TFLOP/s", "frac": top["frac"], "traffic": None,
                         "kernel": "fwd_kernel<128, bf16, causal>", "peak_source": peak_src},
            "curve": curve, "gpu_launches": launches,
            "clocks": {"per_point": True, "reasons": sorted(all_reasons)}}


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
                         "traffic": (profiled_traffic("fwd_kernel_fp8_causal_B4_S8192.md",
                                                      ["fwd_kernel.cuh", "fwd_launch.cuh",
                                                       "fwd_fp8.cu", "sm100.cuh",
                                                       "fa_internal.h"])
                                     # the capture ran the default exponential split
                                     if os.environ.get("FA_EXP2_EMU") is None else None),
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
    """Prefill TFLOPS through the public host-buffer call (fa_fwd_host): q, k, v and O
    live in pinned host memory, and every step's H2D copies of q, k, v, the kernels and
    the D2H copy of O are inside the timed region (the library overlaps them chunk by
    chunk on its own streams and joins the caller's stream at the end)."""
    hq, hk, hv = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
    hout = torch.empty(hq.shape, dtype=hq.dtype, pin_memory=True)
    B, S, H, d = hq.shape
    ws = torch.empty(fa.fa_fwd_host_workspace_size(B, S, k.shape[1], H, k.shape[2], d, False),
                     dtype=torch.uint8, device=dev)
    for _ in range(2):
        fa.fa_fwd_host(hq, hk, hv, out=hout, causal=True, return_lse=False, workspace=ws,
                       stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fa.fa_fwd_host(hq, hk, hv, out=hout, causal=True, return_lse=False, workspace=ws,
                       stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    ms = max_over_ranks(ms, world)
    h2d = 3 * hq.numel() * hq.element_size()
    d2h = hout.numel() * hout.element_size()
    return {"value": round(flops / (ms * 1e-3) / 1e12 * world, 2), "unit": "TFLOPS",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "what": "prefill via fa_fwd_host: pinned host q, k, v in, O out, every step; "
                    "copies overlapped with the kernels in chunks of whole sequences"}


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


def _max_abs(a, b):
    import numpy as np
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    fin = np.isfinite(b)
    if not np.array_equal(np.isfinite(a), fin) or not np.array_equal(a[~fin], b[~fin]):
        return float("inf")
    return float(np.abs(a[fin] - b[fin]).max()) if fin.any() else 0.0


def cpu_baseline(args, gpu=None):
    """The fp64 oracle on the host cores: timed on a bounded sample of the prefill
    workload's own (b, h) problems (eight per core, about 10 s on 16 cores), whose
    outputs also give the sample's max |dO| and |dLSE| against the GPU run; plus
    single-thread times of the two small parity configurations."""
    import numpy as np

    import oracle
    cores = max(1, os.cpu_count() or 1)
    c = PREFILL
    res = {"unit": "TFLOPS", "cores": cores, "kind": "oracle"}
    if gpu is not None and gpu["out"] is not None:
        q, k, v = gpu["q"], gpu["k"], gpu["v"]
        problems = min(c["B"] * c["H"], 8 * cores)
        nb = (problems + c["H"] - 1) // c["H"]
        ro_all, rl_all = [], []
        t0 = time.perf_counter()
        for b in range(nb):
            nh = min(c["H"], problems - b * c["H"])
            ro, rl = oracle.attention_dense(q[b:b + 1, :, :nh], k[b:b + 1, :, :nh],
                                            v[b:b + 1, :, :nh], causal=True, threads=cores)
            ro_all.append((b, nh, ro))
            rl_all.append((b, nh, rl))
        dt = time.perf_counter() - t0
        flops = 4.0 * c["d"] * problems * causal_pairs(c["S"], c["S"])
        go = gpu["out"].float().cpu().numpy()
        gl = gpu["lse"].cpu().numpy()
        d_o = max(_max_abs(go[b:b + 1, :, :nh], ro) for b, nh, ro in ro_all)
        d_l = max(_max_abs(gl[b:b + 1, :nh], rl) for b, nh, rl in rl_all)
        res.update(value=round(flops / dt / 1e12, 6),
                   sample=(f"prefill workload, its first {problems} of {c['B'] * c['H']} (b, h) "
                           f"problems, full S={c['S']} causal (fp64 C oracle, OpenMP over "
                           f"problems, {cores} threads), {dt:.1f} s"),
                   parity={"prefill": {"max_abs_dO": d_o, "max_abs_dLSE": d_l,
                                       "problems": problems,
                                       "tolerance": {"dO": 2e-3 if c["dtype"] == "fp16" else 1e-2,
                                                     "dLSE": 1e-3}}})
    else:
        problems = min(c["B"] * c["H"], 8 * cores)
        tf, dt = oracle_prefill_sample(problems, cores)
        res.update(value=round(tf, 6),
                   sample=f"{problems} (b, h) problems of S={c['S']} causal, {dt:.1f} s")
    if gpu is not None and gpu["decode"] is not None:
        # the first eight sequences of the decode batch, every head, at each split count
        n = min(8, len(gpu["lens"]))
        dev, D = gpu["dev"], DECODE
        # only their pages reach the host: a compact pool and a remapped block table
        bt_n = gpu["bt"][:n].clone()
        ids = sorted({int(x) for x in bt_n.flatten().tolist() if x >= 0})
        remap = {b: i for i, b in enumerate(ids)}
        bt_c = bt_n.apply_(lambda x: remap[x] if x >= 0 else -1)
        idx = torch.tensor(ids, dtype=torch.long, device=gpu["kp"].device)
        kc = gpu["kp"].index_select(0, idx).cpu()
        vc = gpu["vp"].index_select(0, idx).cpu()
        ro, rl = oracle.attention_paged(gpu["dq"][:n], kc, vc, bt_c, gpu["cs"][:n], causal=True,
                                        threads=cores)
        par = {}
        for x in gpu["splits"]:
            o = torch.empty((D["B"], D["Sq"], D["H"], D["d"]), dtype=torch.bfloat16, device=dev)
            lz = torch.empty((D["B"], D["H"], D["Sq"]), dtype=torch.float32, device=dev)
            gpu["decode"](x, o, lz)
            torch.cuda.synchronize(dev)
            par[str(x)] = {"max_abs_dO": _max_abs(o[:n].float().cpu().numpy(), ro),
                           "max_abs_dLSE": _max_abs(lz[:n].cpu().numpy(), rl)}
        res.setdefault("parity", {})["decode"] = dict(
            by_num_splits=par, sequences=n, tolerance={"dO": 1e-2, "dLSE": 1e-3})
    # single-thread oracle times of the tiny and the causal Sq != Sk configurations
    one = {}
    for name, (B, Sq, Sk, H, d, dt_, causal) in {
            "tiny B1 H2 S128 d64 fp16": (1, 128, 128, 2, 64, torch.float16, False),
            "causal B2 H8 Sq384 Sk1024 d128 bf16": (2, 384, 1024, 8, 128, torch.bfloat16, True)
    }.items():
        qq, kk, vv = synth.dense(B, Sq, Sk, H, H, d, dt_, seed=1001)
        t0 = time.perf_counter()
        oracle.attention_dense(qq, kk, vv, causal=causal, threads=1)
        one[name] = round((time.perf_counter() - t0) * 1e3, 3)
    res["single_thread_ms"] = one
    return res


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle, on all host cores (one OpenMP thread per
    (b, h) problem, as many problems per step as cores), on bounded samples of the
    prefill workload."""
    cores = max(1, os.cpu_count() or 1)
    heads = max(1, min(PREFILL["B"] * PREFILL["H"], cores))
    times = []
    for i in range(args.warmup + args.steps):
        tf, dt = oracle_prefill_sample(heads, cores)
        if i >= args.warmup:
            times.append((tf, dt))
    tf = statistics.median(t for t, _ in times)
    ms = statistics.median(d for _, d in times) * 1e3
    return {"metric": METRIC, "impl": "reference", "value": round(tf, 6), "unit": "TFLOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
            "config": {"workload": "causal prefill B=4 S=4096 H=32 d=64 (bounded sample: "
                                   f"{heads} (b, h) problems per step)"},
            "cpu_baseline": {"value": round(tf, 6), "unit": "TFLOPS", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{heads} heads x full S=4096 causal per step, "
                                       f"{cores} threads"},
            "e2e": {"value": round(tf, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--num-splits", type=int, default=4,
                    help="the decode's headline split count (16 and 1 are timed beside it)")
    ap.add_argument("--repeat", type=int, default=10,
                    help="back-to-back launches of each kernel per step (inputs exceed L2)")
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
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

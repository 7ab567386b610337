"""Host-side pieces of bench.py that need no GPU: the algorithmic work counts,
the clock-record parser and the traffic lookup keyed to the kernel sources."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def brute_pairs(Sq, Sk):
    off = Sk - Sq
    return sum(1 for i in range(Sq) for j in range(Sk) if j <= i + off)


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (5, 5), (3, 7), (7, 3), (1, 1025), (384, 1024)])
def test_causal_pairs_brute_force(Sq, Sk):
    assert bench.causal_pairs(Sq, Sk) == brute_pairs(Sq, Sk)


def test_prefill_flops_of_the_headline_workload():
    # causal B=4 S=4096 H=32 d=64: 4 d FLOPs per allowed pair, S (S + 1) / 2 pairs per head
    S = 4096
    assert bench.causal_pairs(S, S) == S * (S + 1) // 2
    assert bench.prefill_flops() == pytest.approx(4 * 64 * 4 * 32 * S * (S + 1) / 2)
    assert bench.prefill_flops() == pytest.approx(2.7495e11, rel=1e-4)


def test_decode_bytes_counts_valid_tokens_only():
    lens = [1, 256, 257]
    c = bench.DECODE
    kv = sum(lens) * c["Hkv"] * c["d"] * 2 * 2
    io = c["B"] * c["Sq"] * c["H"] * c["d"] * 2 * 2 + c["B"] * c["H"] * c["Sq"] * 4
    bt = (1 + 1 + 2) * 4 + c["B"] * 4      # pages touched, plus cache_seqlens
    assert bench.decode_bytes(lens) == kv + io + bt


def test_clock_summary_parses_reasons_and_ignores_idle_samples():
    clk = bench.Clocks(0)
    clk.lines = [
        "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1965, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1905, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 345, 1965, 120.0, 0x1, Not Active, Not Active, Not Active, Not Active",  # idle
        "garbage",
    ]
    s = clk.summary()
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1965.0            # median of the busy samples
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 4


def test_clock_summary_without_samples():
    clk = bench.Clocks(0)
    clk.lines = []
    assert clk.summary()["reasons"] == ["unsampled"]


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "io_aware_online_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "a.cuh").write_bytes(b"kernel one")
    (csrc / "b.cu").write_bytes(b"kernel two")
    h = hashlib.sha256(b"kernel one" + b"kernel two").hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        f"# summary\ntraffic_bytes_per_launch: 12345\nsource_sha256_16: {h}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k.md", ["a.cuh", "b.cu"]) == 12345
    (csrc / "b.cu").write_bytes(b"kernel two, changed")
    assert bench.profiled_traffic("k.md", ["a.cuh", "b.cu"]) is None
    assert bench.profiled_traffic("missing.md", ["a.cuh"]) is None



def test_stats_report_median_min_and_mean():
    st = bench._stats([3.0, 1.0, 2.0, 10.0])
    assert st["median_ms"] == 2.5 and st["min_ms"] == 1.0 and st["mean_ms"] == 4.0
    assert st["launch_samples"] == 4


def test_max_abs_requires_the_same_infinities():
    import math
    assert bench._max_abs([1.0, 2.0], [1.5, 2.0]) == 0.5
    assert bench._max_abs([-math.inf, 1.0], [-math.inf, 1.25]) == 0.25
    # a -inf LSE on one side only is a mismatch, reported as an infinite difference
    assert bench._max_abs([0.0, 1.0], [-math.inf, 1.0]) == math.inf

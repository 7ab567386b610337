"""Parity at the full benchmark sizes, on sampled rows.

The kernels run on the whole workload exactly as bench.py launches them; the
oracle then recomputes a sample of rows one by one.  Under a causal mask a
single query row i of a problem with Sq queries and Sk keys is reproduced
exactly by the one-row problem with keys 0 .. i + Sk - Sq (same alignment, same
ALiBi distances, same window).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import ATOL, check_lse, check_out

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from io_aware_online_b200 import build
    build.build()
    import io_aware_online_b200 as fa
    fa.load()
    fa.fa_device_status(clear=True)
    yield
    assert fa.fa_device_status(clear=True) == 0


def fa():
    import io_aware_online_b200 as m
    return m


def oracle_causal_rows(q, k, v, rows, window=(-1, -1), softcap=0.0, slopes=None):
    """q [Sq, H, d], k/v [Sk, Hkv, d] of one sequence -> {row: (O [H, d], LSE [H])}."""
    Sq, Sk = q.shape[0], k.shape[0]
    res = {}
    for i in rows:
        kend = min(Sk, i + Sk - Sq + 1)
        H, d = q.shape[1], q.shape[2]
        if kend <= 0:
            res[i] = (np.zeros((H, d)), np.full(H, -math.inf))
            continue
        o, l = oracle.attention_dense(q[i:i + 1][None], k[:kend][None], v[:kend][None],
                                      causal=True, window=window, softcap=softcap,
                                      alibi_slopes=slopes)
        res[i] = (o[0, 0], l[0, :, 0])
    return res


def test_causal_prefill_benchmark_shape_fp16_d64():
    """B=4, S=4096, H=32, d=64, fp16, causal: the prefill benchmark workload."""
    B, S, H, d = 4, 4096, 32, 64
    q, k, v = synth.dense(B, S, S, H, H, d, torch.float16, seed=1003)
    out, lse = fa().fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    torch.cuda.synchronize()
    out, lse = out.cpu(), lse.cpu()
    assert torch.isfinite(out.float()).all()
    rows = [0, 1, 127, 128, 129, 255, 256, 1000, 2047, 2048, 3071, 4094, 4095]
    for b in (0, 3):
        ref = oracle_causal_rows(q[b], k[b], v[b], rows)
        for i, (ro, rl) in ref.items():
            assert check_out(out[b, i], ro, torch.float16) <= ATOL[torch.float16]
            check_lse(lse[b, :, i], rl)


@pytest.mark.parametrize("S,d,dtype", [(16384, 128, torch.bfloat16), (8192, 128, torch.float16),
                                       (512, 64, torch.bfloat16)])
def test_prefill_sweep_points(S, d, dtype):
    B, H = 4, 32
    q, k, v = synth.dense(B, S, S, H, H, d, dtype, seed=1003 + S + d)
    out, lse = fa().fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    torch.cuda.synchronize()
    out, lse = out.cpu(), lse.cpu()
    rows = [0, 255, 256, S // 2 + 17, S - 129, S - 1]
    b = 1
    ref = oracle_causal_rows(q[b], k[b], v[b], rows)
    for i, (ro, rl) in ref.items():
        assert check_out(out[b, i], ro, dtype) <= ATOL[dtype]
        check_lse(lse[b, :, i], rl)


def test_varlen_gqa_variants_full():
    """16 sequences, lengths U{256..8192}, H=32, Hkv=8, d=128, bf16; causal,
    window (4096, 0), softcap 50, ALiBi slopes 2^(-8i/32)."""
    lens = synth.varlen_lengths(16, 256, 8192, seed=1004)
    H, Hkv, d = 32, 8, 128
    q, k, v, cq, ck = synth.varlen(lens, lens, H, Hkv, d, torch.bfloat16, seed=1004)
    slopes = synth.alibi_slopes(H)
    out, lse = fa().fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), cu_seqlens_q=cq.to(DEV),
                           cu_seqlens_k=ck.to(DEV), max_seqlen_q=max(lens), max_seqlen_k=max(lens),
                           causal=True, window_size=(4096, 0), softcap=50.0,
                           alibi_slopes=slopes.to(DEV))
    torch.cuda.synchronize()
    out, lse = out.cpu(), lse.cpu()
    assert torch.isfinite(out.float()).all()
    for b in (0, 5, 11, 15):
        s0, L = int(cq[b]), lens[b]
        rows = sorted({0, 1, 200, L // 2, max(0, L - 4097), L - 1} & set(range(L)))
        ref = oracle_causal_rows(q[s0:s0 + L], k[s0:s0 + L], v[s0:s0 + L], rows,
                                 window=(4096, 0), softcap=50.0, slopes=slopes)
        for i, (ro, rl) in ref.items():
            check_out(out[s0 + i], ro, torch.bfloat16)
            check_lse(lse[:, s0 + i], rl)


@pytest.mark.parametrize("splits", [1, 4, 16])
def test_paged_decode_benchmark_shape(splits):
    """B=64, Sq=1, H=32, Hkv=8, d=128, bf16, cache lengths U{1K..32K}, pages of 256,
    random-permutation block_table, NaN page tails."""
    B, H, Hkv, d, page = 64, 32, 8, 128, 256
    lens = synth.varlen_lengths(B, 1024, 32768, seed=1005)
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, torch.bfloat16, seed=1005,
                                       device=DEV)
    g = torch.Generator().manual_seed(1006)
    q = torch.randn(B, 1, H, d, generator=g).to(torch.bfloat16)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kp, vp, cache_seqlens=cs.to(DEV),
                                   block_table=bt.to(DEV), causal=True, num_splits=splits)
    torch.cuda.synchronize()
    out, lse = out.cpu(), lse.cpu()
    for b in (0, 17, 42, 63):
        L = lens[b]
        npg = (L + page - 1) // page
        idx = bt[b, :npg].long().to(DEV)
        kc = kp[idx].reshape(-1, Hkv, d)[:L].cpu()
        vc = vp[idx].reshape(-1, Hkv, d)[:L].cpu()
        ro, rl = oracle.attention_dense(q[b:b + 1], kc[None], vc[None], causal=True)
        assert check_out(out[b:b + 1], ro, torch.bfloat16) <= ATOL[torch.bfloat16]
        check_lse(lse[b:b + 1], rl)
    del kp, vp
    torch.cuda.empty_cache()

"""GPU parity of fa_fwd_kvcache (split-KV decode over a paged or contiguous cache)
and fa_combine against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import ATOL, check_lse, check_out, to_np

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


def fa():
    import io_aware_online_b200 as m
    return m


def paged_case(lens, Sq, H, Hkv, d, dtype, page, seed, **kw):
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, dtype, seed=seed, spare_blocks=3)
    g = torch.Generator().manual_seed(seed + 1)
    q = torch.randn(len(lens), Sq, H, d, generator=g).to(dtype)
    return q, kp, vp, bt, cs


@pytest.mark.parametrize("splits", [1, 4, 16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("d", [128, 64])
def test_paged_decode_gqa(splits, dtype, d):
    lens = [1, 255, 256, 257, 1000, 3000, 64, 777]
    H, Hkv, page = 32, 8, 256
    q, kp, vp, bt, cs = paged_case(lens, 1, H, Hkv, d, dtype, page, seed=500 + d)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), cache_seqlens=cs.to(DEV),
                                   block_table=bt.to(DEV), causal=True, num_splits=splits)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_paged(q, kp, vp, bt, cs, causal=True)
    dmax = check_out(out, ro, dtype)
    check_lse(lse, rl)
    assert dmax <= ATOL[dtype]
    assert fa().fa_device_status(clear=True) == 0


def test_split_count_does_not_change_result_beyond_rounding():
    lens = [4000, 1500, 60]
    q, kp, vp, bt, cs = paged_case(lens, 1, 16, 4, 128, torch.bfloat16, 128, seed=12)
    outs = []
    for s in (1, 2, 5, 16, 0):
        o, l = fa().fa_fwd_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), cache_seqlens=cs.to(DEV),
                                   block_table=bt.to(DEV), num_splits=s)
        outs.append((o.float().cpu(), l.cpu()))
    for o, l in outs[1:]:
        assert (o - outs[0][0]).abs().max() <= 2e-2
        assert (l - outs[0][1]).abs().max() <= 1e-4


@pytest.mark.parametrize("Sq", [1, 2, 4])
@pytest.mark.parametrize("variant", ["causal", "window_softcap_alibi", "noncausal"])
def test_multirow_decode_variants(Sq, variant):
    lens = [700, 130, 2048, 5]
    H, Hkv, d, page = 8, 2, 128, 64
    q, kp, vp, bt, cs = paged_case(lens, Sq, H, Hkv, d, torch.bfloat16, page, seed=40 + Sq)
    kw = dict(causal=True)
    if variant == "window_softcap_alibi":
        kw = dict(causal=True, window_size=(300, -1), softcap=15.0)
        slopes = synth.alibi_slopes(H)
    else:
        slopes = None
    if variant == "noncausal":
        kw = dict(causal=False)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), cache_seqlens=cs.to(DEV),
                                   block_table=bt.to(DEV), num_splits=3,
                                   alibi_slopes=None if slopes is None else slopes.to(DEV), **kw)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_paged(q, kp, vp, bt, cs, causal=kw["causal"],
                                    window=kw.get("window_size", (-1, -1)),
                                    softcap=kw.get("softcap", 0.0), alibi_slopes=slopes)
    check_out(out, ro, torch.bfloat16)
    check_lse(lse, rl)


@pytest.mark.parametrize("splits", [1, 3])
def test_contiguous_cache_sq1_sk1025(splits):
    """Config: Sq=1, Sk=1025 causal through the KV-cache entry (contiguous cache)."""
    q, k, v = synth.dense(2, 1, 1025, 8, 8, 128, torch.bfloat16, seed=1012)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), k.to(DEV), v.to(DEV), causal=True,
                                   num_splits=splits)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_dense(q, k, v, causal=True)
    check_out(out, ro, torch.bfloat16)
    check_lse(lse, rl)


def test_contiguous_cache_with_seqlens():
    q, k, v = synth.dense(3, 2, 900, 8, 4, 64, torch.float16, seed=4)
    cs = torch.tensor([900, 1, 333], dtype=torch.int32)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), k.to(DEV), v.to(DEV), cache_seqlens=cs.to(DEV),
                                   causal=True, num_splits=2)
    torch.cuda.synchronize()
    for b in range(3):
        L = int(cs[b])
        ro, rl = oracle.attention_dense(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], causal=True)
        check_out(out[b:b + 1], ro, torch.float16)
        check_lse(lse[b:b + 1], rl)


def test_bad_block_table_entry_is_reported_not_faulted():
    lens = [300, 200]
    q, kp, vp, bt, cs = paged_case(lens, 1, 8, 8, 64, torch.float16, 64, seed=2)
    bt = bt.clone()
    bt[1, 0] = 10_000          # outside the pool
    fa().fa_device_status(clear=True)
    fa().fa_fwd_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), cache_seqlens=cs.to(DEV),
                        block_table=bt.to(DEV), num_splits=1)
    flags = fa().fa_device_status(clear=True)
    assert flags & fa().FA_DEV_BAD_BLOCK
    assert fa().fa_device_status(clear=True) == 0


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("layout", ["pages", "split_major"])
def test_combine(out_dtype, layout):
    g = torch.Generator().manual_seed(21)
    B, S, H, d, sp = 3, 2, 4, 128, 7
    op = torch.randn(B, S, H, d, sp, generator=g)
    lp = torch.randn(B, S, H, sp, generator=g) * 3
    lp[0, 0, 0, :] = -math.inf                 # a row with no contribution at all
    lp[1, 1, 2, 3] = -math.inf                 # one empty split
    op[1, 1, 2, :, 3] = float("nan")           # whose partial must never be read as a factor
    ro, rl = oracle.combine(op.double().numpy().copy(), lp.double().numpy())
    if layout == "pages":
        opd, lpd = op.to(DEV), lp.to(DEV)
    else:  # [splits, B, S, H, d] storage viewed in the pages' logical order
        opd = op.permute(4, 0, 1, 2, 3).contiguous().to(DEV).permute(1, 2, 3, 4, 0)
        lpd = lp.permute(3, 0, 1, 2).contiguous().to(DEV).permute(1, 2, 3, 0)
    out, lse = fa().fa_combine(opd, lpd, out_dtype=out_dtype)
    torch.cuda.synchronize()
    got = to_np(out)
    tol = {torch.float32: 1e-5, torch.bfloat16: 1e-2, torch.float16: 2e-3}[out_dtype]
    rel = {torch.float32: 1e-6, torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}[out_dtype]
    assert np.all(np.abs(got - ro) <= tol + rel * np.abs(ro))
    check_lse(lse, rl.transpose(0, 2, 1))
    assert np.all(got[0, 0, 0] == 0.0)

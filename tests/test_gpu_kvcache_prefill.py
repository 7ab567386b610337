"""GPU parity of fa_fwd_kvcache with many query rows per KV head (chunked prefill
against a paged or contiguous cache), which runs the tcgen05 prefill kernel with
K/V read through the block table ("flash attention" tag page, section 3.3; the
changelog's v2.5 paged KV cache).  Page tails and spare blocks hold NaN, so any
key or value read past a sequence's end would show in the output."""
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
    assert fa.fa_device_status(clear=True) == 0, "a kernel raised a device status flag"


def fa():
    import io_aware_online_b200 as m
    return m


def run_paged(lens, Sq, H, Hkv, d, dtype, page, seed, **kw):
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, dtype, seed=seed, spare_blocks=3)
    g = torch.Generator().manual_seed(seed + 1)
    q = torch.randn(len(lens), Sq, H, d, generator=g).to(dtype)
    dkw = dict(kw)
    if dkw.get("alibi_slopes") is not None:
        dkw["alibi_slopes"] = dkw["alibi_slopes"].to(DEV)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kp.to(DEV), vp.to(DEV), cache_seqlens=cs.to(DEV),
                                   block_table=bt.to(DEV), **dkw)
    torch.cuda.synchronize()
    okw = {("window" if k == "window_size" else k): v for k, v in kw.items()}
    ro, rl = oracle.attention_paged(q, kp, vp, bt, cs, **okw)
    return out, lse, ro, rl


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float16, 64)],
                         ids=["bf16-d128", "fp16-d64"])
@pytest.mark.parametrize("Sq", [5, 128, 300])
@pytest.mark.parametrize("page", [64, 256])
def test_chunk_against_paged_cache_causal(dtype, d, Sq, page):
    lens = [Sq, 1000, 4097, 333]        # the chunk's own keys are the last Sq of each
    out, lse, ro, rl = run_paged(lens, Sq, 32, 8, d, dtype, page, seed=1200 + Sq + d,
                                 causal=True)
    assert check_out(out, ro, dtype) <= ATOL[dtype]
    check_lse(lse, rl)


@pytest.mark.parametrize("variant", ["noncausal", "window_softcap_alibi", "short_cache"])
def test_chunk_variants(variant):
    H, Hkv, d, Sq = 16, 4, 128, 160
    kw = dict(causal=True)
    lens = [700, 160, 2049]
    if variant == "noncausal":
        kw = dict(causal=False)
    elif variant == "window_softcap_alibi":
        kw = dict(causal=True, window_size=(200, -1), softcap=20.0,
                  alibi_slopes=synth.alibi_slopes(H))
    else:
        lens = [100, 1, 159]            # fewer keys than query rows: leading rows see none
    out, lse, ro, rl = run_paged(lens, Sq, H, Hkv, d, torch.bfloat16, 128, seed=1300, **kw)
    assert check_out(out, ro, torch.bfloat16) <= ATOL[torch.bfloat16]
    check_lse(lse, rl)


def test_contiguous_cache_equals_dense_prefill_bitwise():
    """With every sequence's cache full, attending the contiguous cache equals fa_fwd
    on the same K/V: the same kernel and arithmetic, K/V loaded in 64-row boxes."""
    B, S, Sq, H, Hkv, d = 2, 640, 192, 16, 4, 64
    q, k, v = synth.dense(B, Sq, S, H, Hkv, d, torch.float16, seed=1400)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    cs = torch.full((B,), S, dtype=torch.int32, device=DEV)
    o1, l1 = fa().fa_fwd_kvcache(q, k, v, cache_seqlens=cs, causal=True)
    o2, l2 = fa().fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_chunked_prefill_with_append():
    """Chunked prefill: a chunk of 200 new tokens is appended after each sequence's
    cached keys and attends (causally) the cache including itself."""
    lens, s_new, H, Hkv, d, page = [0, 300, 1024], 200, 32, 8, 128, 64
    dtype = torch.bfloat16
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, dtype, seed=1500, spare_blocks=1)
    need = [(L + s_new + page - 1) // page for L in lens]
    bt = torch.cat([bt, torch.full((3, max(need) - bt.shape[1]), -1, dtype=torch.int32)], 1)
    nxt = kp.shape[0]
    for b, L in enumerate(lens):
        for pg in range((L + page - 1) // page, need[b]):
            bt[b, pg] = nxt
            nxt += 1
    fill = torch.full((nxt - kp.shape[0], page, Hkv, d), float("nan")).to(dtype)
    kp, vp = torch.cat([kp, fill]), torch.cat([vp, fill.clone()])
    g = torch.Generator().manual_seed(1501)
    kn = torch.randn(3, s_new, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(3, s_new, Hkv, d, generator=g).to(dtype)
    q = torch.randn(3, s_new, H, d, generator=g).to(dtype)
    kd, vd = kp.to(DEV), vp.to(DEV)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kd, vd, kn.to(DEV), vn.to(DEV),
                                   cache_seqlens=cs.to(DEV), block_table=bt.to(DEV), causal=True)
    torch.cuda.synchronize()
    ke, ve = oracle.append(kp, vp, kn, vn, cs, bt)
    assert torch.equal(kd.view(torch.int16).cpu(), ke.view(torch.int16))
    ro, rl = oracle.attention_paged(q, ke, ve, bt, cs + s_new, causal=True)
    assert check_out(out, ro, dtype) <= ATOL[dtype]
    check_lse(lse, rl)

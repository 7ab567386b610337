"""GPU parity of the in-place KV-cache append (fa_kvcache_append and
fa_fwd_kvcache_append; "flash attention" tag page, section 3.3, with k and v given).

The cache after the call must equal the oracle's append bit for bit (16-bit
copies: nothing else may change), and the attention over the grown cache must
match the fp64 oracle within the decode tolerances."""
import pytest
import torch

import oracle
import synth
from parity import ATOL, check_lse, check_out

pytestmark = pytest.mark.gpu
DEV = "cuda"
FA_DEV_BAD_LENGTH = 4


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


def bits(t):
    return t.contiguous().view(torch.int16).cpu()


def grown_paged_cache(lens, s_new, page, Hkv, d, dtype, seed):
    """A paged cache for `lens` plus fresh NaN-filled blocks for the pages the
    appended rows open (the block table grows accordingly)."""
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, dtype, seed=seed, spare_blocks=2)
    need = [(L + s_new + page - 1) // page for L in lens]
    width = max(max(need), bt.shape[1])
    bt = torch.cat([bt, torch.full((len(lens), width - bt.shape[1]), -1, dtype=torch.int32)], 1)
    nxt = kp.shape[0]
    for b, L in enumerate(lens):
        for pg in range((L + page - 1) // page, need[b]):
            bt[b, pg] = nxt
            nxt += 1
    fill = torch.full((nxt - kp.shape[0], page, Hkv, d), float("nan")).to(dtype)
    return torch.cat([kp, fill]), torch.cat([vp, fill.clone()]), bt, cs


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float16, 64)],
                         ids=["bf16-d128", "fp16-d64"])
@pytest.mark.parametrize("s_new", [1, 3])
@pytest.mark.parametrize("page,splits", [(64, 0), (256, 4), (64, 1)])
def test_append_then_attend_paged(dtype, d, s_new, page, splits):
    lens = [0, 63, 255, 1000, 64, 7]
    H, Hkv = 32, 8
    if H // Hkv * s_new > 16:
        pytest.skip("more than 16 query rows per KV head")
    kp, vp, bt, cs = grown_paged_cache(lens, s_new, page, Hkv, d, dtype, seed=900 + d + s_new)
    g = torch.Generator().manual_seed(901)
    kn = torch.randn(len(lens), s_new, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(len(lens), s_new, Hkv, d, generator=g).to(dtype)
    q = torch.randn(len(lens), s_new, H, d, generator=g).to(dtype)
    kd, vd, csd = kp.to(DEV), vp.to(DEV), cs.to(DEV)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kd, vd, kn.to(DEV), vn.to(DEV), cache_seqlens=csd,
                                   block_table=bt.to(DEV), causal=True, num_splits=splits)
    torch.cuda.synchronize()
    ke, ve = oracle.append(kp, vp, kn, vn, cs, bt)
    assert torch.equal(bits(kd), bits(ke)) and torch.equal(bits(vd), bits(ve))
    assert torch.equal(csd.cpu(), cs)                       # the caller advances it
    ro, rl = oracle.attention_paged(q, ke, ve, bt, cs + s_new, causal=True)
    dmax = check_out(out, ro, dtype)
    check_lse(lse, rl)
    assert dmax <= ATOL[dtype]
    assert fa().fa_device_status(clear=True) == 0


def test_append_then_attend_contiguous():
    lens = [0, 5, 130, 200]
    B, s_new, H, Hkv, d, sk_max = len(lens), 2, 16, 4, 64, 256
    dtype = torch.float16
    g = torch.Generator().manual_seed(910)
    kc = torch.randn(B, sk_max, Hkv, d, generator=g).to(dtype)
    vc = torch.randn(B, sk_max, Hkv, d, generator=g).to(dtype)
    kn = torch.randn(B, s_new, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(B, s_new, Hkv, d, generator=g).to(dtype)
    q = torch.randn(B, s_new, H, d, generator=g).to(dtype)
    cs = torch.tensor(lens, dtype=torch.int32)
    kd, vd = kc.to(DEV), vc.to(DEV)
    out, lse = fa().fa_fwd_kvcache(q.to(DEV), kd, vd, kn.to(DEV), vn.to(DEV),
                                   cache_seqlens=cs.to(DEV), causal=True)
    torch.cuda.synchronize()
    ke, ve = oracle.append(kc, vc, kn, vn, cs)
    assert torch.equal(bits(kd), bits(ke)) and torch.equal(bits(vd), bits(ve))
    for b, L in enumerate(lens):
        n = L + s_new
        ro, rl = oracle.attention_dense(q[b:b + 1], ke[b:b + 1, :n], ve[b:b + 1, :n], causal=True)
        assert check_out(out[b:b + 1], ro, dtype) <= ATOL[dtype]
        check_lse(lse[b:b + 1], rl)
    assert fa().fa_device_status(clear=True) == 0


def test_append_alone_then_attend_equals_fused_call():
    lens = [100, 256, 3]
    s_new, H, Hkv, d, page = 2, 8, 2, 128, 64
    dtype = torch.bfloat16
    kp, vp, bt, cs = grown_paged_cache(lens, s_new, page, Hkv, d, dtype, seed=920)
    g = torch.Generator().manual_seed(921)
    kn = torch.randn(len(lens), s_new, Hkv, d, generator=g).to(dtype).to(DEV)
    vn = torch.randn(len(lens), s_new, Hkv, d, generator=g).to(dtype).to(DEV)
    q = torch.randn(len(lens), s_new, H, d, generator=g).to(dtype).to(DEV)
    bt_d, cs_d = bt.to(DEV), cs.to(DEV)
    k1, v1 = kp.to(DEV), vp.to(DEV)
    o1, l1 = fa().fa_fwd_kvcache(q, k1, v1, kn, vn, cache_seqlens=cs_d, block_table=bt_d,
                                 causal=True, num_splits=2)
    k2, v2 = kp.to(DEV), vp.to(DEV)
    fa().fa_kvcache_append(k2, v2, kn, vn, cs_d, block_table=bt_d)
    o2, l2 = fa().fa_fwd_kvcache(q, k2, v2, cache_seqlens=cs_d + s_new, block_table=bt_d,
                                 causal=True, num_splits=2)
    torch.cuda.synchronize()
    assert torch.equal(bits(k1), bits(k2)) and torch.equal(bits(v1), bits(v2))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert fa().fa_device_status(clear=True) == 0


def test_append_with_no_query_rows_still_writes():
    lens = [10, 0]
    s_new, H, Hkv, d, page = 4, 8, 2, 64, 64
    dtype = torch.float16
    kp, vp, bt, cs = grown_paged_cache(lens, s_new, page, Hkv, d, dtype, seed=930)
    g = torch.Generator().manual_seed(931)
    kn = torch.randn(2, s_new, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(2, s_new, Hkv, d, generator=g).to(dtype)
    kd, vd = kp.to(DEV), vp.to(DEV)
    q = torch.empty(2, 0, H, d, dtype=dtype, device=DEV)
    fa().fa_fwd_kvcache(q, kd, vd, kn.to(DEV), vn.to(DEV), cache_seqlens=cs.to(DEV),
                        block_table=bt.to(DEV), return_lse=False)
    torch.cuda.synchronize()
    ke, ve = oracle.append(kp, vp, kn, vn, cs, bt)
    assert torch.equal(bits(kd), bits(ke)) and torch.equal(bits(vd), bits(ve))


def test_append_beyond_capacity_is_skipped_and_reported():
    """Rows past the end of the block table are not written; the kernel's own
    bounds check raises FA_DEV_BAD_LENGTH, and the attention clamps its length."""
    page, Hkv, d, H = 64, 2, 128, 8
    dtype = torch.bfloat16
    kp, vp, bt, cs = synth.paged_cache([127, 30], page, Hkv, d, dtype, seed=940)
    g = torch.Generator().manual_seed(941)
    kn = torch.randn(2, 3, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(2, 3, Hkv, d, generator=g).to(dtype)
    q = torch.randn(2, 3, H, d, generator=g).to(dtype)
    kd, vd = kp.to(DEV), vp.to(DEV)
    fa().fa_device_status(clear=True)
    fa().fa_fwd_kvcache(q.to(DEV), kd, vd, kn.to(DEV), vn.to(DEV), cache_seqlens=cs.to(DEV),
                        block_table=bt.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert fa().fa_device_status(clear=True) & FA_DEV_BAD_LENGTH
    # sequence 0 has room for one more key (position 127); sequence 1 for all three
    ke, ve = oracle.append(kp, vp, kn[:, :1], vn[:, :1], cs, bt)
    ke, ve = oracle.append(ke, ve, kn[1:, 1:], vn[1:, 1:], cs[1:] + 1, bt[1:])
    assert torch.equal(bits(kd), bits(ke)) and torch.equal(bits(vd), bits(ve))

"""GPU parity of fa_fwd (dense and varlen prefill) against the fp64 oracle.

Every case draws seeded inputs from ``synth``, runs the CUDA kernel through the
C ABI (python binding) and compares O and LSE element by element with the
oracle on the same 16-bit values.  Sizes span several 128-row tiles and ragged
tails; the full benchmark shapes are covered on sampled rows in
test_gpu_fullsize.py.
"""
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
    assert fa.fa_device_status(clear=True) == 0, "a kernel raised a device status flag"


def run_dense(q, k, v, **kw):
    import io_aware_online_b200 as fa
    out, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


def oracle_dense(q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1), softcap=0.0,
                 alibi_slopes=None):
    return oracle.attention_dense(q, k, v, scale=softmax_scale, causal=causal, window=window_size,
                                  softcap=softcap, alibi_slopes=alibi_slopes)


def compare(q, k, v, **kw):
    out, lse = run_dense(q, k, v, **kw)
    kw_o = dict(kw)
    if kw_o.get("alibi_slopes") is not None:
        kw_o["alibi_slopes"] = kw_o["alibi_slopes"].cpu()
    ro, rl = oracle_dense(q, k, v, **kw_o)
    dmax = check_out(out, ro, q.dtype)
    lmax = check_lse(lse, rl)
    # rows with no allowed key: exactly zero output
    dead = rl == -math.inf                  # [B, H, Sq]
    if dead.any():
        o = to_np(out).transpose(0, 2, 1, 3)  # [B, H, Sq, d]
        assert np.all(o[dead] == 0.0)
    return dmax, lmax


# ------------------------------------------------------------------ named configs
def test_tiny_dense_fp16():
    """B=1, H=2, Sq=Sk=128, d=64, fp16, non-causal, default scale."""
    q, k, v = synth.dense(1, 128, 128, 2, 2, 64, torch.float16, seed=1001)
    dmax, _ = compare(q, k, v)
    assert dmax <= ATOL[torch.float16]


def test_causal_bottom_right_bf16():
    """B=2, H=8, Sq=384, Sk=1024, d=128, bf16, causal (offset 640)."""
    q, k, v = synth.dense(2, 384, 1024, 8, 8, 128, torch.bfloat16, seed=1002)
    dmax, _ = compare(q, k, v, causal=True)
    assert dmax <= ATOL[torch.bfloat16]


def test_decode_step_sq1_sees_all_keys():
    """Sq=1, Sk=1025 causal: the single query attends every key (changelog example)."""
    q, k, v = synth.dense(2, 1, 1025, 8, 8, 128, torch.bfloat16, seed=1012)
    out_c, lse_c = run_dense(q, k, v, causal=True)
    out_n, lse_n = run_dense(q, k, v, causal=False)
    assert torch.equal(out_c, out_n) and torch.equal(lse_c, lse_n)
    compare(q, k, v, causal=True)


# ------------------------------------------------------------------ mask / variant grid
SHAPES = [(1, 200, 333, 4, 2), (2, 129, 129, 2, 2), (1, 300, 70, 2, 1), (1, 1, 257, 4, 4)]
MASKS = [(False, (-1, -1)), (True, (-1, -1)), (False, (64, 32)), (True, (100, -1)),
         (False, (-1, 0)), (True, (0, 0))]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}Sq{}Sk{}H{}kv{}".format(*s))
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: f"c{int(m[0])}w{m[1][0]},{m[1][1]}")
def test_mask_grid(dtype, d, shape, mask):
    B, Sq, Sk, H, Hkv = shape
    causal, window = mask
    q, k, v = synth.dense(B, Sq, Sk, H, Hkv, d, dtype, seed=hash((shape, mask, d)) % 10000)
    compare(q, k, v, causal=causal, window_size=window)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("softcap,alibi", [(30.0, False), (0.0, True), (5.0, True)])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap_alibi(dtype, d, softcap, alibi, causal):
    B, Sq, Sk, H, Hkv = 2, 260, 390, 4, 2
    q, k, v = synth.dense(B, Sq, Sk, H, Hkv, d, dtype, seed=77)
    q = (q.float() * 3).to(dtype)           # larger scores exercise the cap
    slopes = synth.alibi_slopes(H).to(DEV) if alibi else None
    compare(q, k, v, causal=causal, softcap=softcap, alibi_slopes=slopes,
            window_size=(200, -1) if causal else (-1, -1))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_row_max_growing_across_blocks(dtype, d, causal):
    """Every 128-key block raises each row's max by well over 8 (base 2): the
    running max is replaced, and O rescaled, at each block (online softmax,
    FlashAttention-2 section 3.1)."""
    q, k, v = synth.dense(1, 512, 512, 2, 2, d, dtype, seed=1031)
    # a shared direction: q . k gains 2 * a_j with a_j = 40 * (j // 128)
    a = 40.0 * (torch.arange(512) // 128).float()
    q = (q.float() + 2.0).to(dtype)
    k = (k.float() + (a / d)[None, :, None, None]).to(dtype)
    dmax, _ = compare(q, k, v, causal=causal)
    assert dmax <= ATOL[dtype]


def test_more_queries_than_keys_gives_dead_rows():
    q, k, v = synth.dense(1, 300, 100, 2, 2, 64, torch.float16, seed=5)
    compare(q, k, v, causal=True)


def test_explicit_scale_and_zero_scale():
    q, k, v = synth.dense(1, 130, 200, 2, 2, 64, torch.float16, seed=6)
    compare(q, k, v, softmax_scale=0.3)
    compare(q, k, v, softmax_scale=0.0, causal=True)


def test_strided_bhsd_views():
    """Transposed [b, h, s, d] storage passed as [b, s, h, d] views (no copy)."""
    g = torch.Generator().manual_seed(9)
    qt = torch.randn(2, 4, 200, 64, generator=g).to(torch.float16)
    kt = torch.randn(2, 2, 300, 64, generator=g).to(torch.float16)
    vt = torch.randn(2, 2, 300, 64, generator=g).to(torch.float16)
    import io_aware_online_b200 as fa
    qd, kd, vd = (t.to(DEV).transpose(1, 2) for t in (qt, kt, vt))
    assert not qd.is_contiguous()
    out, lse = fa.fa_fwd(qd, kd, vd, causal=True)
    ro, rl = oracle_dense(qt.transpose(1, 2), kt.transpose(1, 2), vt.transpose(1, 2), causal=True)
    check_out(out, ro, torch.float16)
    check_lse(lse, rl)


def test_deterministic_bitwise():
    q, k, v = synth.dense(2, 512, 512, 4, 4, 128, torch.bfloat16, seed=8)
    a = run_dense(q, k, v, causal=True)
    b = run_dense(q, k, v, causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ------------------------------------------------------------------ varlen
def run_varlen(q, k, v, cq, ck, lq, lk, **kw):
    import io_aware_online_b200 as fa
    out, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), cu_seqlens_q=cq.to(DEV),
                         cu_seqlens_k=ck.to(DEV), max_seqlen_q=max(lq), max_seqlen_k=max(lk),
                         **kw)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant", ["plain", "causal", "all"])
def test_varlen(dtype, d, variant):
    lq = [1, 130, 300, 0, 257, 64]
    lk = [5, 130, 450, 3, 0, 600]
    H, Hkv = 4, 2
    q, k, v, cq, ck = synth.varlen(lq, lk, H, Hkv, d, dtype, seed=31)
    kw = {}
    if variant == "causal":
        kw = dict(causal=True)
    elif variant == "all":
        kw = dict(causal=True, window_size=(96, -1), softcap=20.0,
                  alibi_slopes=synth.alibi_slopes(H).to(DEV))
    out, lse = run_varlen(q, k, v, cq, ck, lq, lk, **kw)
    kwo = dict(kw)
    if "alibi_slopes" in kwo:
        kwo["alibi_slopes"] = kwo["alibi_slopes"].cpu()
    ro, rl = oracle.attention(q, k, v, cq, ck, scale=None,
                              causal=kwo.get("causal", False),
                              window=kwo.get("window_size", (-1, -1)),
                              softcap=kwo.get("softcap", 0.0),
                              alibi_slopes=kwo.get("alibi_slopes"))
    check_out(out, ro, dtype)
    check_lse(lse, rl.T)


def test_varlen_pages_example_equals_dense_calls():
    """Section 3.2 example: lengths [512, 1024, 768] packed; equals three dense calls."""
    lens = [512, 1024, 768]
    q, k, v, cq, ck = synth.varlen(lens, lens, 8, 8, 64, torch.float16, seed=3)
    assert cq.tolist() == [0, 512, 1536, 2304]
    out, lse = run_varlen(q, k, v, cq, ck, lens, lens, causal=True)
    for b, L in enumerate(lens):
        s = slice(int(cq[b]), int(cq[b + 1]))
        o1, l1 = run_dense(q[s][None], k[s][None], v[s][None], causal=True)
        assert torch.equal(out[s], o1[0])
        assert torch.equal(lse[:, s], l1[0])

"""GPU parity of fa_fwd_fp8 (E4M3 q, k, v; "FlashAttention common interfaces",
workflow three: cast the inputs to float8 and call the same function).

The reference is the fp64 oracle on the dequantised inputs (q8 * q_descale, ...),
which the kernel sees exactly.  The kernel rounds P to E4M3 before P.V, so O may
differ from it by the bound stated in include/fa.h, evaluated element by element:

    |dO_ic| <= 2^-4 * sum_j w_ij |v_jc| + n_k * 2^-18 * max_j |v_jc|
               + 2^-8 * |O_ic| (bf16 output) + 1e-5

with w the exact attention weights; sum_j w_ij |v_jc| is the oracle's output for
|V| in place of V.  The LSE comes from the exact fp32 sum (tolerance as for the
16-bit paths).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_lse

pytestmark = pytest.mark.gpu
DEV = "cuda"
E4M3 = torch.float8_e4m3fn


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


def quantise(x, descale):
    """Real tensor -> (E4M3 tensor, its exact dequantised fp32 value)."""
    x8 = (x.float() / descale).to(E4M3)
    return x8, x8.float() * descale


def check_fp8(out, ref, ref_absv, vmax, n_k):
    o = out.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    tol = (2.0 ** -4) * np.asarray(ref_absv) + n_k * 2.0 ** -18 * vmax \
        + 2.0 ** -8 * np.abs(ref) + 1e-5
    err = np.abs(o - ref)
    assert np.all(np.isfinite(o))
    worst = np.max(err - tol)
    assert worst <= 0.0, f"exceeds the E4M3 bound by {worst:.3g}"
    # rounding errors of many probabilities largely cancel: far inside the bound
    assert err.mean() <= 0.5 * tol.mean()
    return float(err.max())


def run_dense(B, Sq, Sk, H, Hkv, descales, seed, **kw):
    q, k, v = synth.dense(B, Sq, Sk, H, Hkv, 128, torch.float32, seed=seed)
    (q8, qd), (k8, kd), (v8, vd) = (quantise(x, s) for x, s in zip((q, k, v), descales))
    dkw = dict(kw)
    if dkw.get("alibi_slopes") is not None:
        dkw["alibi_slopes"] = dkw["alibi_slopes"].to(DEV)
    out, lse = fa().fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), q_descale=descales[0],
                               k_descale=descales[1], v_descale=descales[2], **dkw)
    torch.cuda.synchronize()
    okw = {("window" if kk == "window_size" else kk): vv for kk, vv in kw.items()}
    ro, rl = oracle.attention_dense(qd, kd, vd, **okw)
    ra, _ = oracle.attention_dense(qd, kd, vd.abs(), **okw)
    vmax = float(vd.abs().max())
    return out, lse, ro, rl, ra, vmax


@pytest.mark.parametrize("causal", [True, False])
def test_plain_cast_dense(causal):
    """Descale 1: the pages' q.to(torch.float8_e4m3fn) workflow."""
    out, lse, ro, rl, ra, vmax = run_dense(2, 600, 600, 8, 8, (1.0, 1.0, 1.0), 1700,
                                           causal=causal)
    assert out.dtype == torch.bfloat16
    check_fp8(out, ro, ra, vmax, 600)
    check_lse(lse.cpu(), rl)


def test_descales_gqa_bottom_right():
    out, lse, ro, rl, ra, vmax = run_dense(2, 384, 1000, 16, 4, (0.5, 2.0, 0.25), 1701,
                                           causal=True)
    check_fp8(out, ro, ra, vmax, 1000)
    check_lse(lse.cpu(), rl)


def test_window_softcap_alibi():
    H = 8
    out, lse, ro, rl, ra, vmax = run_dense(1, 300, 700, H, 2, (1.0, 1.0, 1.0), 1702,
                                           causal=True, window_size=(128, -1), softcap=10.0,
                                           alibi_slopes=synth.alibi_slopes(H))
    check_fp8(out, ro, ra, vmax, 700)
    check_lse(lse.cpu(), rl)


def test_dead_rows_and_growing_max():
    """More queries than keys (causal): leading rows see no key, O = 0, LSE = -inf.
    Scores rise block by block, so the running max moves at every block."""
    B, S, Sk, H = 1, 512, 384, 2
    q, k, v = synth.dense(B, S, Sk, H, H, 128, torch.float32, seed=1703)
    a = 30.0 * (torch.arange(Sk) // 128).float()
    q = q + 1.0
    k = k + (a / 128)[None, :, None, None]
    (q8, qd), (k8, kd), (v8, vd) = (quantise(x, 1.0) for x in (q, k, v))
    out, lse = fa().fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_dense(qd, kd, vd, causal=True)
    ra, _ = oracle.attention_dense(qd, kd, vd.abs(), causal=True)
    check_fp8(out, ro, ra, float(vd.abs().max()), Sk)
    dead = rl == -math.inf
    assert dead.any()
    o = out.float().cpu().numpy().transpose(0, 2, 1, 3)
    assert np.all(o[dead] == 0.0)
    check_lse(lse.cpu(), rl)


def test_slowly_growing_max_within_the_lazy_threshold():
    """Each 128-key block raises the rows' scores by about 0.6 (log2 units), under the
    0.8 threshold of the lazy running max: the running max is often stale, P then goes
    above 2^8 (up to 2^8.8 < 448, E4M3's largest) without a rescale, and every few
    blocks the accumulated growth forces one.  The stated bound must hold throughout."""
    B, S, H, d = 1, 1024, 2, 128
    q, k, v = synth.dense(B, S, S, H, H, d, torch.float32, seed=1705)
    # q . k gains about 128 * 0.037 = 4.7 per block: 0.6 in log2 units at scale d^-1/2
    step = 0.6 * math.log(2.0) / (d ** -0.5) / d
    a = step * (torch.arange(S) // 128).float()
    q = q * 0.25 + 1.0
    k = k * 0.25 + a[None, :, None, None]
    (q8, qd), (k8, kd), (v8, vd) = (quantise(x, 1.0) for x in (q, k, v))
    for causal in (False, True):
        out, lse = fa().fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), causal=causal)
        torch.cuda.synchronize()
        ro, rl = oracle.attention_dense(qd, kd, vd, causal=causal)
        ra, _ = oracle.attention_dense(qd, kd, vd.abs(), causal=causal)
        check_fp8(out, ro, ra, float(vd.abs().max()), S)
        check_lse(lse.cpu(), rl)


def test_varlen():
    lq = [1, 130, 300]
    q, k, v, cq, ck = synth.varlen(lq, lq, 8, 2, 128, dtype=torch.float32, seed=1704)
    (q8, qd), (k8, kd), (v8, vd) = (quantise(x, 1.0) for x in (q, k, v))
    out, lse = fa().fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), cu_seqlens_q=cq.to(DEV),
                               cu_seqlens_k=ck.to(DEV), max_seqlen_q=max(lq),
                               max_seqlen_k=max(lq), causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(qd, kd, vd, cq, ck, causal=True)
    ra, _ = oracle.attention(qd, kd, vd.abs(), cq, ck, causal=True)
    check_fp8(out, ro, ra, float(vd.abs().max()), max(lq))
    check_lse(lse.cpu(), rl.T)                  # kernel [H, total_q], oracle [total_q, H]


def test_fp8_rejects_other_head_dims():
    import io_aware_online_b200 as m
    q = torch.zeros(1, 128, 2, 64, dtype=E4M3, device=DEV)
    with pytest.raises(m.FAError):
        m.fa_fwd_fp8(q, q, q)

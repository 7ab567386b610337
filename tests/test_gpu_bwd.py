"""GPU parity of fa_bwd (dQ, dK, dV) against the fp64 backward oracle.

The kernel is given the oracle's O (rounded to the input dtype) and LSE, so that
only the backward's own arithmetic is checked.  Its rounding steps, with u the
unit roundoff of the input dtype (2^-11 fp16, 2^-8 bf16), give the per-element
bound used here (doubled for the compounding of two roundings, plus a floor for
fp32 accumulation and the approximate exp2):

    dD_i  = u * sum_c |dO_ic| |O_ic|                  (D from the rounded O)
    |ddV| <= u * sum_i P_ij |dO_ic|  + u |dV|          (P rounded before P^T dO)
    |ddK| <= scale * sum_i (u |dS_ij| + P_ij dD_i) |Q_ic| + u |dK|
    |ddQ| <= scale * sum_j (u |dS_ij| + P_ij dD_i) |K_jc| + u |dQ|

P and dS are the oracle's exact values.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


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


def f64(t):
    return t.detach().float().cpu().double().numpy()


def bounds(q, k, do, o, P, dS, dq, dk, dv, scale, G, u):
    """Per-element tolerances of dq, dk, dv (see the module docstring)."""
    q, k, do, o = f64(q), f64(k), f64(do), np.asarray(o)
    B, Sq, H, d = q.shape
    Hkv = k.shape[2]
    tq = np.zeros_like(q)
    tk = np.zeros((B, k.shape[1], Hkv, d))
    tv = np.zeros_like(tk)
    for b in range(B):
        for h in range(H):
            hk = h // G
            dD = u * (np.abs(do[b, :, h]) * np.abs(o[b, :, h])).sum(axis=1)   # [Sq]
            W = u * np.abs(dS[b, h]) + P[b, h] * dD[:, None]                    # [Sq, Sk]
            tq[b, :, h] = scale * W @ np.abs(k[b, :, hk])
            tk[b, :, hk] += scale * W.T @ np.abs(q[b, :, h])
            tv[b, :, hk] += u * P[b, h].T @ np.abs(do[b, :, h])
    fl = 1e-5
    return (2 * (tq + u * np.abs(dq)) + fl * max(1.0, np.abs(dq).max()),
            2 * (tk + u * np.abs(dk)) + fl * max(1.0, np.abs(dk).max()),
            2 * (tv + u * np.abs(dv)) + fl * max(1.0, np.abs(dv).max()))


def check(name, got, ref, tol):
    g = f64(got)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    err = np.abs(g - ref)
    worst = np.max(err - tol)
    assert worst <= 0.0, f"{name}: exceeds its bound by {worst:.3g} (max err {err.max():.3g})"


def run_case(B, Sq, Sk, H, Hkv, d, dtype, seed, scale=None, **kw):
    q, k, v = synth.dense(B, Sq, Sk, H, Hkv, d, dtype, seed=seed)
    do = synth.randn((B, Sq, H, d), dtype, torch.Generator().manual_seed(seed + 5))
    okw = {("window" if kk == "window_size" else kk): vv for kk, vv in kw.items()}
    dq_r, dk_r, dv_r, o_r, lse_r, P, dS = oracle.attention_backward(q, k, v, do, scale=scale,
                                                                    return_probs=True, **okw)
    o16 = torch.from_numpy(o_r).to(dtype)
    lse = torch.from_numpy(lse_r).float()
    dkw = dict(kw)
    if dkw.get("alibi_slopes") is not None:
        dkw["alibi_slopes"] = dkw["alibi_slopes"].to(DEV)
    dq, dk, dv = fa().fa_bwd(do.to(DEV), q.to(DEV), k.to(DEV), v.to(DEV), o16.to(DEV),
                             lse.to(DEV), softmax_scale=scale, **dkw)
    torch.cuda.synchronize()
    sc = scale if scale is not None else d ** -0.5
    # the kernel computes D from the rounded O it is given: bound against that O
    tq, tk, tv = bounds(q, k, do, f64(o16), P, dS, dq_r, dk_r, dv_r, sc, H // Hkv, U[dtype])
    check("dq", dq, dq_r, tq)
    check("dk", dk, dk_r, tk)
    check("dv", dv, dv_r, tv)
    return dq, dk, dv


def test_dense_fp16_d64():
    run_case(1, 300, 300, 2, 2, 64, torch.float16, 1800)


def test_causal_bf16_d128():
    run_case(1, 384, 384, 4, 4, 128, torch.bfloat16, 1801, causal=True)


def test_gqa_bottom_right_window_fp16_d128():
    run_case(2, 200, 520, 8, 2, 128, torch.float16, 1802, causal=True, window_size=(100, -1))


def test_alibi_bf16_d64():
    run_case(1, 256, 256, 4, 4, 64, torch.bfloat16, 1803, causal=True,
             alibi_slopes=synth.alibi_slopes(4))


def test_dead_rows_get_zero_dq():
    dq, _, _ = run_case(1, 300, 130, 2, 2, 64, torch.float16, 1804, causal=True)
    assert torch.all(dq[0, :170].float() == 0)


def test_deterministic():
    q, k, v = synth.dense(1, 256, 256, 2, 2, 64, torch.bfloat16, seed=1805)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = fa().fa_fwd(q, k, v, causal=True)
    do = torch.randn_like(q)
    a = fa().fa_bwd(do, q, k, v, out, lse, causal=True)
    b = fa().fa_bwd(do, q, k, v, out, lse, causal=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_forward_then_backward_matches_oracle():
    """Integration: fa_fwd's own O and LSE feed fa_bwd.  The forward's rounding of O
    (within its parity tolerance) enters D, so this checks the relative error norm
    (1e-2 for bf16) instead of the element bound."""
    B, S, H, d = 1, 512, 4, 128
    q, k, v = synth.dense(B, S, S, H, H, d, torch.bfloat16, seed=1806)
    do = synth.randn((B, S, H, d), torch.bfloat16, torch.Generator().manual_seed(1807))
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = fa().fa_fwd(qd, kd, vd, causal=True)
    dq, dk, dv = fa().fa_bwd(do.to(DEV), qd, kd, vd, out, lse, causal=True)
    torch.cuda.synchronize()
    dq_r, dk_r, dv_r, _, _ = oracle.attention_backward(q, k, v, do, causal=True)
    for name, got, ref in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        rel = np.linalg.norm(f64(got) - ref) / np.linalg.norm(ref)
        assert rel <= 1e-2, f"{name}: relative error {rel:.3g}"

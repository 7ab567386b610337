"""GPU parity of fa_bwd (dQ, dK, dV) against the fp64 backward oracle.

The kernel is given the oracle's O (rounded to the input dtype) and LSE, so that
only the backward's own arithmetic is checked.  Its rounding steps, with u the
unit roundoff of the input dtype (2^-11 fp16, 2^-8 bf16), give the per-element
bound used here (doubled for the compounding of two roundings, plus a floor for
fp32 accumulation and the approximate exp2):

    dD_i  = u * sum_c |dO_ic| |O_ic|                  (D from the rounded O)
    |ddV| <= u * sum_i P_ij |dO_ic|  + u |dV|          (P rounded before P^T dO)
    |ddK| <= scale * sum_i (u |dX_ij| + P_ij dD_i) |Q_ic| + u |dK|
    |ddQ| <= scale * sum_j (u |dX_ij| + P_ij dD_i) |K_jc| + u |dQ|

P and dX (the gradient with respect to scale Q K^T: dS, times 1 - tanh^2 under a
softcap, whose factor is at most 1) are the oracle's exact values.  Varlen cases
take these bounds sequence by sequence.
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


def test_long_gqa_causal_bf16_d128():
    """Four query heads per KV head over 9 query blocks: the dK/dV kernel streams up to
    36 (head, query block) iterations through its 3-slot Q and 2-slot dO rings, so every
    slot and barrier phase comes round many times."""
    run_case(1, 1100, 1100, 4, 1, 128, torch.bfloat16, 1810, causal=True)


def test_long_gqa_window_fp16_d64():
    run_case(1, 1000, 1000, 8, 2, 64, torch.float16, 1811, window_size=(300, 50))


def test_grid_groups_end_ragged_fp16_d64():
    """Nine (sequence, KV head) pairs for the dK/dV CTAs and eighteen (sequence, head)
    pairs for the dQ CTAs: the grid's groups of eight pairs end on a partial group in
    both passes, with three blocks per pair."""
    run_case(3, 300, 300, 6, 3, 64, torch.float16, 1812, causal=True)


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


def test_softcap_causal_bf16_d128():
    """softcap 2: most scores sit on the curved part of c tanh(x / c)."""
    run_case(1, 384, 384, 4, 2, 128, torch.bfloat16, 1810, causal=True, softcap=2.0)


def test_softcap_alibi_window_fp16_d64():
    run_case(1, 320, 320, 4, 4, 64, torch.float16, 1811, causal=True, window_size=(150, -1),
             softcap=3.0, alibi_slopes=synth.alibi_slopes(4))


def run_varlen(lq, lk, H, Hkv, d, dtype, seed, **kw):
    """Packed sequences (section 3.2): each sequence against the dense oracle on its
    own rows, with that sequence's bounds."""
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lq), sum(lk)
    q = synth.randn((tq, H, d), dtype, g)
    k = synth.randn((tk, Hkv, d), dtype, g)
    v = synth.randn((tk, Hkv, d), dtype, g)
    do = synth.randn((tq, H, d), dtype, g)
    cu_q, cu_k = synth.cu_seqlens(lq), synth.cu_seqlens(lk)
    okw = {("window" if kk == "window_size" else kk): vv for kk, vv in kw.items()}
    o_r, l_r = np.zeros((tq, H, d)), np.full((H, tq), -np.inf)
    refs = []
    for b in range(len(lq)):
        qa, qb, ka, kb = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if qb == qa or kb == ka:
            refs.append(None)
            continue
        r = oracle.attention_backward(q[None, qa:qb], k[None, ka:kb], v[None, ka:kb],
                                      do[None, qa:qb], return_probs=True, **okw)
        refs.append(r)
        o_r[qa:qb], l_r[:, qa:qb] = r[3][0], r[4][0]
    o16 = torch.from_numpy(o_r).to(dtype)
    dkw = dict(kw)
    if dkw.get("alibi_slopes") is not None:
        dkw["alibi_slopes"] = dkw["alibi_slopes"].to(DEV)
    dq, dk, dv = fa().fa_bwd(do.to(DEV), q.to(DEV), k.to(DEV), v.to(DEV), o16.to(DEV),
                             torch.from_numpy(l_r).float().contiguous().to(DEV),
                             cu_seqlens_q=cu_q.to(DEV), cu_seqlens_k=cu_k.to(DEV),
                             max_seqlen_q=max(lq), max_seqlen_k=max(lk), **dkw)
    torch.cuda.synchronize()
    sc = d ** -0.5
    for b, r in enumerate(refs):
        qa, qb, ka, kb = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if r is None:
            # no keys or no queries: the gradients of the sequence's rows are zero
            assert torch.all(dq[qa:qb].float() == 0) and torch.all(dk[ka:kb].float() == 0)
            assert torch.all(dv[ka:kb].float() == 0)
            continue
        dq_r, dk_r, dv_r, _, _, P, dX = r
        tq_, tk_, tv_ = bounds(q[None, qa:qb], k[None, ka:kb], do[None, qa:qb],
                               f64(o16[None, qa:qb]), P, dX, dq_r, dk_r, dv_r, sc, H // Hkv,
                               U[dtype])
        check(f"dq[seq {b}]", dq[None, qa:qb], dq_r, tq_)
        check(f"dk[seq {b}]", dk[None, ka:kb], dk_r, tk_)
        check(f"dv[seq {b}]", dv[None, ka:kb], dv_r, tv_)


def test_varlen_causal_bf16_d128():
    # lengths off the 128 grid, more keys than queries, a one-row sequence, and a
    # sequence longer than two blocks
    run_varlen([1, 130, 300, 64], [1, 257, 300, 200], 4, 2, 128, torch.bfloat16, 1820,
               causal=True)


def test_varlen_softcap_window_fp16_d64():
    run_varlen([200, 77, 129], [200, 150, 129], 4, 4, 64, torch.float16, 1821, causal=True,
               window_size=(64, -1), softcap=5.0)


def test_varlen_matches_dense_per_sequence_bitwise():
    """A packed batch gives, row for row, the bits of separate dense calls."""
    lq = [150, 260]
    g = torch.Generator().manual_seed(1822)
    H, d, dt = 2, 64, torch.bfloat16
    q, k, v, do = (synth.randn((sum(lq), H, d), dt, g) for _ in range(4))
    cu = synth.cu_seqlens(lq)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    out, lse = fa().fa_fwd(qd, kd, vd, cu_seqlens_q=cu.to(DEV), cu_seqlens_k=cu.to(DEV),
                           max_seqlen_q=max(lq), max_seqlen_k=max(lq), causal=True)
    dq, dk, dv = fa().fa_bwd(dod, qd, kd, vd, out, lse, cu_seqlens_q=cu.to(DEV),
                             cu_seqlens_k=cu.to(DEV), max_seqlen_q=max(lq),
                             max_seqlen_k=max(lq), causal=True)
    for b in range(len(lq)):
        a, e = int(cu[b]), int(cu[b + 1])
        sl = slice(a, e)
        # the same forward outputs, sliced: only the backward is compared
        o1 = out[None, sl].contiguous()
        l1 = lse[:, sl][None].contiguous()
        g1 = fa().fa_bwd(dod[None, sl].contiguous(), qd[None, sl].contiguous(),
                         kd[None, sl].contiguous(), vd[None, sl].contiguous(), o1, l1,
                         causal=True)
        torch.cuda.synchronize()
        for name, x, y in (("dq", dq, g1[0]), ("dk", dk, g1[1]), ("dv", dv, g1[2])):
            assert torch.equal(x[sl], y[0]), f"{name}: sequence {b} differs from its dense call"

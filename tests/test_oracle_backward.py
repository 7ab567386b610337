"""Pins for the fp64 backward oracle (CPU only): central finite differences of the
pinned forward oracle (dense, softcap and varlen forms), torch's float64 autograd
through scaled_dot_product_attention (a library routine), and torch autograd of
the softcapped scores written with torch.tanh -- none shares code with
oracle/backward.py."""
import numpy as np
import pytest
import torch

import oracle


def loss_grads_fd(q, k, v, do, h=1e-6, **kw):
    """Central differences of L = sum(O * dO), O from the C forward oracle."""
    def L(qq, kk, vv):
        o, _ = oracle.attention_dense(qq, kk, vv, **kw)
        return float((o * do).sum())
    grads = []
    for x in (q, k, v):
        g = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            g[idx] = (L(*args_p) - L(*args_m)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("kw", [dict(), dict(causal=True), dict(causal=True, window=(2, -1)),
                                dict(window=(1, 1)),
                                dict(causal=True, alibi_slopes=np.array([0.5, 0.125])),
                                dict(alibi_slopes=np.array([0.25, 1.0]), scale=0.7),
                                dict(softcap=1.5), dict(softcap=0.8, causal=True),
                                dict(softcap=2.0, causal=True,
                                     alibi_slopes=np.array([0.5, 0.25]), scale=0.9)],
                         ids=["plain", "causal", "causal-window", "window", "causal-alibi",
                              "alibi-scale", "softcap", "softcap-causal",
                              "softcap-causal-alibi"])
def test_backward_matches_finite_differences(kw):
    rng = np.random.default_rng(7)
    B, Sq, Sk, H, Hkv, d = 1, 4, 6, 2, 1, 3
    q = rng.standard_normal((B, Sq, H, d))
    k = rng.standard_normal((B, Sk, Hkv, d))
    v = rng.standard_normal((B, Sk, Hkv, d))
    do = rng.standard_normal((B, Sq, H, d))
    dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, do, **kw)
    fq, fk, fv = loss_grads_fd(q, k, v, do, **kw)
    np.testing.assert_allclose(dq, fq, atol=1e-7, rtol=1e-6)
    np.testing.assert_allclose(dk, fk, atol=1e-7, rtol=1e-6)
    np.testing.assert_allclose(dv, fv, atol=1e-7, rtol=1e-6)
    o_ref, l_ref = oracle.attention_dense(q, k, v, **kw)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_backward_matches_torch_autograd_gqa_causal():
    g = torch.Generator().manual_seed(11)
    B, S, H, Hkv, d = 2, 37, 4, 2, 16
    q = torch.randn(B, S, H, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, S, H, d, generator=g, dtype=torch.float64)
    dq, dk, dv, o, _ = oracle.attention_backward(q, k, v, do, causal=True, scale=0.3)
    qt, kt, vt = (x.transpose(1, 2).clone().requires_grad_(True) for x in (q, k, v))
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.3,
                                                          enable_gqa=True)
    ot.backward(do.transpose(1, 2))
    np.testing.assert_allclose(o, ot.detach().transpose(1, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, qt.grad.transpose(1, 2).numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, kt.grad.transpose(1, 2).numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, vt.grad.transpose(1, 2).numpy(), atol=1e-10)


def test_rows_without_keys_have_zero_gradient():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 6, 1, 4))
    k = rng.standard_normal((1, 3, 1, 4))
    v = rng.standard_normal((1, 3, 1, 4))
    do = rng.standard_normal((1, 6, 1, 4))
    dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, do, causal=True)
    assert np.all(np.isneginf(lse[0, 0, :3])) and np.all(dq[0, :3] == 0.0)
    assert np.all(o[0, :3] == 0.0)


def test_softcap_backward_matches_torch_autograd_of_tanh_scores():
    """S = c tanh(scale Q K^T / c) with a causal mask, differentiated by torch."""
    g = torch.Generator().manual_seed(12)
    B, S, H, Hkv, d, c, scale = 1, 23, 4, 2, 8, 1.7, 0.45
    q = torch.randn(B, S, H, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, S, H, d, generator=g, dtype=torch.float64)
    dq, dk, dv, o, _ = oracle.attention_backward(q, k, v, do, causal=True, scale=scale,
                                                 softcap=c)
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    kr = kt.repeat_interleave(H // Hkv, dim=2)
    vr = vt.repeat_interleave(H // Hkv, dim=2)
    x = torch.einsum("bihd,bjhd->bhij", qt, kr) * scale
    s = c * torch.tanh(x / c)
    s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    ot = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1), vr)
    ot.backward(do)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-10)


@pytest.mark.parametrize("kw", [dict(causal=True), dict(softcap=1.2, causal=True),
                                dict(window=(2, 0))], ids=["causal", "softcap", "window"])
def test_varlen_backward_matches_finite_differences(kw):
    """Packed sequences (section 3.2) against central differences of the C varlen
    forward oracle; one sequence has more queries than keys (rows without keys)."""
    rng = np.random.default_rng(21)
    lq, lk = [3, 2, 4], [5, 1, 4]
    cu_q = np.cumsum([0] + lq)
    cu_k = np.cumsum([0] + lk)
    H, Hkv, d = 2, 1, 3
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], Hkv, d))
    v = rng.standard_normal((cu_k[-1], Hkv, d))
    do = rng.standard_normal((cu_q[-1], H, d))
    dq, dk, dv, o, lse = oracle.attention_backward_varlen(q, k, v, do, cu_q, cu_k, **kw)
    o_ref, l_ref = oracle.attention(q, k, v, cu_q, cu_k, **kw)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref.T, atol=1e-12)

    def L(qq, kk, vv):
        oo, _ = oracle.attention(qq, kk, vv, cu_q, cu_k, **kw)
        return float((oo * do).sum())
    h = 1e-6
    for x, gx in ((q, dq), (k, dk), (v, dv)):
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            ap = [xp if y is x else y for y in (q, k, v)]
            am = [xm if y is x else y for y in (q, k, v)]
            fd = (L(*ap) - L(*am)) / (2 * h)
            assert abs(gx[idx] - fd) <= 1e-7 + 1e-6 * abs(fd), (idx, gx[idx], fd)

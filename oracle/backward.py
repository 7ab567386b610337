"""fp64 oracle of the attention backward pass -- TEST INFRASTRUCTURE ONLY.

The gradients of O = softmax(mask(softcap(scale Q K^T)) + ALiBi) V with respect
to Q, K and V for a given output gradient dO, written out from their definition
(the tag page "flash attention": the backward recomputes the attention matrix
from Q, K and the saved softmax statistics instead of storing it; the formulas
below are the chain rule through softmax and, with a softcap c > 0 (changelog
v2.6; "FlashAttention common interfaces" section 5.2), through c tanh(x / c),
whose derivative is 1 - tanh(x / c)^2):

    X  = scale * Q K^T
    T  = tanh(X / c),  S = c T (+ bias)       (c = 0: S = X + bias)
    P  = softmax_j(S), masked entries -inf
    dV = P^T dO
    dP = dO V^T
    D  = rowsum(dO * O)          (= sum_j P_ij dP_ij)
    dS = P * (dP - D)
    dX = dS * (1 - T^2)          (c = 0: dX = dS)
    dQ = scale * dX K,   dK = scale * dX^T Q

Rows with no allowed key have P = 0 (and contribute nothing).  GQA: the K/V
gradients of a KV head are the sums over the query heads that read it.  Varlen
batches ("FlashAttention common interfaces" section 3.2: sequences packed along
the rows, offsets in cu_seqlens) are the dense definition applied to each
sequence's rows in turn.  Plain numpy in float64, one (batch, head) at a time; a
matrix product is the only library step.
"""
from __future__ import annotations

import math

import numpy as np


def _np64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def _allowed(Sq, Sk, causal, window):
    """Boolean [Sq, Sk]: key j allowed for query i (bottom-right aligned)."""
    wl, wr = window
    i = np.arange(Sq)[:, None] + (Sk - Sq)
    j = np.arange(Sk)[None, :]
    ok = np.ones((Sq, Sk), dtype=bool)
    if causal:
        ok &= j <= i
    if wl >= 0:
        ok &= j >= i - wl
    if wr >= 0:
        ok &= j <= i + wr
    return ok


def attention_backward(q, k, v, do, *, scale=None, causal=False, window=(-1, -1),
                       softcap=0.0, alibi_slopes=None, return_probs=False):
    """q [B, Sq, H, d], k/v [B, Sk, Hkv, d], do like q.
    Returns (dq like q, dk, dv like k, o like q, lse [B, H, Sq]) in float64, and
    with return_probs also P and dX [B, H, Sq, Sk] (the gradient with respect to
    scale Q K^T: dS, times 1 - T^2 under a softcap)."""
    q, k, v, do = _np64(q), _np64(k), _np64(v), _np64(do)
    B, Sq, H, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    slopes = None if alibi_slopes is None else _np64(alibi_slopes).reshape(H)
    ok = _allowed(Sq, Sk, causal, window)
    dist = np.abs(np.arange(Sq)[:, None] + (Sk - Sq) - np.arange(Sk)[None, :])
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.zeros_like(q)
    lse = np.full((B, H, Sq), -np.inf)
    probs = np.zeros((B, H, Sq, Sk)) if return_probs else None
    dss = np.zeros((B, H, Sq, Sk)) if return_probs else None
    for b in range(B):
        for h in range(H):
            hk = h // G
            Q, K, V, dO = q[b, :, h], k[b, :, hk], v[b, :, hk], do[b, :, h]
            X = scale * (Q @ K.T)
            if softcap > 0:
                T = np.tanh(X / softcap)
                S = softcap * T
            else:
                S = X
            if slopes is not None:
                S = S - slopes[h] * dist
            S = np.where(ok, S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            live = np.isfinite(m[:, 0])
            E = np.where(ok, np.exp(S - np.where(live[:, None], m, 0.0)), 0.0)
            den = E.sum(axis=1, keepdims=True)
            P = np.where(live[:, None], E / np.where(live[:, None], den, 1.0), 0.0)
            O = P @ V
            dP = dO @ V.T
            D = (dO * O).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dX = dS * (1.0 - T * T) if softcap > 0 else dS
            dq[b, :, h] = scale * (dX @ K)
            dk[b, :, hk] += scale * (dX.T @ Q)
            dv[b, :, hk] += P.T @ dO
            o[b, :, h] = O
            if return_probs:
                probs[b, h] = P
                dss[b, h] = dX
            lse[b, h] = np.where(live, m[:, 0] + np.log(np.where(live, den[:, 0], 1.0)),
                                 -np.inf)
    if return_probs:
        return dq, dk, dv, o, lse, probs, dss
    return dq, dk, dv, o, lse


def attention_backward_varlen(q, k, v, do, cu_q, cu_k, **kw):
    """Packed rows: q/do [total_q, H, d], k/v [total_k, Hkv, d], cu_q/cu_k [nseq + 1].
    Returns (dq, dk, dv, o, lse [H, total_q]) in float64: sequence b is the dense
    problem on rows cu_q[b] .. cu_q[b+1]-1 and cu_k[b] .. cu_k[b+1]-1 (its mask
    aligned bottom-right within the sequence)."""
    q, k, v, do = _np64(q), _np64(k), _np64(v), _np64(do)
    cu_q = [int(x) for x in _np64(cu_q)]
    cu_k = [int(x) for x in _np64(cu_k)]
    H = q.shape[1]
    dq, dk, dv, o = (np.zeros_like(x) for x in (q, k, v, q))
    lse = np.full((H, q.shape[0]), -np.inf)
    for b in range(len(cu_q) - 1):
        qa, qb, ka, kb = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if qb == qa:
            continue
        if kb == ka:  # no keys at all: O = 0, LSE = -inf, zero gradients
            continue
        gq, gk, gv, go, gl = attention_backward(q[None, qa:qb], k[None, ka:kb], v[None, ka:kb],
                                                do[None, qa:qb], **kw)
        dq[qa:qb], dk[ka:kb], dv[ka:kb], o[qa:qb] = gq[0], gk[0], gv[0], go[0]
        lse[:, qa:qb] = gl[0]
    return dq, dk, dv, o, lse

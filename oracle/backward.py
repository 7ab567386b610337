"""fp64 oracle of the attention backward pass -- TEST INFRASTRUCTURE ONLY.

The gradients of O = softmax(mask(scale Q K^T) + ALiBi) V with respect to Q, K
and V for a given output gradient dO, written out from their definition (the
tag page "flash attention": the backward recomputes the attention matrix from Q,
K and the saved softmax statistics instead of storing it; the formulas below
are the chain rule through softmax):

    P  = softmax_j(S),  S = scale * Q K^T + bias, masked entries -inf
    dV = P^T dO
    dP = dO V^T
    D  = rowsum(dO * O)          (= sum_j P_ij dP_ij)
    dS = P * (dP - D)
    dQ = scale * dS K,   dK = scale * dS^T Q

Rows with no allowed key have P = 0 (and contribute nothing).  GQA: the K/V
gradients of a KV head are the sums over the query heads that read it.  Plain
numpy in float64, one (batch, head) at a time; a matrix product is the only
library step.
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
                       alibi_slopes=None, return_probs=False):
    """q [B, Sq, H, d], k/v [B, Sk, Hkv, d], do like q.
    Returns (dq like q, dk, dv like k, o like q, lse [B, H, Sq]) in float64, and
    with return_probs also P and dS [B, H, Sq, Sk]."""
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
            S = scale * (Q @ K.T)
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
            dq[b, :, h] = scale * (dS @ K)
            dk[b, :, hk] += scale * (dS.T @ Q)
            dv[b, :, hk] += P.T @ dO
            o[b, :, h] = O
            if return_probs:
                probs[b, h] = P
                dss[b, h] = dS
            lse[b, h] = np.where(live, m[:, 0] + np.log(np.where(live, den[:, 0], 1.0)),
                                 -np.inf)
    if return_probs:
        return dq, dk, dv, o, lse, probs, dss
    return dq, dk, dv, o, lse

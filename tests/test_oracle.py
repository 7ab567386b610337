"""Pins for the fp64 oracle (CPU only).

Each test ties the oracle to something other than itself: hand-written golden
masks and slopes, closed forms, textbook library routines (scipy softmax /
logsumexp, torch's fp64 scaled_dot_product_attention on the CPU), and invariants
the pages state (exactness: the same result whatever the key order or split).
They are chosen so that a dropped term, a wrong sign, a wrong index or a
swapped operand in the oracle fails at least one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from conftest import read_masks, read_slopes

RNG = np.random.default_rng(1234)


def rnd(*shape):
    return RNG.standard_normal(shape)


def onehot_v(Sk):
    """V rows are unit vectors: O row i then lists the attention weights of row i."""
    return np.eye(Sk).reshape(1, Sk, 1, Sk)


def pad_last(x, d):
    """Zero-pad the head dim to d (leaves every dot product unchanged)."""
    out = np.zeros(x.shape[:-1] + (d,))
    out[..., : x.shape[-1]] = x
    return out


# ---------------------------------------------------------------- golden masks
@pytest.mark.parametrize("case", read_masks(), ids=lambda c: "sq{sq}sk{sk}c{causal}w{wl},{wr}".format(**c[0]))
def test_mask_golden(case):
    """Zero queries make every score 0: O row i = uniform weights over its allowed keys."""
    p, rows = case
    sq, sk = p["sq"], p["sk"]
    q = np.zeros((1, sq, 1, sk))
    k = rnd(1, sk, 1, sk)
    out, lse = oracle.attention_dense(q, k, onehot_v(sk), scale=0.7, causal=bool(p["causal"]),
                                      window=(p["wl"], p["wr"]))
    for i, row in enumerate(rows):
        n = sum(row)
        if n == 0:
            assert np.all(out[0, i, 0] == 0.0)
            assert lse[0, 0, i] == -math.inf
        else:
            np.testing.assert_allclose(out[0, i, 0], np.array(row) / n, rtol=0, atol=1e-15)
            assert abs(lse[0, 0, i] - math.log(n)) < 1e-14


# ---------------------------------------------------------------- ALiBi
@pytest.mark.parametrize("sq,sk,causal,window", [(5, 5, True, (-1, -1)), (3, 6, False, (-1, -1)),
                                                  (4, 7, False, (2, 1)), (6, 3, True, (-1, -1))])
def test_alibi_dyadic_closed_form(sq, sk, causal, window):
    """slope = ln 2 and zero scores: weight of key j is 2^-|i + Sk - Sq - j| (exact dyadics).

    A flipped sign gives 2^+|.|, a dropped offset gives 2^-|i - j|; both fail.
    """
    q = np.zeros((1, sq, 1, sk))
    k = rnd(1, sk, 1, sk)
    slopes = np.array([math.log(2.0)])
    out, lse = oracle.attention_dense(q, k, onehot_v(sk), scale=1.0, causal=causal,
                                      window=window, alibi_slopes=slopes)
    off = sk - sq
    for i in range(sq):
        c = i + off
        allowed = [j for j in range(sk)
                   if (not causal or j <= c) and (window[0] < 0 or j >= c - window[0])
                   and (window[1] < 0 or j <= c + window[1])]
        if not allowed:
            assert lse[0, 0, i] == -math.inf
            continue
        w = {j: Fraction(1, 2 ** abs(c - j)) for j in allowed}
        Z = sum(w.values())
        expect = np.array([float(w.get(j, 0) / Z) for j in range(sk)])
        np.testing.assert_allclose(out[0, i, 0], expect, rtol=1e-14, atol=1e-15)
        assert abs(lse[0, 0, i] - math.log(float(Z))) < 1e-13


# ---------------------------------------------------------------- softcap
def test_softcap_saturates_to_cap():
    """Scores far beyond the cap land on +-cap (pages: softcap keeps scores within [-cap, cap])."""
    cap = 3.0
    q = np.ones((1, 1, 1, 1))
    k = np.array([1e6, -1e6, 1e6, -1e6, -1e6]).reshape(1, 5, 1, 1)
    v = onehot_v(5)
    out, lse = oracle.attention_dense(pad_last(q, 5), pad_last(k, 5), v, scale=1.0, softcap=cap)
    Z = 2 * math.exp(cap) + 3 * math.exp(-cap)
    assert abs(lse[0, 0, 0] - math.log(Z)) < 1e-13
    expect = np.array([math.exp(cap), math.exp(-cap), math.exp(cap), math.exp(-cap),
                       math.exp(-cap)]) / Z
    np.testing.assert_allclose(out[0, 0, 0], expect, rtol=1e-13)


@pytest.mark.parametrize("cap", [0.5, 5.0, 50.0])
def test_softcap_divides_inside_multiplies_outside(cap):
    """Raw score cap*atanh(1/2) must come out as cap/2: pins cap*tanh(s/cap)."""
    q = np.ones((1, 1, 1, 1))
    k = np.array([cap * math.atanh(0.5), 0.0]).reshape(1, 2, 1, 1)
    out, lse = oracle.attention_dense(pad_last(q, 2), pad_last(k, 2), onehot_v(2), scale=1.0,
                                      softcap=cap)
    assert abs(lse[0, 0, 0] - math.log(math.exp(cap / 2) + 1.0)) < 1e-12
    assert abs(out[0, 0, 0, 0] - 1.0 / (1.0 + math.exp(-cap / 2))) < 1e-14


def test_softcap_large_cap_is_no_cap():
    q, k, v = rnd(2, 6, 2, 8), rnd(2, 9, 2, 8), rnd(2, 9, 2, 8)
    a = oracle.attention_dense(q, k, v, causal=True, softcap=1e9)
    b = oracle.attention_dense(q, k, v, causal=True)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- library routines
def test_plain_matches_scipy_softmax():
    B, Sq, Sk, H, d = 2, 7, 9, 3, 5
    q, k, v = rnd(B, Sq, H, d), rnd(B, Sk, H, d), rnd(B, Sk, H, d)
    out, lse = oracle.attention_dense(q, k, v)          # default scale 1/sqrt(d)
    s = np.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(d)
    p = scipy.special.softmax(s, axis=-1)
    np.testing.assert_allclose(out, np.einsum("bhij,bjhd->bihd", p, v), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=-1), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("case", read_masks(), ids=lambda c: "sq{sq}sk{sk}c{causal}w{wl},{wr}".format(**c[0]))
@pytest.mark.parametrize("alibi", [False, True])
def test_masked_matches_torch_sdpa(case, alibi):
    """torch's fp64 CPU SDPA with the golden mask (and an additive ALiBi bias)."""
    p, rows = case
    sq, sk, d, H = p["sq"], p["sk"], 6, 2
    q, k, v = rnd(1, sq, H, d), rnd(1, sk, H, d), rnd(1, sk, H, d)
    slopes = np.array([0.3, 0.05]) if alibi else None
    out, lse = oracle.attention_dense(q, k, v, causal=bool(p["causal"]),
                                      window=(p["wl"], p["wr"]), alibi_slopes=slopes)
    mask = torch.tensor(rows, dtype=torch.bool)
    ok = mask.any(dim=1)
    off = sk - sq
    dist = (torch.arange(sq)[:, None] + off - torch.arange(sk)[None, :]).abs().double()
    for h in range(H):
        bias = torch.zeros(sq, sk, dtype=torch.float64)
        if alibi:
            bias = -slopes[h] * dist
        bias = bias.masked_fill(~mask, -math.inf)
        tq = torch.from_numpy(q[0, :, h]).unsqueeze(0)
        tk = torch.from_numpy(k[0, :, h]).unsqueeze(0)
        tv = torch.from_numpy(v[0, :, h]).unsqueeze(0)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=bias)[0]
        np.testing.assert_allclose(out[0, ok.numpy(), h], ref[ok].numpy(), rtol=1e-11, atol=1e-12)
        s = (tq[0] @ tk[0].T) / math.sqrt(d) + bias
        ref_lse = torch.logsumexp(s, dim=-1)
        np.testing.assert_allclose(lse[0, h, ok.numpy()], ref_lse[ok].numpy(), rtol=1e-12, atol=1e-12)
        assert np.all(lse[0, h, ~ok.numpy()] == -math.inf)
        assert np.all(out[0, ~ok.numpy(), h] == 0.0)


# ---------------------------------------------------------------- closed forms
def test_single_allowed_key_returns_that_value_row():
    """Window (0, 0): each row sees exactly key i + Sk - Sq."""
    Sq, Sk, d = 4, 6, 3
    q, k, v = rnd(1, Sq, 1, d), rnd(1, Sk, 1, d), rnd(1, Sk, 1, d)
    out, lse = oracle.attention_dense(q, k, v, scale=0.9, window=(0, 0))
    for i in range(Sq):
        j = i + Sk - Sq
        np.testing.assert_array_equal(out[0, i, 0], v[0, j, 0])
        assert abs(lse[0, 0, i] - 0.9 * float(q[0, i, 0] @ k[0, j, 0])) < 1e-14


def test_zero_scale_gives_mean_of_allowed_values():
    Sq, Sk, d = 5, 8, 4
    q, k, v = rnd(1, Sq, 2, d), rnd(1, Sk, 2, d), rnd(1, Sk, 2, d)
    out, lse = oracle.attention_dense(q, k, v, scale=0.0, causal=True)
    for i in range(Sq):
        n = i + Sk - Sq + 1
        np.testing.assert_allclose(out[0, i], v[0, :n].mean(axis=0), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[0, :, i], math.log(n), rtol=1e-14)


def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    q, k, v = rnd(1, 6, 2, 4), rnd(1, 3, 2, 4), rnd(1, 3, 2, 4)
    out, lse = oracle.attention_dense(q, k, v, causal=True)
    assert np.all(out[0, :3] == 0.0) and np.all(lse[0, :, :3] == -math.inf)
    assert np.all(np.isfinite(lse[0, :, 3:]))


def test_decode_example_one_query_sees_all_keys():
    """Changelog example: 1 query, N+1 keys, causal -> attends all N+1 keys."""
    q, k, v = rnd(2, 1, 2, 16), rnd(2, 1025, 2, 16), rnd(2, 1025, 2, 16)
    a = oracle.attention_dense(q, k, v, causal=True)
    b = oracle.attention_dense(q, k, v, causal=False)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_value_rows_of_ones_give_ones():
    """Probabilities of every row with an allowed key sum to 1."""
    q, k = rnd(2, 7, 4, 5), rnd(2, 9, 2, 5)
    v = np.ones((2, 9, 2, 5))
    out, lse = oracle.attention_dense(q, k, v, causal=True, window=(3, -1), softcap=2.0,
                                      alibi_slopes=np.array([0.5, 0.1, 0.2, 0.0]))
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- invariants
def test_gqa_equals_repeated_kv_heads():
    B, Sq, Sk, H, Hkv, d = 2, 5, 7, 6, 2, 4
    q, k, v = rnd(B, Sq, H, d), rnd(B, Sk, Hkv, d), rnd(B, Sk, Hkv, d)
    a = oracle.attention_dense(q, k, v, causal=True)
    kr, vr = np.repeat(k, H // Hkv, axis=2), np.repeat(v, H // Hkv, axis=2)
    b = oracle.attention_dense(q, kr, vr, causal=True)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    # and a wrong grouping (h % Hkv) would differ
    kw, vw = np.tile(k, (1, 1, H // Hkv, 1)), np.tile(v, (1, 1, H // Hkv, 1))
    c = oracle.attention_dense(q, kw, vw, causal=True)
    assert not np.allclose(a[0], c[0])


def test_cu_seqlens_matches_pages_example():
    """Section 3.2: lengths [512, 1024, 768] -> cu_seqlens [0, 512, 1536, 2304]."""
    assert synth.cu_seqlens([512, 1024, 768]).tolist() == [0, 512, 1536, 2304]


def test_varlen_equals_per_sequence_dense():
    lq, lk = [5, 9, 3], [7, 9, 1]
    q, k, v, cq, ck = synth.varlen(lq, lk, 4, 2, 8, dtype=torch.float32, seed=3)
    out, lse = oracle.attention(q, k, v, cq, ck, causal=True, window=(4, -1), softcap=3.0,
                                alibi_slopes=synth.alibi_slopes(4))
    for b in range(3):
        qs, ks = slice(int(cq[b]), int(cq[b + 1])), slice(int(ck[b]), int(ck[b + 1]))
        o1, l1 = oracle.attention_dense(q[qs][None], k[ks][None], v[ks][None], causal=True,
                                        window=(4, -1), softcap=3.0,
                                        alibi_slopes=synth.alibi_slopes(4))
        np.testing.assert_array_equal(out[qs], o1[0])
        np.testing.assert_array_equal(lse[qs], l1[0].T)


def test_paged_equals_contiguous_bitwise():
    lens = [37, 5, 64, 1]
    page = 16
    kp, vp, bt, cs = synth.paged_cache(lens, page, 2, 8, dtype=torch.float32, seed=5,
                                       spare_blocks=3)
    q = torch.randn(4, 3, 4, 8, generator=torch.Generator().manual_seed(9))
    out, lse = oracle.attention_paged(q, kp, vp, bt, cs, causal=True, softcap=4.0,
                                      alibi_slopes=synth.alibi_slopes(4))
    for b, L in enumerate(lens):
        rows = []
        for j in range(L):
            rows.append(int(bt[b, j // page]) * page + j % page)
        kc = kp.reshape(-1, 2, 8)[rows][None]
        vc = vp.reshape(-1, 2, 8)[rows][None]
        o1, l1 = oracle.attention_dense(q[b:b + 1], kc, vc, causal=True, softcap=4.0,
                                        alibi_slopes=synth.alibi_slopes(4))
        np.testing.assert_array_equal(out[b], o1[0])
        np.testing.assert_array_equal(lse[b], l1[0])
        assert np.all(np.isfinite(out[b]))   # NaN page tails never reached the result


def test_split_then_combine_equals_unsplit():
    """Changelog v2.2 split-KV + section 3.4 combine: exact for any split of the keys."""
    B, Sq, Sk, H, d = 2, 3, 23, 2, 5
    q, k, v = rnd(B, Sq, H, d), rnd(B, Sk, H, d), rnd(B, Sk, H, d)
    full_o, full_l = oracle.attention_dense(q, k, v)
    bounds = [0, 4, 4, 15, 23]     # includes an empty split
    ops, lps = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        if a == b:
            ops.append(np.zeros((B, Sq, H, d)))
            lps.append(np.full((B, Sq, H), -math.inf))
            continue
        o, l = oracle.attention_dense(q, k[:, a:b], v[:, a:b], scale=1 / math.sqrt(d))
        ops.append(o)
        lps.append(l.transpose(0, 2, 1))
    op = np.stack(ops, axis=-1)
    lp = np.stack(lps, axis=-1)
    out, lse = oracle.combine(op, lp)
    np.testing.assert_allclose(out, full_o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, full_l.transpose(0, 2, 1), rtol=1e-13, atol=1e-13)


def test_combine_special_cases():
    op = rnd(3, 4, 2)
    out, lse = oracle.combine(op, np.full((3, 2), -math.inf))
    assert np.all(out == 0) and np.all(lse == -math.inf)
    out, lse = oracle.combine(op[..., :1], np.array([[0.3], [1.0], [-2.0]]))
    np.testing.assert_array_equal(out, op[..., 0])
    np.testing.assert_array_equal(lse, [0.3, 1.0, -2.0])
    out, lse = oracle.combine(op, np.array([[0.5, 0.5]] * 3))
    np.testing.assert_allclose(out, op.mean(axis=-1), rtol=1e-14)
    np.testing.assert_allclose(lse, 0.5 + math.log(2.0), rtol=1e-15)


def test_key_permutation_invariance():
    q, k, v = rnd(1, 4, 2, 6), rnd(1, 11, 2, 6), rnd(1, 11, 2, 6)
    perm = RNG.permutation(11)
    a = oracle.attention_dense(q, k, v, softcap=5.0)
    b = oracle.attention_dense(q, k[:, perm], v[:, perm], softcap=5.0)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13)


def test_linear_in_values():
    q, k, v1, v2 = rnd(1, 5, 2, 4), rnd(1, 8, 2, 4), rnd(1, 8, 2, 4), rnd(1, 8, 2, 4)
    kw = dict(causal=True, alibi_slopes=np.array([0.25, 0.5]))
    o1 = oracle.attention_dense(q, k, v1, **kw)[0]
    o2 = oracle.attention_dense(q, k, v2, **kw)[0]
    o3 = oracle.attention_dense(q, k, 2.0 * v1 - 3.0 * v2, **kw)[0]
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-12, atol=1e-12)


def test_constant_score_shift_moves_lse_only():
    """q' = [q, 1], k' = [k, c] adds scale*c to every score: O unchanged, LSE + scale*c."""
    q, k, v = rnd(1, 5, 1, 4), rnd(1, 7, 1, 4), rnd(1, 7, 1, 4)
    c, scale = 2.5, 0.4
    q2 = np.concatenate([q, np.ones((1, 5, 1, 1))], axis=-1)
    k2 = np.concatenate([k, np.full((1, 7, 1, 1), c)], axis=-1)
    v2 = np.concatenate([v, np.zeros((1, 7, 1, 1))], axis=-1)
    a = oracle.attention_dense(q, k, v, scale=scale, causal=True)
    b = oracle.attention_dense(q2, k2, v2, scale=scale, causal=True)
    np.testing.assert_allclose(b[0][..., :4], a[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b[1], a[1] + scale * c, rtol=1e-13)


def test_online_blockwise_softmax_equals_oracle():
    """The method (tiles of keys, running max and sum, rescaled accumulator) reaches
    the oracle's two-pass result: the pages' exactness claim, checked in fp64."""
    Sq, Sk, d, BN = 6, 29, 5, 8
    q, k, v = rnd(Sq, d), rnd(Sk, d), rnd(Sk, d)
    scale = 1 / math.sqrt(d)
    o_ref, l_ref = oracle.attention_dense(q[None, :, None], k[None, :, None], v[None, :, None],
                                          causal=True)
    off = Sk - Sq
    for i in range(Sq):
        m, l, acc = -math.inf, 0.0, np.zeros(d)
        for j0 in range(0, Sk, BN):
            s = np.array([scale * q[i] @ k[j] if j <= i + off else -math.inf
                          for j in range(j0, min(Sk, j0 + BN))])
            m_new = max(m, s.max())
            if m_new == -math.inf:
                continue
            alpha = math.exp(m - m_new) if m != -math.inf else 0.0
            p = np.exp(s - m_new)
            l = l * alpha + p.sum()
            acc = acc * alpha + p @ v[j0:j0 + len(s)]
            m = m_new
        np.testing.assert_allclose(acc / l, o_ref[0, i, 0], rtol=1e-12, atol=1e-13)
        assert abs(m + math.log(l) - l_ref[0, 0, i]) < 1e-12


# ---------------------------------------------------------------- input generator
def test_alibi_slopes_golden():
    for n, exps in read_slopes().items():
        np.testing.assert_allclose(synth.alibi_slopes(n).double().numpy(),
                                   [2.0 ** e for e in exps], rtol=1e-7)


def test_generators_are_seeded():
    a = synth.dense(1, 4, 4, 2, 2, 8, seed=7)
    b = synth.dense(1, 4, 4, 2, 2, 8, seed=7)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    kp, vp, bt, cs = synth.paged_cache([300, 20], 256, 1, 4, seed=1, spare_blocks=2)
    assert sorted(bt[bt >= 0].tolist()) != []
    used = set(bt[bt >= 0].tolist())
    assert len(used) == 3 and all(0 <= x < 5 for x in used)
    assert torch.isnan(kp[int(bt[1, 0]), 20:]).all()


# ------------------------------------------------------------------ KV-cache append
def test_append_hand_positions_paged():
    """Page 2, sequence 0 holds 1 key, blocks [3, 0]: its two new rows land at key
    positions 1 and 2 = (block 3, row 1) and (block 0, row 0); sequence 1 holds 2
    keys, blocks [1, 2]: its rows land at positions 2, 3 = (block 2, rows 0 and 1).
    Nothing else changes."""
    kp = torch.zeros(4, 2, 1, 2)
    vp = torch.zeros(4, 2, 1, 2)
    bt = torch.tensor([[3, 0, -1], [1, 2, -1]], dtype=torch.int32)
    cs = torch.tensor([1, 2], dtype=torch.int32)
    kn = torch.arange(1, 9, dtype=torch.float32).reshape(2, 2, 1, 2)
    vn = -kn
    ko, vo = oracle.append(kp, vp, kn, vn, cs, bt)
    want = torch.zeros(4, 2, 1, 2)
    want[3, 1, 0] = torch.tensor([1., 2.])
    want[0, 0, 0] = torch.tensor([3., 4.])
    want[2, 0, 0] = torch.tensor([5., 6.])
    want[2, 1, 0] = torch.tensor([7., 8.])
    assert torch.equal(ko, want)
    assert torch.equal(vo, -want)
    assert torch.equal(kp, torch.zeros(4, 2, 1, 2))   # inputs untouched


def test_append_hand_positions_contiguous():
    kc = torch.zeros(2, 4, 1, 1)
    kn = torch.tensor([[[[5.]], [[6.]]], [[[7.]], [[8.]]]])
    ko, _ = oracle.append(kc, kc, kn, kn, torch.tensor([0, 2]))
    assert ko[:, :, 0, 0].tolist() == [[5., 6., 0., 0.], [0., 0., 7., 8.]]


def test_append_outside_the_cache_raises():
    kc = torch.zeros(1, 4, 1, 1)
    kn = torch.ones(1, 2, 1, 1)
    with pytest.raises(IndexError):
        oracle.append(kc, kc, kn, kn, torch.tensor([3]))
    bt = torch.tensor([[0, 1]], dtype=torch.int32)
    with pytest.raises(IndexError):
        oracle.append(torch.zeros(2, 2, 1, 1), torch.zeros(2, 2, 1, 1), kn, kn,
                      torch.tensor([3]), bt)


def test_append_then_attend_equals_attention_on_the_concatenation():
    """Decoding step of section 3.3: attending the appended cache equals dense
    attention over (cached keys ++ new keys), the new queries at the last positions."""
    lens = [5, 16, 0]
    page, Hkv, d, H, s_new = 8, 2, 8, 4, 3
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, dtype=torch.float32, seed=21,
                                       spare_blocks=2, tail_fill=0.0)
    # room for the new rows: fresh zero blocks for the pages they open
    need = [(L + s_new + page - 1) // page for L in lens]
    bt = torch.cat([bt, torch.full((len(lens), max(need) - bt.shape[1]), -1,
                                   dtype=torch.int32)], dim=1)
    nxt = kp.shape[0]
    for b, L in enumerate(lens):
        for pg in range((L + page - 1) // page, need[b]):
            bt[b, pg] = nxt
            nxt += 1
    kp = torch.cat([kp, torch.zeros(nxt - kp.shape[0], page, Hkv, d)])
    vp = torch.cat([vp, torch.zeros(nxt - vp.shape[0], page, Hkv, d)])
    g = torch.Generator().manual_seed(22)
    kn = torch.randn(3, s_new, Hkv, d, generator=g)
    vn = torch.randn(3, s_new, Hkv, d, generator=g)
    q = torch.randn(3, s_new, H, d, generator=g)
    ka, va = oracle.append(kp, vp, kn, vn, cs, bt)
    out, lse = oracle.attention_paged(q, ka, va, bt, cs + s_new, causal=True)
    for b, L in enumerate(lens):
        rows = [int(bt[b, j // page]) * page + j % page for j in range(L)]
        kc = torch.cat([kp.reshape(-1, Hkv, d)[rows], kn[b]])[None]
        vc = torch.cat([vp.reshape(-1, Hkv, d)[rows], vn[b]])[None]
        o1, l1 = oracle.attention_dense(q[b:b + 1], kc, vc, causal=True)
        np.testing.assert_allclose(out[b], o1[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], l1[0], rtol=0, atol=1e-12)


def brute_attention(q, k, v, scale, causal, window, softcap, slopes):
    """Per-element pure-Python fp64 attention (math.exp / math.tanh), written out
    from the definition: bottom-right aligned mask, softcap inside the exponent,
    ALiBi as -slope * |i + Sk - Sq - j|, empty rows give O = 0 and LSE = -inf."""
    B, Sq, H, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = H // Hkv
    wl, wr = window
    out = np.zeros((B, Sq, H, d))
    lse = np.full((B, H, Sq), -math.inf)
    for b in range(B):
        for h in range(H):
            hk = h // G
            for i in range(Sq):
                c = i + Sk - Sq
                scores = []
                for j in range(Sk):
                    if causal and j > c:
                        continue
                    if wl >= 0 and j < c - wl:
                        continue
                    if not causal and wr >= 0 and j > c + wr:
                        continue
                    s = scale * sum(float(q[b, i, h, t]) * float(k[b, j, hk, t]) for t in range(d))
                    if softcap > 0:
                        s = softcap * math.tanh(s / softcap)
                    if slopes is not None:
                        s -= float(slopes[h]) * abs(c - j)
                    scores.append((j, s))
                if not scores:
                    continue
                m = max(s for _, s in scores)
                z = sum(math.exp(s - m) for _, s in scores)
                lse[b, h, i] = m + math.log(z)
                for j, s in scores:
                    w = math.exp(s - lse[b, h, i])
                    for t in range(d):
                        out[b, i, h, t] += w * float(v[b, j, hk, t])
    return out, lse


@pytest.mark.parametrize("sq,sk", [(4, 4), (3, 7), (6, 2)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", [(-1, -1), (1, -1), (-1, 1), (2, 0)])
@pytest.mark.parametrize("softcap", [0.0, 1.5])
@pytest.mark.parametrize("alibi", [False, True])
def test_brute_force_every_flag_combination(sq, sk, causal, window, softcap, alibi):
    """Tiny shapes (B=2, H=2 over Hkv=1, d=3), every flag combination, against the
    per-element pure-Python definition above: agreement to 1e-12."""
    rng = np.random.default_rng(sq * 100 + sk * 10 + causal)
    q = rng.standard_normal((2, sq, 2, 3))
    k = rng.standard_normal((2, sk, 1, 3))
    v = rng.standard_normal((2, sk, 1, 3))
    slopes = np.array([0.5, 0.125]) if alibi else None
    kw = dict(scale=0.8, causal=causal, window=window, softcap=softcap)
    if alibi:
        kw["alibi_slopes"] = slopes
    o, l = oracle.attention_dense(q, k, v, **kw)
    ro, rl = brute_attention(q, k, v, 0.8, causal, window, softcap, slopes)
    np.testing.assert_allclose(o, ro, atol=1e-12, rtol=0)
    assert np.array_equal(np.isneginf(l), np.isneginf(rl))
    fin = np.isfinite(rl)
    np.testing.assert_allclose(l[fin], rl[fin], atol=1e-12, rtol=0)

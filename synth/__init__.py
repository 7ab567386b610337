"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws inputs only: it holds none of the attention arithmetic, so both
the oracle side and the CUDA side can take their inputs from it without sharing
any of the method.  Every tensor is drawn on the host from a ``torch.Generator``
seeded explicitly, as N(0, 1) fp32 values cast to the 16-bit input dtype (the
pages' examples all use ``torch.randn`` inputs in fp16/bf16).

Recipes
-------
dense(B, Sq, Sk, H, Hkv, d, dtype, seed)          q/k/v in [batch, seq, heads, dim]
varlen_lengths(n, lo, hi, seed)                   sequence lengths ~ U{lo..hi}
varlen(lengths_q, lengths_k, H, Hkv, d, ...)      packed [total, heads, dim] + cu_seqlens
paged_cache(seqlens, page, Hkv, d, ...)           pool + random-permutation block_table
alibi_slopes(n)                                   the pages' get_alibi_slopes rule
"""
from __future__ import annotations

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, dtype, gen: torch.Generator) -> torch.Tensor:
    """N(0,1) fp32 draw cast to ``dtype`` (round to nearest even), on the
    generator's device (large inputs are drawn on the GPU in chunks)."""
    dev = gen.device
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=dtype, device=dev)
    step = 1 << 26
    for i in range(0, n, step):
        m = min(step, n - i)
        out[i:i + m] = torch.randn(m, generator=gen, dtype=torch.float32, device=dev).to(dtype)
    return out.view(*shape)


def dense(B, Sq, Sk, H, Hkv, d, dtype=torch.float16, seed=0):
    """q [B,Sq,H,d], k/v [B,Sk,Hkv,d] (section 3.1 layout)."""
    g = _gen(seed)
    q = randn((B, Sq, H, d), dtype, g)
    k = randn((B, Sk, Hkv, d), dtype, g)
    v = randn((B, Sk, Hkv, d), dtype, g)
    return q, k, v


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> list[int]:
    """``n`` lengths drawn uniformly from the integers lo..hi inclusive."""
    g = _gen(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def cu_seqlens(lengths) -> torch.Tensor:
    """int32 [n+1] running offsets (section 3.2: [0, 512, 1536, 2304] for [512, 1024, 768])."""
    out = [0]
    for L in lengths:
        out.append(out[-1] + int(L))
    return torch.tensor(out, dtype=torch.int32)


def varlen(lengths_q, lengths_k, H, Hkv, d, dtype=torch.bfloat16, seed=0):
    """Packed q [total_q,H,d], k/v [total_k,Hkv,d] plus int32 cu_seqlens (section 3.2)."""
    g = _gen(seed)
    tq, tk = int(sum(lengths_q)), int(sum(lengths_k))
    q = randn((tq, H, d), dtype, g)
    k = randn((tk, Hkv, d), dtype, g)
    v = randn((tk, Hkv, d), dtype, g)
    return q, k, v, cu_seqlens(lengths_q), cu_seqlens(lengths_k)


def paged_cache(seqlens, page: int, Hkv: int, d: int, dtype=torch.bfloat16, seed=0,
                tail_fill: float = float("nan"), spare_blocks: int = 0, device="cpu"):
    """A paged KV pool for sequences of the given lengths (changelog v2.5 paged KV).

    Returns (kpool, vpool [num_blocks, page, Hkv, d], block_table int32 [B, max_blocks],
    cache_seqlens int32 [B]).  Physical blocks are a random permutation of the
    pool; unused block_table entries are -1.  Slots past each sequence's end and
    the ``spare_blocks`` extra blocks hold ``tail_fill`` (NaN by default) so that
    a kernel which reads them shows it.
    """
    g = _gen(seed, device)
    gh = _gen(seed + 7919)               # block permutation drawn on the host
    B = len(seqlens)
    nb = [(int(L) + page - 1) // page for L in seqlens]
    total = sum(nb) + int(spare_blocks)
    max_blocks = max(1, max(nb) if nb else 1)
    kpool = randn((total, page, Hkv, d), dtype, g)
    vpool = randn((total, page, Hkv, d), dtype, g)
    perm = torch.randperm(total, generator=gh).to(torch.int32)
    bt = torch.full((B, max_blocks), -1, dtype=torch.int32)
    used = torch.zeros(total, dtype=torch.bool)
    pos = 0
    for b, L in enumerate(seqlens):
        for p in range(nb[b]):
            blk = int(perm[pos])
            pos += 1
            bt[b, p] = blk
            used[blk] = True
            valid = min(page, int(L) - p * page)
            if valid < page:
                kpool[blk, valid:] = tail_fill
                vpool[blk, valid:] = tail_fill
    unused = (~used).nonzero().flatten().to(kpool.device)
    kpool[unused] = tail_fill
    vpool[unused] = tail_fill
    return kpool, vpool, bt, torch.tensor([int(L) for L in seqlens], dtype=torch.int32)


def alibi_slopes(n: int) -> torch.Tensor:
    """ALiBi slopes by the pages' ``get_alibi_slopes`` rule (section 5.1).

    For a power of two n: a geometric sequence with first term and ratio
    2^(-8/n).  Otherwise the slopes of the largest power of two m < n, followed
    by every other slope of the 2m sequence, taken until n slopes exist.
    (The page writes ``torch.math``; it is read as Python's ``math``.)
    """
    def geometric(m: int) -> list[float]:
        # slope i (0-based) of an m-head model is 2^(-8 (i+1) / m)
        return [2.0 ** (-8.0 * (i + 1) / m) for i in range(m)]

    if n <= 0:
        raise ValueError("alibi_slopes: n must be positive")
    m = 1 << (n.bit_length() - 1)          # largest power of two <= n
    slopes = geometric(m)
    if m != n:
        slopes += geometric(2 * m)[0::2][: n - m]
    return torch.tensor(slopes, dtype=torch.float32)

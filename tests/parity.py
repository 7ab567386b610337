"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (max abs difference against the unrounded fp64 oracle):
  O:   2e-3 (fp16 inputs) / 1e-2 (bf16 inputs), plus half an ulp of the output
       format at the reference value (|ref| * 2^-11 for fp16, 2^-8 for bf16): the
       output is rounded to the 16-bit input type, and for rows that attend very
       few keys |O| can exceed 4, where bf16 rounding alone is above 1e-2.
  LSE: 1e-3 absolute on finite values; rows with no allowed key must give
       LSE = -inf and O = 0 exactly.
"""
import math

import numpy as np
import torch

ATOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}
RTOL = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}
LSE_ATOL = 1e-3


def to_np(t):
    return t.detach().float().cpu().double().numpy()


def check_out(out_gpu, out_ref, dtype, what="O"):
    """Element-by-element check of O; returns the max abs difference."""
    got = to_np(out_gpu)
    ref = np.asarray(out_ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values in the GPU output"
    diff = np.abs(got - ref)
    bound = ATOL[dtype] + RTOL[dtype] * np.abs(ref)
    bad = diff > bound
    if bad.any():
        idx = np.unravel_index(np.argmax(diff - bound), diff.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; worst at "
                             f"{idx}: got {got[idx]!r} ref {ref[idx]!r} (bound {bound[idx]:.3g})")
    return float(diff.max()) if diff.size else 0.0


def check_lse(lse_gpu, lse_ref, what="LSE"):
    got = to_np(lse_gpu)
    ref = np.asarray(lse_ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    ninf = ref == -math.inf
    assert np.array_equal(got == -math.inf, ninf), f"{what}: -inf pattern differs"
    fin = ~ninf
    assert np.all(np.isfinite(got[fin])), f"{what}: non-finite where the oracle is finite"
    diff = np.abs(got[fin] - ref[fin])
    if diff.size and diff.max() > LSE_ATOL:
        raise AssertionError(f"{what}: max |dLSE| = {diff.max():.3g} > {LSE_ATOL}")
    return float(diff.max()) if diff.size else 0.0

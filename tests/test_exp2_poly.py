"""The FMA-pipe exp2 used by the prefill kernel (exp2_fma2 in sm100.cuh), replayed in
float32 numpy: coefficients match the Remez fit of gen_exp2_poly.py, and the
round/split/polynomial/exponent-add method stays within its error bound against
numpy's exp2 on [-126, 8] (the argument range of x - running max, with the lazy
rescale threshold of 8)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "io_aware_online_b200", "csrc")


def kernel_coeffs():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    m = re.search(r"kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", src)
    assert m, "coefficients not found in sm100.cuh"
    return [np.float32(float(g)) for g in m.groups()]


def replay(x):
    """float32 replay of exp2_fma2 (same operation order)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    kr = np.float32(12582912.0)
    t = (x + kr).astype(np.float32)
    j = (t - kr).astype(np.float32)
    f = (x - j).astype(np.float32)
    c0, c1, c2, c3 = kernel_coeffs()
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_match_the_remez_fit():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, err = gen.remez_exp2(3)
    np.testing.assert_allclose(kernel_coeffs(), c, rtol=2e-7)
    assert err < 8e-5


def test_relative_error_bound():
    x = np.linspace(-125.9, 8.0, 2_000_001, dtype=np.float32)
    y = replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.0e-4      # 7.5e-5 polynomial + float32 rounding


def test_exact_integers_and_special_values():
    assert replay(np.float32(0.0)) == np.float32(np.float32(0.99992806))  # c0
    for k in range(-20, 9):
        assert abs(float(replay(np.float32(k))) / 2.0 ** k - 1) < 1e-4
    tiny = replay(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -126)

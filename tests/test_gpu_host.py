"""GPU tests of fa_fwd_host: the dense forward on operands in host memory, with the
batch moved through a device workspace in chunks on the library's own streams.

Every case compares the host-buffer call element by element with the fp64 oracle and
bit for bit with one fa_fwd call on device copies of the same inputs (each chunk is
an fa_fwd call over whole sequences, so nothing may differ).  Batches of 5 and 7
give ragged chunking (2, 2, 1 and 2, 2, 2, 1 sequences per chunk).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from io_aware_online_b200 import build
    build.build()
    import io_aware_online_b200 as fa
    fa.load()
    fa.fa_device_status(clear=True)
    yield
    assert fa.fa_device_status(clear=True) == 0, "a kernel raised a device status flag"


CASES = [
    # B, Sq, Sk, H, Hkv, d, dtype, kwargs
    (5, 300, 300, 4, 2, 64, torch.float16, dict(causal=True)),
    (7, 200, 333, 2, 2, 128, torch.bfloat16, dict(causal=True, window_size=(150, 0))),
    (3, 129, 257, 4, 1, 64, torch.bfloat16, dict(softcap=5.0)),
    (4, 256, 256, 2, 2, 128, torch.float16, dict(alibi=True)),
    (1, 130, 130, 2, 2, 64, torch.float16, dict()),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}-d{c[5]}-{str(c[6])[6:]}-{i}"
                                             for i, c in enumerate(CASES)])
def test_host_buffers_match_oracle_and_device_call(case):
    import io_aware_online_b200 as fa
    B, sq, sk, H, Hkv, d, dt, kw = case
    kw = dict(kw)
    q, k, v = synth.dense(B, sq, sk, H, Hkv, d, dt, seed=2100 + B)
    alibi = None
    if kw.pop("alibi", False):
        alibi = torch.linspace(0.05, 0.6, H, dtype=torch.float32)
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out, lse = fa.fa_fwd_host(hq, hk, hv, alibi_slopes=alibi, **kw)
    torch.cuda.synchronize()
    # the same inputs through one device-side call
    dout, dlse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV),
                           alibi_slopes=None if alibi is None else alibi.to(DEV), **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, dout.cpu()), "host-buffer call differs from fa_fwd"
    assert torch.equal(lse, dlse.cpu())
    ro, rl = oracle.attention_dense(q, k, v, scale=None, causal=kw.get("causal", False),
                                    window=kw.get("window_size", (-1, -1)),
                                    softcap=kw.get("softcap", 0.0),
                                    alibi_slopes=None if alibi is None else alibi.numpy())
    check_out(out, ro, dt)
    check_lse(lse, rl)


def test_host_call_orders_on_the_callers_stream():
    """Work the caller enqueued before the call finishes first, and the caller's stream
    does not pass the call before the last copy into `out` has landed."""
    import io_aware_online_b200 as fa
    B, S, H, d = 4, 512, 4, 64
    q, k, v = synth.dense(B, S, S, H, H, d, torch.float16, seed=2200)
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out = torch.full(q.shape, float("nan"), dtype=q.dtype).pin_memory()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        torch.cuda._sleep(20_000_000)  # keep the caller's stream busy for a while
        fa.fa_fwd_host(hq, hk, hv, out=out, return_lse=False, causal=True, stream=s)
        done = torch.cuda.Event()
        done.record(s)
    done.synchronize()
    ref, _ = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.cpu())


def test_host_call_without_lse_and_with_pageable_memory():
    import io_aware_online_b200 as fa
    B, S, H, d = 3, 200, 2, 128
    q, k, v = synth.dense(B, S, S, H, H, d, torch.bfloat16, seed=2300)
    out = torch.empty_like(q)  # pageable
    o, l = fa.fa_fwd_host(q, k, v, out=out, return_lse=False, causal=True)
    torch.cuda.synchronize()
    assert l is None and o is out
    ro, _ = oracle.attention_dense(q, k, v, causal=True)
    check_out(out, ro, torch.bfloat16)

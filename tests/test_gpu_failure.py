"""Failure detection on the GPU without a fault: a wait on a barrier phase that
nothing completes gives up after its limit, reports FA_DEV_WAIT_TIMEOUT through the
device status word, and leaves the context usable for the next call."""
import time

import pytest
import torch

import oracle
import synth
from parity import ATOL, check_lse, check_out

pytestmark = pytest.mark.gpu
FA_DEV_WAIT_TIMEOUT = 1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from io_aware_online_b200 import build
    build.build()
    import io_aware_online_b200 as fa
    fa.load()
    fa.fa_device_status(clear=True)
    yield


def test_bounded_wait_gives_up_reports_and_context_survives():
    import io_aware_online_b200 as fa
    assert fa.fa_device_status(clear=True) == 0
    t0 = time.perf_counter()
    fa.fa_selftest_wait_timeout(50)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert fa.fa_device_status(clear=True) & FA_DEV_WAIT_TIMEOUT
    assert waited >= 0.045                       # it waited its limit, then stopped
    # the next call works and is exact
    q, k, v = synth.dense(1, 256, 256, 2, 2, 64, torch.float16, seed=1600)
    out, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_dense(q, k, v, causal=True)
    assert check_out(out.cpu(), ro, torch.float16) <= ATOL[torch.float16]
    check_lse(lse.cpu(), rl)
    assert fa.fa_device_status(clear=True) == 0

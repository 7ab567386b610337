"""fa_fwd_kvcache_static: the decode for callers that cannot allocate device memory
at the call (a framework that owns all device memory through its own pool, or a
serving loop that must not risk the synchronisation a cudaMalloc can cause).

It runs the same split-KV decode with its scratch in the library's fixed device
array.  Checked through the C ABI against fa_fwd_kvcache (caller workspace) on the
same inputs, within the decode tolerances, on two calls in a row: the array keeps
the previous call's contents, so the second call also shows that what must start
at zero is cleared.  Each call is also checked against the fp64 oracle directly.
The file sorts last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import pytest
import torch

import oracle
import synth
from parity import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_static_scratch_decode_matches_workspace_decode():
    import io_aware_online_b200 as fa
    from io_aware_online_b200 import build
    build.build()
    lib = fa.load()
    assert lib.fa_kvcache_static_scratch_bytes() == 24 << 20
    lens = [1, 300, 2048, 4097, 777, 64]
    H, Hkv, d, page = 32, 8, 128, 256
    kp, vp, bt, cs = synth.paged_cache(lens, page, Hkv, d, torch.bfloat16, seed=91, spare_blocks=2)
    q = synth.randn((len(lens), 1, H, d), torch.bfloat16, torch.Generator().manual_seed(92))
    ro, rl = oracle.attention_paged(q, kp, vp, bt, cs, causal=True)
    kp, vp, bt, cs, q = kp.to(DEV), vp.to(DEV), bt.to(DEV), cs.to(DEV), q.to(DEV)
    for splits in (4, 16):
        ref_o, ref_l = fa.fa_fwd_kvcache(q, kp, vp, cache_seqlens=cs, block_table=bt,
                                         causal=True, num_splits=splits)
        for call in range(2):
            out = torch.full_like(q, float("nan"))
            lse = torch.full((len(lens), H, 1), float("nan"), dtype=torch.float32, device=DEV)
            rc = lib.fa_fwd_kvcache_static(
                ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kp.data_ptr()),
                ctypes.c_void_p(vp.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                ctypes.c_void_p(lse.data_ptr()), 1, len(lens), 1, H, Hkv, d,
                ctypes.c_void_p(bt.data_ptr()), bt.shape[1], page, kp.shape[0], 0,
                ctypes.c_void_p(cs.data_ptr()), float("nan"), 1, -1, -1, 0.0, None, splits,
                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert rc == 0, lib.fa_last_error()
            torch.cuda.synchronize()
            check_out(out, to_np(ref_o), torch.bfloat16, what=f"O (splits {splits}, call {call})")
            check_lse(lse, to_np(ref_l), what=f"LSE (splits {splits}, call {call})")
            check_out(out, ro, torch.bfloat16, what=f"O vs oracle (splits {splits}, call {call})")
            check_lse(lse, rl, what=f"LSE vs oracle (splits {splits}, call {call})")
    assert fa.fa_device_status(clear=True) == 0


def test_static_scratch_rejects_oversized_calls():
    import io_aware_online_b200 as fa
    lib = fa.load()
    # 64 sequences x 32 heads x 129 floats x 128 splits (~135 MB) is far beyond 24 MiB
    q = torch.zeros(64, 1, 32, 128, dtype=torch.bfloat16, device=DEV)
    kp = torch.zeros(300, 256, 8, 128, dtype=torch.bfloat16, device=DEV)
    bt = torch.zeros(64, 128, dtype=torch.int32, device=DEV)
    cs = torch.full((64,), 256, dtype=torch.int32, device=DEV)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_kvcache_static(q, kp, kp, cache_seqlens=cs, block_table=bt, num_splits=128)
    assert e.value.code == 3 and "fixed array" in str(e.value)

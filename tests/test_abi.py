"""C-ABI checks that need no GPU: the library builds, loads and exports every
symbol include/fa.h declares, and argument validation returns the documented
error codes before touching the device."""
import ctypes
import os
import re

import pytest
import torch

import io_aware_online_b200 as fa
from io_aware_online_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load()


def header_symbols():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = set(header_symbols())
    assert {"fa_fwd", "fa_fwd_kvcache", "fa_combine", "fa_kvcache_workspace_size",
            "fa_kvcache_num_splits", "fa_last_error", "fa_device_status"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), f"{name} not exported"


def test_version_and_error_string(lib):
    assert lib.fa_version() >= 100
    assert isinstance(lib.fa_last_error(), bytes)


# fake, 16-byte aligned "device" pointers: validation rejects before any device use
P = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10008)


def fwd(lib, **kw):
    a = dict(q=P, k=P, v=P, out=P, lse=None, dtype=0, B=1, Sq=128, Sk=128, H=2, Hkv=2, d=64,
             qs=None, ks=None, vs=None, os_=None, cuq=None, cuk=None, mq=0, mk=0,
             scale=float("nan"), causal=0, wl=-1, wr=-1, softcap=0.0, alibi=None, stream=None)
    a.update(kw)
    return lib.fa_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dtype"], a["B"], a["Sq"],
                      a["Sk"], a["H"], a["Hkv"], a["d"], a["qs"], a["ks"], a["vs"], a["os_"],
                      a["cuq"], a["cuk"], a["mq"], a["mk"], a["scale"], a["causal"], a["wl"],
                      a["wr"], a["softcap"], a["alibi"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), FA_ERR_UNSUPPORTED),
    (dict(dtype=2), FA_ERR_UNSUPPORTED),
    (dict(H=3, Hkv=2), FA_ERR_INVALID_ARG),
    (dict(Hkv=0), FA_ERR_INVALID_ARG),
    (dict(q=None), FA_ERR_INVALID_ARG),
    (dict(k=MIS), FA_ERR_INVALID_ARG),
    (dict(wl=-2), FA_ERR_INVALID_ARG),
    (dict(wr=-5), FA_ERR_INVALID_ARG),
    (dict(softcap=-1.0), FA_ERR_INVALID_ARG),
    (dict(softcap=float("inf")), FA_ERR_INVALID_ARG),
    (dict(scale=-0.5), FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), FA_ERR_INVALID_ARG),
    (dict(Sq=-1), FA_ERR_INVALID_ARG),
    (dict(cuq=P), FA_ERR_INVALID_ARG),                       # varlen needs both offsets
    (dict(cuq=P, cuk=P, mq=300, mk=10), FA_ERR_INVALID_ARG),  # max_seqlen beyond total rows
])
def test_fwd_validation(lib, kw, code):
    assert fwd(lib, **kw) == code
    assert lib.fa_last_error()


def test_fwd_bad_strides(lib):
    bad = (ctypes.c_int64 * 3)(128 * 2 * 64, 2 * 64, 60)     # head stride not a multiple of 8
    assert fwd(lib, qs=bad) == FA_ERR_INVALID_ARG


def test_fwd_empty_is_a_noop(lib):
    assert fwd(lib, B=0) == FA_OK
    assert fwd(lib, Sq=0) == FA_OK


def kvc(lib, **kw):
    a = dict(q=P, kc=P, vc=P, out=P, lse=None, dtype=1, B=2, Sq=1, H=32, Hkv=8, d=128, bt=P,
             maxb=4, page=256, nblk=8, skmax=0, cs=P, scale=float("nan"), causal=1, wl=-1,
             wr=-1, softcap=0.0, alibi=None, splits=1, ws=None, wsb=0, stream=None)
    a.update(kw)
    return lib.fa_fwd_kvcache(a["q"], a["kc"], a["vc"], a["out"], a["lse"], a["dtype"], a["B"],
                              a["Sq"], a["H"], a["Hkv"], a["d"], a["bt"], a["maxb"], a["page"],
                              a["nblk"], a["skmax"], a["cs"], a["scale"], a["causal"], a["wl"],
                              a["wr"], a["softcap"], a["alibi"], a["splits"], a["ws"], a["wsb"],
                              a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(page=100), FA_ERR_INVALID_ARG),
    (dict(cs=None), FA_ERR_INVALID_ARG),            # paged cache needs cache_seqlens
    (dict(nblk=0), FA_ERR_INVALID_ARG),
    (dict(d=80), FA_ERR_UNSUPPORTED),
    (dict(splits=4, ws=None, wsb=0), FA_ERR_WORKSPACE),
    (dict(splits=1, ws=None, wsb=0), FA_ERR_WORKSPACE),       # the item counter lives there
    (dict(bt=None, skmax=-1), FA_ERR_INVALID_ARG),
    # the combine step weighs at most 256 partials: larger split counts are refused
    # before any device use (also on the path whose need fits a workspace)
    (dict(splits=257, ws=P, wsb=1 << 40), FA_ERR_INVALID_ARG),
    (dict(splits=512, maxb=1024, ws=P, wsb=1 << 40), FA_ERR_INVALID_ARG),
    # max_blocks_per_seq * page_size must fit an int
    (dict(maxb=1 << 24, page=256, ws=P, wsb=1 << 40), FA_ERR_INVALID_ARG),
])
def test_kvcache_validation(lib, kw, code):
    assert kvc(lib, **kw) == code


def test_splits_and_workspace_size(lib):
    # explicit split counts are clamped to the number of pages
    assert lib.fa_kvcache_num_splits(64, 1, 32, 8, 128, 32768, 256, 16) == 16
    assert lib.fa_kvcache_num_splits(64, 1, 32, 8, 128, 512, 256, 16) == 2
    assert lib.fa_kvcache_workspace_size(64, 1, 32, 8, 128, 32768, 256, 1) == 256
    assert lib.fa_kvcache_workspace_size(64, 1, 32, 8, 128, 32768, 256, 4) == 256 + 4 * 64 * 32 * 129 * 4
    # more than 16 query rows per KV head run the tensor-core kernel: no split partials
    assert lib.fa_kvcache_num_splits(4, 128, 32, 8, 128, 32768, 256, 16) == 1
    assert lib.fa_kvcache_workspace_size(4, 128, 32, 8, 128, 32768, 256, 16) == 256
    # split counts above 256 (the combine's limit) are bad input, whatever the route
    assert lib.fa_kvcache_num_splits(1, 1, 8, 8, 128, 1 << 20, 256, 256) == 256
    assert lib.fa_kvcache_num_splits(1, 1, 8, 8, 128, 1 << 20, 256, 257) <= 0
    assert lib.fa_kvcache_num_splits(4, 128, 32, 8, 128, 32768, 256, 300) <= 0
    assert lib.fa_kvcache_workspace_size(1, 1, 8, 8, 128, 1 << 20, 256, 512) == 256


def test_static_scratch_validation(lib):
    # the arguments the scratch-size check reads are validated first: a malformed
    # call gets FA_ERR_INVALID_ARG, as from fa_fwd_kvcache, before any device use
    st = lib.fa_fwd_kvcache_static
    args = [P, P, P, P, None, 1, 64, 1, 32, 8, 128, P, 128, 256, 8192, 0, P, float("nan"), 1,
            -1, -1, 0.0, None]
    assert st(*args, 300, None) == FA_ERR_INVALID_ARG             # num_splits > 256
    big = list(args)
    big[12] = 1 << 24                                             # max_blocks_per_seq * page
    assert st(*big, 4, None) == FA_ERR_INVALID_ARG
    # 64 x 32 x 129 fp32 partials at 128 splits need ~135 MB: beyond the fixed array
    assert st(*args, 128, None) == FA_ERR_WORKSPACE
    assert lib.fa_kvcache_static_scratch_bytes() == 24 << 20


def test_host_entry_validation(lib):
    # argument and workspace errors come back before any device use
    h = lib.fa_fwd_host
    ws = lib.fa_fwd_host_workspace_size(4, 256, 256, 8, 2, 64, 1)
    # 256 B of slopes, then two slots of one sequence each: q, k, v, out, lse
    q1, kv1, l1 = 256 * 8 * 64 * 2, 256 * 2 * 64 * 2, 8 * 256 * 4
    assert ws == 256 + 2 * (2 * q1 + 2 * kv1 + l1)
    assert lib.fa_fwd_host_workspace_size(4, 256, 256, 8, 2, 64, 0) == 256 + 2 * (2 * q1 + 2 * kv1)
    assert lib.fa_fwd_host_workspace_size(0, 256, 256, 8, 2, 64, 1) == 0
    # B=9: chunks of 3 sequences
    assert lib.fa_fwd_host_workspace_size(9, 128, 128, 1, 1, 128, 0) == \
        256 + 2 * (2 * 3 * 128 * 128 * 2 + 2 * 3 * 128 * 128 * 2)
    W = ctypes.c_void_p(1 << 20)  # never dereferenced: every case fails validation first
    good = [P, P, P, P, None, 0, 4, 256, 256, 8, 2, 64, float("nan"), 1, -1, -1, 0.0, None]
    ws0 = lib.fa_fwd_host_workspace_size(4, 256, 256, 8, 2, 64, 0)  # lse is NULL below
    def call(args, ws_ptr=W, ws_bytes=ws0):
        return h(*args, ws_ptr, ws_bytes, None)
    bad = list(good); bad[0] = None
    assert call(bad) == FA_ERR_INVALID_ARG
    bad = list(good); bad[5] = 2                                   # fp32 inputs
    assert call(bad) == FA_ERR_UNSUPPORTED
    bad = list(good); bad[10] = 3                                  # 8 heads over 3 KV heads
    assert call(bad) == FA_ERR_INVALID_ARG
    bad = list(good); bad[11] = 96
    assert call(bad) == FA_ERR_UNSUPPORTED
    assert call(good, ws_bytes=ws0 - 1) == FA_ERR_WORKSPACE
    assert call(good, ws_ptr=None) == FA_ERR_WORKSPACE
    assert call(good, ws_ptr=ctypes.c_void_p((1 << 20) + 16)) == FA_ERR_WORKSPACE  # alignment
    empty = list(good); empty[6] = 0
    assert call(empty) == FA_OK                                    # nothing to do


def test_combine_validation(lib):
    assert lib.fa_combine(P, P, P, None, 0, 1, 1, 1, 64, 0, None, None, None) == FA_ERR_INVALID_ARG
    assert lib.fa_combine(P, P, P, None, 0, 1, 1, 1, 64, 300, None, None, None) == FA_ERR_INVALID_ARG
    assert lib.fa_combine(P, P, P, None, 7, 1, 1, 1, 64, 2, None, None, None) == FA_ERR_UNSUPPORTED
    assert lib.fa_combine(P, P, P, None, 0, 1, 1, 1, 62, 2, None, None, None) == FA_ERR_INVALID_ARG


def test_timeout_setter(lib):
    assert lib.fa_set_wait_timeout_ms(0) == FA_ERR_INVALID_ARG
    assert lib.fa_set_wait_timeout_ms(1000) == FA_OK


def app(lib, **kw):
    a = dict(kc=P, vc=P, kn=P, vn=P, dtype=1, B=2, S=1, Hkv=8, d=128, bt=P, maxb=4, page=256,
             nblk=8, skmax=0, cs=P, stream=None)
    a.update(kw)
    return lib.fa_kvcache_append(a["kc"], a["vc"], a["kn"], a["vn"], a["dtype"], a["B"], a["S"],
                                 a["Hkv"], a["d"], a["bt"], a["maxb"], a["page"], a["nblk"],
                                 a["skmax"], a["cs"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(cs=None), FA_ERR_INVALID_ARG),            # the pre-append lengths are required
    (dict(dtype=2), FA_ERR_UNSUPPORTED),
    (dict(d=12), FA_ERR_UNSUPPORTED),
    (dict(kn=None), FA_ERR_INVALID_ARG),
    (dict(vc=MIS), FA_ERR_INVALID_ARG),
    (dict(Hkv=0), FA_ERR_INVALID_ARG),
    (dict(S=-1), FA_ERR_INVALID_ARG),
    (dict(page=0), FA_ERR_INVALID_ARG),
    (dict(bt=None, skmax=-1), FA_ERR_INVALID_ARG),
])
def test_append_validation(lib, kw, code):
    assert app(lib, **kw) == code
    assert lib.fa_last_error()


def test_append_empty_is_a_noop(lib):
    assert app(lib, B=0) == FA_OK
    assert app(lib, S=0) == FA_OK


def test_fwd_kvcache_append_validation(lib):
    args = [P, P, P, P, P, 1, P, None, 1, 2, 1, 32, 8, 128, P, 4, 256, 8, 0]
    tail = [float("nan"), 1, -1, -1, 0.0, None, 1, P, 4096, None]
    assert lib.fa_fwd_kvcache_append(*args, None, *tail) == FA_ERR_INVALID_ARG   # no cache_seqlens
    assert lib.fa_fwd_kvcache_append(*args, P, *tail[:-3], None, 0, None) == FA_ERR_WORKSPACE


def test_selftest_limit_validation(lib):
    assert lib.fa_selftest_wait_timeout(0, None) == FA_ERR_INVALID_ARG
    assert lib.fa_selftest_wait_timeout(20000, None) == FA_ERR_INVALID_ARG


def test_fp8_validation(lib):
    def f8(**kw):
        a = dict(qd=1.0, kd=1.0, vd=1.0, d=128)
        a.update(kw)
        return lib.fa_fwd_fp8(P, P, P, P, None, a["qd"], a["kd"], a["vd"], 1, 128, 128, 2, 2,
                              a["d"], None, None, None, None, None, None, 0, 0,
                              float("nan"), 0, -1, -1, 0.0, None, None)
    assert f8(d=64) == FA_ERR_UNSUPPORTED
    assert f8(qd=0.0) == FA_ERR_INVALID_ARG
    assert f8(vd=float("inf")) == FA_ERR_INVALID_ARG


def bwd(lib, **kw):
    a = dict(dout=P, q=P, k=P, v=P, out=P, lse=P, dq=P, dk=P, dv=P, dtype=1, B=1, Sq=256, Sk=256,
             H=2, Hkv=2, d=128, cuq=None, cuk=None, mq=0, mk=0, scale=float("nan"), causal=1,
             wl=-1, wr=-1, softcap=0.0, alibi=None, ws=P, ws_bytes=None, stream=None)
    a.update(kw)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = lib.fa_bwd_workspace_size(1 if a["cuq"] else a["B"], a["Sq"], a["H"])
    return lib.fa_bwd(a["dout"], a["q"], a["k"], a["v"], a["out"], a["lse"], a["dq"], a["dk"],
                      a["dv"], a["dtype"], a["B"], a["Sq"], a["Sk"], a["H"], a["Hkv"], a["d"],
                      a["cuq"], a["cuk"], a["mq"], a["mk"], a["scale"], a["causal"], a["wl"],
                      a["wr"], a["softcap"], a["alibi"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), FA_ERR_UNSUPPORTED),
    (dict(dtype=2), FA_ERR_UNSUPPORTED),
    (dict(softcap=-1.0), FA_ERR_INVALID_ARG),
    (dict(cuq=P), FA_ERR_INVALID_ARG),                      # varlen needs both offsets
    (dict(cuq=P, cuk=P, mq=300), FA_ERR_INVALID_ARG),      # max_seqlen above the total
    (dict(cuq=P, cuk=P, mq=200, mk=-1), FA_ERR_INVALID_ARG),
    (dict(H=3, Hkv=2), FA_ERR_INVALID_ARG),
    (dict(dout=None), FA_ERR_INVALID_ARG),
    (dict(lse=None), FA_ERR_INVALID_ARG),
    (dict(dk=MIS), FA_ERR_INVALID_ARG),
    (dict(lse=ctypes.c_void_p(0x10002)), FA_ERR_INVALID_ARG),  # lse must be 4-byte aligned
    (dict(Sk=-1), FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), FA_ERR_INVALID_ARG),
    (dict(ws=None), FA_ERR_WORKSPACE),
    (dict(ws_bytes=16), FA_ERR_WORKSPACE),
    (dict(ws=MIS), FA_ERR_WORKSPACE),
])
def test_bwd_validation(lib, kw, code):
    assert bwd(lib, **kw) == code
    assert lib.fa_last_error()


def test_bwd_workspace_size(lib):
    # two fp32 arrays (D and LSE * log2 e), rows padded to a multiple of 4, the total
    # rounded up to 256 bytes
    def up256(n):
        return (n + 255) // 256 * 256
    assert lib.fa_bwd_workspace_size(2, 130, 3) == up256(2 * 2 * 3 * 132 * 4)
    assert lib.fa_bwd_workspace_size(1, 128, 1) == up256(2 * 128 * 4)
    assert lib.fa_bwd_workspace_size(0, 128, 1) == 256


def test_bwd_empty_batch_is_a_noop(lib):
    assert bwd(lib, B=0) == FA_OK


def test_bwd_varlen_workspace_is_one_packed_entry(lib):
    # varlen: the statistics cover [num_heads, total_q]; a workspace sized for the
    # packed rows passes the check (an empty batch then returns before any launch)
    assert bwd(lib, B=0, cuq=P, cuk=P, mq=100, mk=100) == FA_OK
    assert bwd(lib, B=3, cuq=P, cuk=P, mq=100, mk=100, ws_bytes=16) == FA_ERR_WORKSPACE


def test_binding_refuses_host_tensors(lib):
    """The binding passes device addresses only: a host tensor is refused before
    any call into the library (stream=0 keeps the call free of CUDA on this host)."""
    q = torch.zeros(1, 128, 2, 64, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA tensors"):
        fa.fa_fwd(q, q, q, stream=0)
    with pytest.raises(ValueError, match="CUDA tensors"):
        fa.fa_bwd(q, q, q, q, q, torch.zeros(1, 2, 128), dq=q, dk=q, dv=q,
                  workspace=torch.zeros(4096, dtype=torch.uint8), stream=0)

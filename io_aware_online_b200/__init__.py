"""Python binding of the io_aware_online_b200 C-ABI attention library.

Argument marshalling only: every step of the computation runs in the CUDA kernels
of ``libfa_b200.so`` (built by ``io_aware_online_b200.build``).  PyTorch supplies
device memory and the current stream; outputs the caller does not pass are
allocated with ``torch.empty`` before the call.  There is no fallback: if the
library is missing or a call fails, an exception is raised.

Functions mirror include/fa.h:
    fa_fwd(q, k, v, ...)                  dense [B,S,H,d] or varlen [total,H,d]
    fa_fwd_host(q, k, v, ...)             dense, q/k/v/out in host memory (transfers
                                          overlapped with the kernels)
    fa_fwd_kvcache(q, k_cache, v_cache, ...)
    fa_fwd_kvcache_static(q, k_cache, v_cache, ...)   (no workspace; fixed device scratch)
    fa_combine(out_partial, lse_partial, ...)
    fa_kvcache_num_splits(...), fa_kvcache_workspace_size(...)
    fa_device_status(clear=True), fa_set_wait_timeout_ms(ms), fa_version()
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = ["FAError", "fa_fwd", "fa_fwd_host", "fa_fwd_host_workspace_size", "fa_fwd_kvcache", "fa_fwd_kvcache_static", "fa_combine",
           "fa_kvcache_num_splits",
           "fa_kvcache_workspace_size", "fa_device_status", "fa_set_wait_timeout_ms",
           "fa_version", "library_path", "load"]

FA_FP16, FA_BF16, FA_FP32 = 0, 1, 2
FA_DEV_WAIT_TIMEOUT, FA_DEV_BAD_BLOCK = 1, 2
_DT = {torch.float16: FA_FP16, torch.bfloat16: FA_BF16, torch.float32: FA_FP32}
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfa_b200.so")
_lib = None


class FAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[fa error {code}] {msg}")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libfa_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: run `python -m io_aware_online_b200.build` "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64p, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int64), ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i64p, i64p,
                           i64p, i64p, vp, vp, i32, i32, f32, i32, i32, i32, f32, vp, vp]
    lib.fa_fwd.restype = i32
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, f32, f32, f32, i32, i32, i32, i32, i32, i32,
                               i64p, i64p, i64p, i64p, vp, vp, i32, i32, f32, i32, i32, i32, f32,
                               vp, vp]
    lib.fa_fwd_fp8.restype = i32
    lib.fa_fwd_host_workspace_size.argtypes = [i32] * 7
    lib.fa_fwd_host_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_host.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                i32, i32, f32, vp, vp, ctypes.c_size_t, vp]
    lib.fa_fwd_host.restype = i32
    lib.fa_kvcache_num_splits.argtypes = [i32] * 8
    lib.fa_kvcache_num_splits.restype = i32
    lib.fa_kvcache_workspace_size.argtypes = [i32] * 8
    lib.fa_kvcache_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_kvcache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, i32,
                                   i32, i32, vp, f32, i32, i32, i32, f32, vp, i32, vp,
                                   ctypes.c_size_t, vp]
    lib.fa_fwd_kvcache.restype = i32
    lib.fa_fwd_kvcache_static.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                          i32, i32, i32, i32, vp, f32, i32, i32, i32, f32, vp,
                                          i32, vp]
    lib.fa_fwd_kvcache_static.restype = i32
    lib.fa_kvcache_append.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, i32, i32, i32,
                                      i32, vp, vp]
    lib.fa_kvcache_append.restype = i32
    lib.fa_fwd_kvcache_append.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                          i32, i32, vp, i32, i32, i32, i32, vp, f32, i32, i32,
                                          i32, f32, vp, i32, vp, ctypes.c_size_t, vp]
    lib.fa_fwd_kvcache_append.restype = i32
    lib.fa_kvcache_static_scratch_bytes.argtypes = []
    lib.fa_kvcache_static_scratch_bytes.restype = ctypes.c_size_t
    lib.fa_combine.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64p, i64p, vp]
    lib.fa_combine.restype = i32
    lib.fa_last_error.argtypes = []
    lib.fa_last_error.restype = ctypes.c_char_p
    lib.fa_device_status.argtypes = [i32, ctypes.POINTER(ctypes.c_uint)]
    lib.fa_device_status.restype = i32
    lib.fa_set_wait_timeout_ms.argtypes = [i32]
    lib.fa_set_wait_timeout_ms.restype = i32
    lib.fa_bwd_workspace_size.argtypes = [i32, i32, i32]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                           vp, vp, i32, i32, f32, i32, i32, i32, f32, vp, vp, ctypes.c_size_t, vp]
    lib.fa_bwd.restype = i32
    lib.fa_selftest_wait_timeout.argtypes = [i32, vp]
    lib.fa_selftest_wait_timeout.restype = i32
    lib.fa_version.argtypes = []
    lib.fa_version.restype = i32
    _lib = lib
    return lib


def _check(rc: int):
    if rc != 0:
        raise FAError(rc, load().fa_last_error().decode(errors="replace"))


def _ptr(t) -> ctypes.c_void_p | None:
    """Device address of a CUDA tensor (None stays NULL).  Host tensors, pinned ones
    included, are refused: every pointer of the C ABI is read by the kernels."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"tensor arguments must be CUDA tensors, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _i64(vals) -> ctypes.Array:
    return (ctypes.c_int64 * len(vals))(*[int(x) for x in vals])


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return ctypes.c_void_p(handle)


def _scale(softmax_scale) -> float:
    return float("nan") if softmax_scale is None else float(softmax_scale)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError(f"inputs must be float16 or bfloat16, got {t.dtype}")
    return _DT[t.dtype]


def fa_version() -> int:
    return load().fa_version()


def fa_set_wait_timeout_ms(ms: int) -> None:
    _check(load().fa_set_wait_timeout_ms(int(ms)))


def fa_device_status(clear: bool = True) -> int:
    """Synchronise and return the device status bits (FA_DEV_*), clearing them."""
    flags = ctypes.c_uint(0)
    rc = load().fa_device_status(int(bool(clear)), ctypes.byref(flags))
    if rc not in (0, 5):
        _check(rc)
    return int(flags.value)


def fa_fwd(q, k, v, *, out=None, lse=None, cu_seqlens_q=None, cu_seqlens_k=None,
           max_seqlen_q=None, max_seqlen_k=None, softmax_scale=None, causal=False,
           window_size=(-1, -1), softcap=0.0, alibi_slopes=None, return_lse=True, stream=None,
           _fp8=None):
    """Exact attention forward (sections 3.1 / 3.2 of the interface page).

    Dense: q [B, Sq, H, d], k/v [B, Sk, Hkv, d] -> out like q, lse [B, H, Sq].
    Varlen: q [total_q, H, d], k/v [total_k, Hkv, d], int32 cu_seqlens [B+1],
    max_seqlen_q/k -> out like q, lse [H, total_q].
    """
    lib = load()
    fp8 = _fp8
    dt = _DT[torch.bfloat16] if fp8 is not None else _dtype(q)
    varlen = cu_seqlens_q is not None or cu_seqlens_k is not None
    if varlen:
        total_q, H, d = q.shape
        total_k, Hkv = k.shape[0], k.shape[1]
        B = cu_seqlens_q.numel() - 1
        sq, sk = total_q, total_k
        qs = (0, q.stride(0), q.stride(1))
        ks = (0, k.stride(0), k.stride(1))
        vs = (0, v.stride(0), v.stride(1))
        if max_seqlen_q is None or max_seqlen_k is None:
            raise ValueError("varlen needs max_seqlen_q and max_seqlen_k")
    else:
        B, sq, H, d = q.shape
        sk, Hkv = k.shape[1], k.shape[2]
        qs = (q.stride(0), q.stride(1), q.stride(2))
        ks = (k.stride(0), k.stride(1), k.stride(2))
        vs = (v.stride(0), v.stride(1), v.stride(2))
        max_seqlen_q = max_seqlen_k = 0
    for t in (q, k, v):
        if t.stride(-1) != 1:
            raise ValueError("the head_dim axis must be contiguous")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    os_ = (0, out.stride(0), out.stride(1)) if varlen else (out.stride(0), out.stride(1),
                                                            out.stride(2))
    if lse is None and return_lse:
        shape = (H, sq) if varlen else (B, H, sq)
        lse = torch.empty(shape, dtype=torch.float32, device=q.device)
    args = (_i64(qs), _i64(ks), _i64(vs), _i64(os_), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
            int(max_seqlen_q), int(max_seqlen_k), _scale(softmax_scale), int(bool(causal)),
            int(window_size[0]), int(window_size[1]), float(softcap), _ptr(alibi_slopes),
            _stream(stream))
    if fp8 is None:
        _check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), dt, B, sq, sk, H, Hkv,
                          d, *args))
    else:
        _check(lib.fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), *fp8, B, sq, sk,
                              H, Hkv, d, *args))
    return out, lse


def _host_ptr(t) -> ctypes.c_void_p | None:
    """Address of a contiguous CPU tensor (page-locked ones let the copies overlap)."""
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("fa_fwd_host takes contiguous CPU tensors")
    return ctypes.c_void_p(t.data_ptr())


def fa_fwd_host_workspace_size(batch, seqlen_q, seqlen_k, num_heads, num_heads_k, head_dim,
                               with_lse=True) -> int:
    return int(load().fa_fwd_host_workspace_size(batch, seqlen_q, seqlen_k, num_heads,
                                                 num_heads_k, head_dim, int(bool(with_lse))))


def fa_fwd_host(q, k, v, *, out=None, lse=None, softmax_scale=None, causal=False,
                window_size=(-1, -1), softcap=0.0, alibi_slopes=None, return_lse=True,
                workspace=None, stream=None):
    """fa_fwd on dense q [B, Sq, H, d], k/v [B, Sk, Hkv, d] in host memory; out (and lse
    [B, H, Sq], and alibi_slopes [H]) in host memory too.  The library copies the batch
    through a device workspace (on the current CUDA device) chunk by chunk, overlapping
    the copies with the kernels.  When `stream` (default: the current stream) has passed
    the call, out and lse hold the results."""
    lib = load()
    dt = _dtype(q)
    B, sq, H, d = q.shape
    sk, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if lse is None and return_lse:
        lse = torch.empty((B, H, sq), dtype=torch.float32, pin_memory=True)
    if workspace is None:
        n = fa_fwd_host_workspace_size(B, sq, sk, H, Hkv, d, lse is not None)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8,
                                device=torch.device("cuda", torch.cuda.current_device()))
    if alibi_slopes is not None and (alibi_slopes.is_cuda or alibi_slopes.dtype != torch.float32):
        raise ValueError("fa_fwd_host takes fp32 CPU alibi_slopes")
    _check(lib.fa_fwd_host(_host_ptr(q), _host_ptr(k), _host_ptr(v), _host_ptr(out),
                           _host_ptr(lse), dt, B, sq, sk, H, Hkv, d, _scale(softmax_scale),
                           int(bool(causal)), int(window_size[0]), int(window_size[1]),
                           float(softcap), _host_ptr(alibi_slopes), _ptr(workspace),
                           workspace.numel(), _stream(stream)))
    return out, lse


def fa_fwd_fp8(q, k, v, *, q_descale=1.0, k_descale=1.0, v_descale=1.0, **kw):
    """fa_fwd on float8_e4m3fn q, k, v (head_dim 128) with per-tensor descale
    factors (the real inputs are q * q_descale etc.); out is bf16.  Other keywords
    as for fa_fwd."""
    for t in (q, k, v):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError("fa_fwd_fp8 takes float8_e4m3fn q, k, v")
    if kw.get("out") is None:
        kw["out"] = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    return fa_fwd(q, k, v, _fp8=(float(q_descale), float(k_descale), float(v_descale)), **kw)


def fa_kvcache_num_splits(batch, seqlen_q, num_heads, num_heads_k, head_dim, max_seqlen_k,
                          page_size=0, num_splits=0) -> int:
    return load().fa_kvcache_num_splits(batch, seqlen_q, num_heads, num_heads_k, head_dim,
                                        max_seqlen_k, page_size, num_splits)


def fa_kvcache_workspace_size(batch, seqlen_q, num_heads, num_heads_k, head_dim, max_seqlen_k,
                              page_size=0, num_splits=0) -> int:
    return int(load().fa_kvcache_workspace_size(batch, seqlen_q, num_heads, num_heads_k,
                                                head_dim, max_seqlen_k, page_size, num_splits))


def _cache_geometry(k_cache, block_table):
    if block_table is not None:
        return k_cache.shape[2], k_cache.shape[0], k_cache.shape[1], block_table.shape[1], 0
    return k_cache.shape[2], 0, 0, 0, k_cache.shape[1]   # Hkv, num_blocks, page, max_blocks, sk_max


def fa_kvcache_append(k_cache, v_cache, k, v, cache_seqlens, *, block_table=None, stream=None):
    """Write k, v [B, S_new, Hkv, d] into the cache at positions cache_seqlens[b] + t
    (cache_seqlens = keys already cached; it is not advanced here)."""
    lib = load()
    dt = _dtype(k)
    B, s_new, Hkv, d = k.shape
    for t in (k_cache, v_cache, k, v):
        if not t.is_contiguous():
            raise ValueError("the caches and the new keys/values must be contiguous")
    _, num_blocks, page, max_blocks, sk_max = _cache_geometry(k_cache, block_table)
    _check(lib.fa_kvcache_append(_ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v), dt, B, s_new,
                                 Hkv, d, _ptr(block_table), max_blocks, page, num_blocks, sk_max,
                                 _ptr(cache_seqlens), _stream(stream)))


def fa_fwd_kvcache(q, k_cache, v_cache, k=None, v=None, *, cache_seqlens=None, block_table=None,
                   softmax_scale=None, causal=False, window_size=(-1, -1), softcap=0.0,
                   alibi_slopes=None, num_splits=0, out=None, lse=None, return_lse=True,
                   workspace=None, stream=None):
    """Split-KV attention against a paged or contiguous KV cache (section 3.3).
    q [B, Sq, H, d]; paged pools [num_blocks, page, Hkv, d] with int32 block_table
    [B, max_blocks]; or contiguous caches [B, Sk_max, Hkv, d].  With k and v
    [B, S_new, Hkv, d] given, they are first written into the cache after the
    cache_seqlens[b] keys already there, and the attention covers
    cache_seqlens[b] + S_new keys (cache_seqlens itself is not advanced)."""
    lib = load()
    dt = _dtype(q)
    B, sq, H, d = q.shape
    for t in (q, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("q and the caches must be contiguous")
    if (k is None) != (v is None):
        raise ValueError("give both k and v, or neither")
    if k is not None and not (k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k and v must be contiguous")
    if block_table is not None:
        num_blocks, page, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
        max_blocks = block_table.shape[1]
        sk_max = 0
        max_k = max_blocks * page
    else:
        num_blocks, page, max_blocks = 0, 0, 0
        sk_max, Hkv = k_cache.shape[1], k_cache.shape[2]
        max_k = sk_max
    need = fa_kvcache_workspace_size(B, sq, H, Hkv, d, max_k, page, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, sq), dtype=torch.float32, device=q.device)
    if k is None:
        _check(lib.fa_fwd_kvcache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                  dt, B, sq, H, Hkv, d, _ptr(block_table), max_blocks, page,
                                  num_blocks, sk_max, _ptr(cache_seqlens), _scale(softmax_scale),
                                  int(bool(causal)), int(window_size[0]), int(window_size[1]),
                                  float(softcap), _ptr(alibi_slopes), int(num_splits),
                                  _ptr(workspace), ws_bytes, _stream(stream)))
    else:
        _check(lib.fa_fwd_kvcache_append(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v),
                                         k.shape[1], _ptr(out), _ptr(lse), dt, B, sq, H, Hkv, d,
                                         _ptr(block_table), max_blocks, page, num_blocks, sk_max,
                                         _ptr(cache_seqlens), _scale(softmax_scale),
                                         int(bool(causal)), int(window_size[0]),
                                         int(window_size[1]), float(softcap),
                                         _ptr(alibi_slopes), int(num_splits), _ptr(workspace),
                                         ws_bytes, _stream(stream)))
    return out, lse


def fa_fwd_kvcache_static(q, k_cache, v_cache, *, cache_seqlens=None, block_table=None,
                          softmax_scale=None, causal=False, window_size=(-1, -1), softcap=0.0,
                          alibi_slopes=None, num_splits=0, out=None, lse=None,
                          return_lse=True, stream=None):
    """fa_fwd_kvcache for callers that cannot allocate device memory at the call:
    the scratch comes from the library's fixed device array (see include/fa.h).
    Outputs not passed in are allocated here by torch, before the call."""
    lib = load()
    dt = _dtype(q)
    B, sq, H, d = q.shape
    for t in (q, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("q and the caches must be contiguous")
    if block_table is not None:
        num_blocks, page, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
        max_blocks, sk_max = block_table.shape[1], 0
    else:
        num_blocks, page, max_blocks = 0, 0, 0
        sk_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, sq), dtype=torch.float32, device=q.device)
    _check(lib.fa_fwd_kvcache_static(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                     dt, B, sq, H, Hkv, d, _ptr(block_table), max_blocks, page,
                                     num_blocks, sk_max, _ptr(cache_seqlens),
                                     _scale(softmax_scale), int(bool(causal)),
                                     int(window_size[0]), int(window_size[1]), float(softcap),
                                     _ptr(alibi_slopes), int(num_splits), _stream(stream)))
    return out, lse


def fa_combine(out_partial, lse_partial, *, out_dtype=torch.float32, out=None, lse=None,
               return_lse=True, stream=None):
    """LSE-weighted combine (section 3.4): out_partial [B, S, H, d, splits] and
    lse_partial [B, S, H, splits] (any strides) -> out [B, S, H, d], lse [B, H, S]."""
    lib = load()
    B, S, H, d, splits = out_partial.shape
    if out is None:
        out = torch.empty((B, S, H, d), dtype=out_dtype, device=out_partial.device)
    if lse is None and return_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=out_partial.device)
    if out_partial.dtype != torch.float32 or lse_partial.dtype != torch.float32:
        raise TypeError("partials must be float32")
    _check(lib.fa_combine(_ptr(out_partial), _ptr(lse_partial), _ptr(out), _ptr(lse),
                          _DT[out.dtype], B, S, H, d, splits, _i64(out_partial.stride()),
                          _i64(lse_partial.stride()), _stream(stream)))
    return out, lse


def fa_selftest_wait_timeout(timeout_ms=20, stream=None):
    """Launch the bounded-wait self-test (include/fa.h): after timeout_ms the waiting
    CTA raises FA_DEV_WAIT_TIMEOUT in the device status word and exits."""
    _check(load().fa_selftest_wait_timeout(int(timeout_ms), _stream(stream)))


def fa_bwd(dout, q, k, v, out, lse, *, cu_seqlens_q=None, cu_seqlens_k=None,
           max_seqlen_q=None, max_seqlen_k=None, softmax_scale=None, causal=False,
           window_size=(-1, -1), softcap=0.0, alibi_slopes=None, dq=None, dk=None, dv=None,
           workspace=None, stream=None):
    """Gradients (dq, dk, dv) of the forward for output gradient dout (same mask,
    scale, softcap and ALiBi arguments as the forward call).
    Dense: q, out, dout [B, Sq, H, d], k, v [B, Sk, Hkv, d] contiguous, lse [B, H, Sq].
    Varlen: q, out, dout [total_q, H, d], k, v [total_k, Hkv, d], int32 cu_seqlens
    [B+1], max_seqlen_q/k, lse [H, total_q] (fa_fwd's varlen outputs)."""
    lib = load()
    dt = _dtype(q)
    varlen = cu_seqlens_q is not None or cu_seqlens_k is not None
    if varlen:
        if cu_seqlens_q is None or cu_seqlens_k is None:
            raise ValueError("varlen needs cu_seqlens_q and cu_seqlens_k")
        if max_seqlen_q is None or max_seqlen_k is None:
            raise ValueError("varlen needs max_seqlen_q and max_seqlen_k")
        B = cu_seqlens_q.numel() - 1
        sq, H, d = q.shape
        sk, Hkv = k.shape[0], k.shape[1]
        ws_b = 1
    else:
        B, sq, H, d = q.shape
        sk, Hkv = k.shape[1], k.shape[2]
        max_seqlen_q = max_seqlen_k = 0
        ws_b = B
    for t in (dout, q, k, v, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_bwd takes contiguous tensors")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = lib.fa_bwd_workspace_size(ws_b, sq, H)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.fa_bwd(_ptr(dout), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dq),
                      _ptr(dk), _ptr(dv), dt, B, sq, sk, H, Hkv, d, _ptr(cu_seqlens_q),
                      _ptr(cu_seqlens_k), int(max_seqlen_q), int(max_seqlen_k),
                      _scale(softmax_scale), int(bool(causal)), int(window_size[0]),
                      int(window_size[1]), float(softcap), _ptr(alibi_slopes), _ptr(workspace),
                      ws_bytes, _stream(stream)))
    return dq, dk, dv

"""fp64 CPU oracle for the exact attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, loads or calls it, and it shares no code with
them.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, two-pass softmax over a
fully materialised score row; see that file's header for the definition and the
passages it follows).  This module only marshals numpy arrays into it and
compiles it with gcc on first use.

Functions
---------
attention(q, k, v, cu_q, cu_k, ...)        dense or varlen (packed rows)
attention_dense(q, k, v, ...)              [B, S, H, d] convenience form
attention_paged(q, kpool, vpool, block_table, cache_seqlens, ...)
combine(out_partial, lse_partial)          LSE-weighted combine of split partials
append(kcache, vcache, k_new, v_new, cache_seqlens, block_table=None)
                                           KV-cache append (returns updated copies)
attention_backward(q, k, v, do, ...)       gradients dq, dk, dv (backward.py, numpy fp64)
attention_backward_varlen(q, k, v, do, cu_q, cu_k, ...)  the same over packed sequences
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            i32p = ctypes.POINTER(ctypes.c_int32)
            lib.oracle_attention.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, i64p, i64p,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_double, dp, ctypes.c_int]
            lib.oracle_attention.restype = ctypes.c_int
            lib.oracle_attention_paged.argtypes = [
                dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_long, i32p,
                ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                dp, ctypes.c_int]
            lib.oracle_attention_paged.restype = ctypes.c_int
            lib.oracle_combine.argtypes = [dp, dp, dp, dp, ctypes.c_long, ctypes.c_int,
                                           ctypes.c_int]
            lib.oracle_combine.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Exact upcast to a C-contiguous fp64 numpy array (accepts torch tensors)."""
    if hasattr(a, "detach"):  # torch tensor: 16-bit values upcast exactly
        a = a.detach().to("cpu").double().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def attention(q, k, v, cu_q, cu_k, *, scale: float | None = None, causal: bool = False,
              window=(-1, -1), softcap: float = 0.0, alibi_slopes=None,
              threads: int | None = None):
    """Packed-row (varlen) attention.

    q [total_q, H, d], k/v [total_k, Hkv, d]; cu_q/cu_k int [nseq+1].
    Returns (out [total_q, H, d] fp64, lse [total_q, H] fp64).
    ``scale`` None means 1/sqrt(d) (section 3.1: softmax_scale default).
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int64))
    cu_k = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int64))
    total_q, H, d = q.shape
    Hkv = k.shape[1]
    assert k.shape == v.shape and k.shape[2] == d
    nseq = len(cu_q) - 1
    assert len(cu_k) == nseq + 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((total_q, H, d), dtype=np.float64)
    lse = np.zeros((total_q, H), dtype=np.float64)
    slopes = None if alibi_slopes is None else _f64(alibi_slopes).reshape(H)
    rc = lib.oracle_attention(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                              _ptr(v, ctypes.c_double), _ptr(out, ctypes.c_double),
                              _ptr(lse, ctypes.c_double), nseq, _ptr(cu_q, ctypes.c_int64),
                              _ptr(cu_k, ctypes.c_int64), H, Hkv, d, float(scale),
                              int(bool(causal)), int(window[0]), int(window[1]),
                              float(softcap),
                              None if slopes is None else _ptr(slopes, ctypes.c_double),
                              int(threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attention: bad arguments")
    return out, lse


def attention_dense(q, k, v, **kw):
    """q [B, Sq, H, d], k/v [B, Sk, Hkv, d] -> (out [B, Sq, H, d], lse [B, H, Sq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, H, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    cu_q = np.arange(B + 1, dtype=np.int64) * Sq
    cu_k = np.arange(B + 1, dtype=np.int64) * Sk
    out, lse = attention(q.reshape(B * Sq, H, d), k.reshape(B * Sk, Hkv, d),
                         v.reshape(B * Sk, Hkv, d), cu_q, cu_k, **kw)
    return out.reshape(B, Sq, H, d), lse.reshape(B, Sq, H).transpose(0, 2, 1).copy()


def attention_paged(q, kpool, vpool, block_table, cache_seqlens, *, scale=None,
                    causal=False, window=(-1, -1), softcap=0.0, alibi_slopes=None,
                    threads=None):
    """q [B, Sq, H, d]; kpool/vpool [num_blocks, page, Hkv, d];
    block_table int32 [B, max_blocks]; cache_seqlens int32 [B].
    Returns (out [B, Sq, H, d], lse [B, H, Sq])."""
    lib = _load()
    q, kpool, vpool = _f64(q), _f64(kpool), _f64(vpool)
    bt = np.ascontiguousarray(np.asarray(
        block_table.cpu() if hasattr(block_table, "cpu") else block_table, dtype=np.int32))
    cs = np.ascontiguousarray(np.asarray(
        cache_seqlens.cpu() if hasattr(cache_seqlens, "cpu") else cache_seqlens,
        dtype=np.int32))
    B, Sq, H, d = q.shape
    nblk, page, Hkv, _ = kpool.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Sq, H, d), dtype=np.float64)
    lse = np.zeros((B, Sq, H), dtype=np.float64)
    slopes = None if alibi_slopes is None else _f64(alibi_slopes).reshape(H)
    rc = lib.oracle_attention_paged(
        _ptr(q, ctypes.c_double), _ptr(kpool, ctypes.c_double), _ptr(vpool, ctypes.c_double),
        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double), B, Sq, H, Hkv, d,
        _ptr(bt, ctypes.c_int32), bt.shape[1], page, nblk, _ptr(cs, ctypes.c_int32),
        float(scale), int(bool(causal)), int(window[0]), int(window[1]), float(softcap),
        None if slopes is None else _ptr(slopes, ctypes.c_double),
        int(threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attention_paged: bad arguments")
    return out, lse.transpose(0, 2, 1).copy()


def combine(out_partial, lse_partial):
    """out_partial [..., d, splits], lse_partial [..., splits] (the pages' layout).
    Returns (out [..., d], lse [...])."""
    lib = _load()
    op, lp = _f64(out_partial), _f64(lse_partial)
    *lead, d, splits = op.shape
    assert list(lp.shape) == list(lead) + [splits]
    rows = int(np.prod(lead)) if lead else 1
    out = np.zeros((rows, d), dtype=np.float64)
    lse = np.zeros((rows,), dtype=np.float64)
    rc = lib.oracle_combine(_ptr(op, ctypes.c_double), _ptr(lp, ctypes.c_double),
                            _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double), rows, d,
                            splits)
    if rc != 0:
        raise ValueError("oracle_combine: bad arguments")
    return out.reshape(*lead, d), lse.reshape(*lead)


def append(kcache, vcache, k_new, v_new, cache_seqlens, block_table=None):
    """KV-cache append ("flash attention" tag page, section 3.3: with k and v given,
    flash_attn_with_kvcache writes them into the cache).  Row t of sequence b goes to
    key position x = cache_seqlens[b] + t, cache_seqlens counting the keys already
    cached.  Paged cache [num_blocks, page, Hkv, d]: position x of sequence b is row
    x % page of block block_table[b, x // page]; contiguous cache [B, Sk_max, Hkv, d]:
    row x of sequence b.  Returns updated copies (inputs untouched) as torch CPU
    tensors of the caches' dtype; a position outside the cache raises IndexError.
    Plain element copies, one (b, t) row at a time."""
    import torch
    kc = torch.as_tensor(kcache).cpu().clone()
    vc = torch.as_tensor(vcache).cpu().clone()
    kn = torch.as_tensor(k_new).cpu()
    vn = torch.as_tensor(v_new).cpu()
    cs = [int(x) for x in torch.as_tensor(cache_seqlens).cpu().tolist()]
    bt = None if block_table is None else torch.as_tensor(block_table).cpu().tolist()
    B, s_new = kn.shape[0], kn.shape[1]
    for b in range(B):
        for t in range(s_new):
            x = cs[b] + t
            if bt is not None:
                page = kc.shape[1]
                if x < 0 or x // page >= len(bt[b]):
                    raise IndexError(f"position {x} of sequence {b} is outside the block table")
                blk = bt[b][x // page]
                if not 0 <= blk < kc.shape[0]:
                    raise IndexError(f"block {blk} outside the pool")
                kc[blk, x % page] = kn[b, t]
                vc[blk, x % page] = vn[b, t]
            else:
                if not 0 <= x < kc.shape[1]:
                    raise IndexError(f"position {x} of sequence {b} is outside the cache")
                kc[b, x] = kn[b, t]
                vc[b, x] = vn[b, t]
    return kc, vc


from .backward import attention_backward, attention_backward_varlen  # noqa: E402,F401  (fp64 gradients; see backward.py)

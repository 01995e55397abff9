"""fp64 CPU oracle for block top-k sparse decode over a paged KV cache.

TEST INFRASTRUCTURE ONLY.  Only tests/, the package's smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path (the CUDA library and its
binding) never imports, links or calls it, and this module imports nothing from the
product package.

Thin numpy/ctypes wrapper over vx_oracle.c; all arithmetic lives in the C file.  bf16
arrays are passed as uint16 bit patterns.  Every function returns freshly allocated
numpy arrays.
"""
import contextlib
import ctypes

import numpy as np

from . import build as _build

_default = None
_override = None


def _declare(lib):
    i32, i64, u64, dbl, p = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
    lib.orc_centroids.argtypes = [p, i32, i32, i32, i32, p, p, p, p, p]
    lib.orc_append.argtypes = [p, p, i32, i32, i32, i32, i32, i32, p, p, p, p, p]
    lib.orc_prefill_write.argtypes = [p, p, i32, i32, i32, i32, i32, i32, i32, p, p, p, p, p, p]
    lib.orc_scores.argtypes = [p, p, p, i32, i32, i32, i32, i32, i32, p, p, p, i32, p]
    lib.orc_topk_exact.argtypes = [p, i32, i32, i32, p, i32, i32, p]
    lib.orc_topk_approx.argtypes = [p, i32, i32, i32, p, i32, i32, i32, u64, p]
    lib.orc_splitmix64.argtypes = [u64, u64]
    lib.orc_splitmix64.restype = u64
    lib.orc_attend.argtypes = [p, p, p, i32, i32, i32, i32, i32, i32, i32, p, p, p, p, i32, dbl, p, p]
    lib.orc_decode_step.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, i32, i64, p, p, p,
                                    i32, i32, dbl, p, p, p, p]
    lib.orc_widen_bf16.argtypes = [p, i64, p]
    lib.orc_narrow_bf16.argtypes = [p, i64, p]
    lib.orc_num_threads.restype = ctypes.c_int
    lib.orc_set_num_threads.argtypes = [ctypes.c_int]
    lib.orc_set_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _default
    if _override is not None:
        return _override
    if _default is None:
        _default = _declare(ctypes.CDLL(_build.build()))
    return _default


@contextlib.contextmanager
def using(lib_path):
    """Route every call to another build of vx_oracle.c while the block runs.

    Used by the mutation test, which plants a mistake in a copy of the C source and
    checks that the pins catch it."""
    global _override
    prev = _override
    _override = _declare(ctypes.CDLL(lib_path))
    try:
        yield
    finally:
        _override = prev


def _c(a, dtype):
    """Contiguous array of the given dtype (bf16 must already be uint16 bits)."""
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        if dtype == np.uint16:
            raise TypeError("bf16 arrays are passed as uint16 bit patterns")
        a = a.astype(dtype)
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> int:
    """Threads the following oracle calls use on this host thread; returns the previous count."""
    return int(_load().orc_set_num_threads(int(n)))


def widen_bf16(bits):
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, np.float64)
    _load().orc_widen_bf16(_p(bits), bits.size, _p(out))
    return out


def narrow_bf16(x):
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().orc_narrow_bf16(_p(x), x.size, _p(out))
    return out


def splitmix64(seed: int, i: int) -> int:
    return int(_load().orc_splitmix64(seed & (2**64 - 1), i & (2**64 - 1)))


def centroids(k_cache, page_ptr, page_indices, seq_lens):
    """Page key centroids keyed by physical page: (exact fp64 mean, stored bf16 bits).

    k_cache: uint16 [Npool][Hkv][P][Dqk].  Unreferenced pages come back as NaN / 0."""
    k_cache = _c(k_cache, np.uint16)
    npool, hkv, P, dqk = k_cache.shape
    page_ptr, page_indices, seq_lens = (_c(page_ptr, np.int32), _c(page_indices, np.int32),
                                        _c(seq_lens, np.int32))
    cen64 = np.full((npool, hkv, dqk), np.nan, np.float64)
    cen16 = np.zeros((npool, hkv, dqk), np.uint16)
    _load().orc_centroids(_p(k_cache), hkv, P, dqk, len(seq_lens), _p(page_ptr), _p(page_indices),
                          _p(seq_lens), _p(cen64), _p(cen16))
    return cen64, cen16


def append(k_cache, v_cache, page_ptr, page_indices, seq_lens, k_new, v_new, mla_shared_kv=False):
    """Write one new token per request into copies of the caches; returns (k, v)."""
    k = np.array(_c(k_cache, np.uint16), copy=True)
    v = None if mla_shared_kv else np.array(_c(v_cache, np.uint16), copy=True)
    npool, hkv, P, dqk = k.shape
    dv = dqk if v is None else v.shape[-1]
    page_ptr, page_indices, seq_lens = (_c(page_ptr, np.int32), _c(page_indices, np.int32),
                                        _c(seq_lens, np.int32))
    k_new = _c(k_new, np.uint16)
    v_new = None if mla_shared_kv else _c(v_new, np.uint16)
    _load().orc_append(_p(k), _p(v), int(mla_shared_kv), hkv, P, dqk, dv, len(seq_lens), _p(page_ptr),
                       _p(page_indices), _p(seq_lens), _p(k_new), _p(v_new))
    return k, v


def prefill_write(k_cache, v_cache, page_ptr, page_indices, seq_lens, first_pos, k_new, v_new, max_len,
                  mla_shared_kv=False):
    """Write positions [first_pos[b], seq_lens[b]) of every request, packed in request order in
    k_new [N][Hkv][Dqk] / v_new [N][Hkv][Dv], into copies of the caches; returns (k, v)."""
    k = np.array(_c(k_cache, np.uint16), copy=True)
    v = None if mla_shared_kv else np.array(_c(v_cache, np.uint16), copy=True)
    npool, hkv, P, dqk = k.shape
    dv = dqk if v is None else v.shape[-1]
    page_ptr, page_indices, seq_lens, first_pos = (_c(page_ptr, np.int32), _c(page_indices, np.int32),
                                                   _c(seq_lens, np.int32), _c(first_pos, np.int32))
    k_new = _c(k_new, np.uint16)
    v_new = None if mla_shared_kv else _c(v_new, np.uint16)
    _load().orc_prefill_write(_p(k), _p(v), int(mla_shared_kv), hkv, P, dqk, dv, len(seq_lens), int(max_len),
                              _p(page_ptr), _p(page_indices), _p(seq_lens), _p(first_pos), _p(k_new), _p(v_new))
    return k, v


def scores(q, page_ptr, page_indices, seq_lens, page_size, max_pages, num_kv_heads,
           centroids_f64=None, centroids_bf16=None, score_dims=0):
    """Group-summed page scores [B][Hkv][max_pages] (NaN where j >= n_b)."""
    q = _c(q, np.uint16)
    B, hq, dqk = q.shape
    page_ptr, page_indices, seq_lens = (_c(page_ptr, np.int32), _c(page_indices, np.int32),
                                        _c(seq_lens, np.int32))
    c64 = None if centroids_f64 is None else _c(centroids_f64, np.float64)
    c16 = None if centroids_bf16 is None else _c(centroids_bf16, np.uint16)
    if c64 is None and c16 is None:
        raise ValueError("pass centroids_f64 or centroids_bf16")
    out = np.full((B, num_kv_heads, max_pages), np.nan, np.float64)
    _load().orc_scores(_p(q), _p(c64), _p(c16), B, hq, num_kv_heads, dqk, score_dims, page_size,
                       _p(page_ptr), _p(page_indices), _p(seq_lens), max_pages, _p(out))
    return out


def topk_exact(scores_, seq_lens, page_size, k):
    """Exact top-k logical pages per (b, h) row, ascending page order, -1 padded."""
    s = _c(scores_, np.float64)
    B, hkv, max_pages = s.shape
    seq_lens = _c(seq_lens, np.int32)
    sel = np.empty((B, hkv, k), np.int32)
    _load().orc_topk_exact(_p(s), B, hkv, max_pages, _p(seq_lens), page_size, k, _p(sel))
    return sel


def topk_approx(scores_f32, seq_lens, page_size, k, seed, bits=12):
    """Approximate top-k (remap to `bits`-bit codes, one histogram, seeded fill)."""
    s = _c(scores_f32, np.float32)
    B, hkv, max_pages = s.shape
    seq_lens = _c(seq_lens, np.int32)
    sel = np.empty((B, hkv, k), np.int32)
    _load().orc_topk_approx(_p(s), B, hkv, max_pages, _p(seq_lens), page_size, k, bits,
                            seed & (2**64 - 1), _p(sel))
    return sel


def attend(q, k_cache, v_cache, page_ptr, page_indices, seq_lens, sel=None, sm_scale=None,
           mla_shared_kv=False, head_dim_v=None):
    """Exact attention over the selected pages (sel=None: every page, i.e. dense).

    Returns (out fp64 [B][Hq][Dv], lse fp64 [B][Hq])."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    B, hq, dqk = q.shape
    npool, hkv, P, _ = k_cache.shape
    if mla_shared_kv:
        dv = head_dim_v
        v_cache = None
    else:
        v_cache = _c(v_cache, np.uint16)
        dv = v_cache.shape[-1]
    page_ptr, page_indices, seq_lens = (_c(page_ptr, np.int32), _c(page_indices, np.int32),
                                        _c(seq_lens, np.int32))
    k = 0
    if sel is not None:
        sel = _c(sel, np.int32)
        k = sel.shape[-1]
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(dqk)
    out = np.empty((B, hq, dv), np.float64)
    lse = np.empty((B, hq), np.float64)
    _load().orc_attend(_p(q), _p(k_cache), _p(v_cache), int(mla_shared_kv), B, hq, hkv, dqk, dv, P,
                       _p(page_ptr), _p(page_indices), _p(seq_lens), _p(sel), k, float(sm_scale),
                       _p(out), _p(lse))
    return out, lse


def decode_step(q, k_cache, v_cache, centroids_bf16, page_ptr, page_indices, seq_lens, max_pages, k,
                sm_scale=None, mla_shared_kv=False, head_dim_v=None):
    """Score + exact top-k + attention, as the method runs one decode step.

    Returns (scores, sel, out, lse)."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    c16 = _c(centroids_bf16, np.uint16)
    B, hq, dqk = q.shape
    npool, hkv, P, _ = k_cache.shape
    if mla_shared_kv:
        dv, v_cache = head_dim_v, None
    else:
        v_cache = _c(v_cache, np.uint16)
        dv = v_cache.shape[-1]
    page_ptr, page_indices, seq_lens = (_c(page_ptr, np.int32), _c(page_indices, np.int32),
                                        _c(seq_lens, np.int32))
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(dqk)
    sc = np.full((B, hkv, max_pages), np.nan, np.float64)
    sel = np.empty((B, hkv, k), np.int32)
    out = np.empty((B, hq, dv), np.float64)
    lse = np.empty((B, hq), np.float64)
    _load().orc_decode_step(_p(q), _p(k_cache), _p(v_cache), _p(c16), int(mla_shared_kv), B, hq, hkv,
                            dqk, dv, P, npool, _p(page_ptr), _p(page_indices), _p(seq_lens), max_pages,
                            k, float(sm_scale), _p(sc), _p(sel), _p(out), _p(lse))
    return sc, sel, out, lse

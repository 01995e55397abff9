"""Python binding of libvx (include/vx.h): argument marshalling only.

Every function has the name of the C entry point it calls and does nothing but turn
torch tensors into pointers and sizes, call the library on the current CUDA stream and
raise VxError on a non-zero status.  All computation runs in libvx's CUDA kernels; there
is no fallback: if libvx.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvx.so")

VX_OK, VX_ERR_INVALID_ARG, VX_ERR_UNSUPPORTED, VX_ERR_WORKSPACE, VX_ERR_CUDA = range(5)
VX_DATA_BAD_PAGE_ID, VX_DATA_BAD_SEQ_LEN, VX_DATA_BAD_SELECTION, VX_DATA_TIMEOUT = 1, 2, 4, 8
NOALLOC_SCRATCH_BYTES = 16 << 20  # VX_NOALLOC_SCRATCH_BYTES of include/vx.h
VX_TABLE_READY = 0x100  # mode flag of the chained steps: the table and lengths are not the previous kernel's output

# every symbol include/vx.h declares
EXPORTS = ["vx_centroid_update", "vx_score_pages", "vx_topk_pages", "vx_sparse_decode",
           "vx_sparse_decode_noalloc", "vx_block_topk_decode", "vx_block_topk_decode_append",
           "vx_block_topk_decode_persistent", "vx_workspace_size", "vx_planned_splits", "vx_status_string",
           "vx_last_error", "vx_version"]


class VxError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class vx_geometry(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim_qk", ctypes.c_int32), ("head_dim_v", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("mla_shared_kv", ctypes.c_int32), ("num_pool_pages", ctypes.c_int64)]


class vx_page_table(ctypes.Structure):
    _fields_ = [("page_ptr", ctypes.c_void_p), ("page_indices", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("max_pages", ctypes.c_int32)]


_lib = None


def lib():
    """The loaded libvx.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libvx.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        p, i32, i64, u64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                     ctypes.c_float, ctypes.c_size_t)
        G, T = ctypes.POINTER(vx_geometry), ctypes.POINTER(vx_page_table)
        L.vx_centroid_update.argtypes = [G, T, p, p, p, p, p, p, p, p]
        L.vx_score_pages.argtypes = [G, T, p, p, i32, p, p, p]
        L.vx_topk_pages.argtypes = [G, T, p, i32, i32, u64, p, p, p]
        L.vx_sparse_decode.argtypes = [G, T, p, p, p, p, i32, f32, i32, p, p, p, sz, p, p]
        L.vx_sparse_decode_noalloc.argtypes = [G, T, p, p, p, p, i32, f32, i32, p, p, p, p]
        L.vx_block_topk_decode_persistent.argtypes = [G, T, p, p, p, p, i32, f32, p, p, p, p, p, sz, p, p]
        L.vx_block_topk_decode.argtypes = [G, T, p, p, p, p, i32, i32, u64, f32, i32, i32, p, p, p, p, p, sz,
                                           p, p]
        L.vx_block_topk_decode_append.argtypes = [G, T, p, p, p, p, p, p, i32, i32, u64, f32, i32, i32, p, p, p, p,
                                                  p, sz, p, p]
        L.vx_workspace_size.argtypes = [G, i32, i32, i32]
        L.vx_workspace_size.restype = sz
        L.vx_planned_splits.argtypes = [G, i32, i32]
        L.vx_planned_splits.restype = i32
        L.vx_status_string.argtypes = [i32]
        L.vx_status_string.restype = ctypes.c_char_p
        L.vx_last_error.restype = ctypes.c_char_p
        L.vx_version.restype = ctypes.c_char_p
        for name in ("vx_centroid_update", "vx_score_pages", "vx_topk_pages", "vx_sparse_decode",
                     "vx_sparse_decode_noalloc", "vx_block_topk_decode", "vx_block_topk_decode_append",
                     "vx_block_topk_decode_persistent"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


@dataclass
class Geometry:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim_qk: int
    head_dim_v: int
    page_size: int
    mla_shared_kv: bool
    num_pool_pages: int

    def c(self) -> vx_geometry:
        return vx_geometry(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim_qk, self.head_dim_v,
                           self.page_size, int(self.mla_shared_kv), self.num_pool_pages)

    @staticmethod
    def of(k_cache: torch.Tensor, num_q_heads: int, batch: int, mla_shared_kv: bool = False,
           head_dim_v: Optional[int] = None) -> "Geometry":
        """Geometry of a cache [Npool][Hkv][P][Dqk]."""
        npool, hkv, P, dqk = k_cache.shape
        dv = head_dim_v if head_dim_v is not None else (512 if mla_shared_kv else dqk)
        return Geometry(batch, num_q_heads, hkv, dqk, dv, P, mla_shared_kv, npool)


@dataclass
class PageTable:
    page_ptr: torch.Tensor      # int32 [B] (device)
    page_indices: torch.Tensor  # int32 (device)
    seq_lens: torch.Tensor      # int32 [B] (device)
    max_pages: int

    def c(self) -> vx_page_table:
        for t in (self.page_ptr, self.page_indices, self.seq_lens):
            _check(t, torch.int32)
        return vx_page_table(self.page_ptr.data_ptr(), self.page_indices.data_ptr(), self.seq_lens.data_ptr(),
                             self.max_pages)


def _check(t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError("tensors passed to libvx must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return None
    _check(t, dtype)
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ok(status: int):
    if status != VX_OK:
        L = lib()
        raise VxError(status, f"{L.vx_status_string(status).decode()}: {L.vx_last_error().decode()}")


def vx_workspace_size(geo: Geometry, max_pages: int, k: int, num_splits: int = 0) -> int:
    n = lib().vx_workspace_size(ctypes.byref(geo.c()), max_pages, k, num_splits)
    if n == 0:
        raise VxError(VX_ERR_INVALID_ARG, lib().vx_last_error().decode())
    return n


def vx_planned_splits(geo: Geometry, max_pages: int, k: int) -> int:
    return int(lib().vx_planned_splits(ctypes.byref(geo.c()), max_pages, k))


def vx_centroid_update(geo: Geometry, table: PageTable, k_cache, centroids, v_cache=None, k_new=None, v_new=None,
                       first_pos=None, err=None, stream=None):
    """Rebuild (k_new None), append one token per request (k_new [B][Hkv][Dqk]) or write a
    prefill chunk (k_new [N][Hkv][Dqk] packed in request order, with first_pos)."""
    _ok(lib().vx_centroid_update(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(k_cache, torch.bfloat16),
                                 _ptr(v_cache, torch.bfloat16), _ptr(centroids, torch.bfloat16),
                                 _ptr(k_new, torch.bfloat16), _ptr(v_new, torch.bfloat16),
                                 _ptr(first_pos, torch.int32), _ptr(err, torch.int32), _stream(stream)))


def vx_score_pages(geo: Geometry, table: PageTable, q, centroids, scores, score_dims=0, err=None, stream=None):
    _ok(lib().vx_score_pages(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(q, torch.bfloat16),
                             _ptr(centroids, torch.bfloat16), score_dims, _ptr(scores, torch.float32),
                             _ptr(err, torch.int32), _stream(stream)))


def vx_topk_pages(geo: Geometry, table: PageTable, scores, k: int, sel, mode=0, seed=0, err=None, stream=None):
    _ok(lib().vx_topk_pages(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(scores, torch.float32), k, mode,
                            seed & (2 ** 64 - 1), _ptr(sel, torch.int32), _ptr(err, torch.int32), _stream(stream)))


def vx_sparse_decode(geo: Geometry, table: PageTable, q, k_cache, v_cache, sel, k: int, out, ws, lse=None,
                     sm_scale=0.0, num_splits=0, err=None, stream=None):
    _ok(lib().vx_sparse_decode(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(q, torch.bfloat16),
                               _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16), _ptr(sel, torch.int32),
                               k, float(sm_scale), num_splits, _ptr(out, torch.bfloat16), _ptr(lse, torch.float32),
                               _ptr(ws), ws.numel() * ws.element_size(), _ptr(err, torch.int32), _stream(stream)))


def vx_sparse_decode_noalloc(geo: Geometry, table: PageTable, q, k_cache, v_cache, sel, k: int, out, lse=None,
                             sm_scale=0.0, num_splits=0, err=None, stream=None):
    """vx_sparse_decode for callers that cannot allocate device memory: the split partials
    live in a fixed scratch array inside the library (see include/vx.h)."""
    _ok(lib().vx_sparse_decode_noalloc(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(q, torch.bfloat16),
                                       _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                                       _ptr(sel, torch.int32), k, float(sm_scale), num_splits,
                                       _ptr(out, torch.bfloat16), _ptr(lse, torch.float32), _ptr(err, torch.int32),
                                       _stream(stream)))


def vx_block_topk_decode(geo: Geometry, table: PageTable, q, k_cache, v_cache, centroids, k: int, out, ws,
                         lse=None, mode=0, seed=0, sm_scale=0.0, score_dims=0, num_splits=0, scores_out=None,
                         sel_out=None, err=None, stream=None):
    _ok(lib().vx_block_topk_decode(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(q, torch.bfloat16),
                                   _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                                   _ptr(centroids, torch.bfloat16), k, mode, seed & (2 ** 64 - 1), float(sm_scale),
                                   score_dims, num_splits, _ptr(out, torch.bfloat16), _ptr(lse, torch.float32),
                                   _ptr(scores_out, torch.float32), _ptr(sel_out, torch.int32), _ptr(ws),
                                   ws.numel() * ws.element_size(), _ptr(err, torch.int32), _stream(stream)))


def vx_block_topk_decode_append(geo: Geometry, table: PageTable, q, k_cache, v_cache, centroids, k_new, v_new,
                                k: int, out, ws, lse=None, mode=0, seed=0, sm_scale=0.0, score_dims=0, num_splits=0,
                                scores_out=None, sel_out=None, err=None, stream=None):
    """One appending decode step: write each request's new token (k_new [B][Hkv][Dqk], v_new
    [B][Hkv][Dv]) into its page and update the page centroid, then score, select and attend."""
    _ok(lib().vx_block_topk_decode_append(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(q, torch.bfloat16),
                                          _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                                          _ptr(centroids, torch.bfloat16), _ptr(k_new, torch.bfloat16),
                                          _ptr(v_new, torch.bfloat16), k, mode, seed & (2 ** 64 - 1),
                                          float(sm_scale), score_dims, num_splits, _ptr(out, torch.bfloat16),
                                          _ptr(lse, torch.float32), _ptr(scores_out, torch.float32),
                                          _ptr(sel_out, torch.int32), _ptr(ws), ws.numel() * ws.element_size(),
                                          _ptr(err, torch.int32), _stream(stream)))


def vx_block_topk_decode_persistent(geo: Geometry, table: PageTable, q, k_cache, v_cache, centroids, k: int, out,
                                    ws, lse=None, sm_scale=0.0, scores_out=None, sel_out=None, err=None,
                                    stream=None):
    """The decode step as one persistent kernel (see include/vx.h).  `ws` (uint8,
    vx_workspace_size bytes) must be zero-filled once before its first use here (torch.zeros);
    every call leaves its counters zero again."""
    _ok(lib().vx_block_topk_decode_persistent(ctypes.byref(geo.c()), ctypes.byref(table.c()), _ptr(q, torch.bfloat16),
                                              _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                                              _ptr(centroids, torch.bfloat16), k, float(sm_scale),
                                              _ptr(out, torch.bfloat16), _ptr(lse, torch.float32),
                                              _ptr(scores_out, torch.float32), _ptr(sel_out, torch.int32), _ptr(ws),
                                              ws.numel() * ws.element_size(), _ptr(err, torch.int32), _stream(stream)))

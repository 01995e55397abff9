"""Shared helpers for the GPU parity tests: run each step through the C ABI on a
workload, and compare with the fp64 oracle on the same seeded inputs.

Tolerances (floating point), each derived in the design notes:
  * centroids: bit-exact (fp64 sums of bf16 are exact; one round-to-nearest-even);
  * scores: |gpu - oracle| <= 1e-5 * max|oracle| per row when the oracle scores the
    same stored centroids (fp32 accumulation error only);
  * exact / approximate top-k: bit-exact sets when the oracle selects on the GPU's own
    fp32 scores;
  * attention outputs (bf16): max |err| <= 2e-2 and relative L2 <= 5e-3 over all outputs;
    lse: |err| <= 1e-3.
"""
import math

import numpy as np
import torch

import oracle
from paged_block_sparse_kv_b200 import synth, vx

ATT_MAX_ABS = 2e-2
ATT_REL_L2 = 5e-3
LSE_ABS = 1e-3
SCORE_REL = 1e-5


def geometry(w):
    s = w.spec
    return vx.Geometry(w.batch, s.num_q_heads, s.num_kv_heads, s.head_dim_qk, s.head_dim_v, s.page_size,
                       s.mla_shared_kv, w.num_pool_pages)


def table(w, seq_lens=None):
    return vx.PageTable(w.page_ptr, w.page_indices, w.seq_lens if seq_lens is None else seq_lens, w.max_pages)


def err_word(device="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=device)


def gpu_centroids(w, err=None):
    cen = torch.zeros((w.num_pool_pages, w.spec.num_kv_heads, w.spec.head_dim_qk), dtype=torch.bfloat16,
                      device=w.k_cache.device)
    vx.vx_centroid_update(geometry(w), table(w), w.k_cache, cen, v_cache=w.v_cache, err=err)
    return cen


def gpu_scores(w, cen, score_dims=0, err=None):
    s = torch.full((w.batch, w.spec.num_kv_heads, w.max_pages), float("nan"), dtype=torch.float32,
                   device=w.k_cache.device)
    vx.vx_score_pages(geometry(w), table(w), w.q, cen, s, score_dims=score_dims, err=err)
    return s


def gpu_topk(w, scores, k=None, mode=0, seed=0, err=None):
    k = w.spec.k if k is None else k
    sel = torch.full((w.batch, w.spec.num_kv_heads, k), -7, dtype=torch.int32, device=w.k_cache.device)
    vx.vx_topk_pages(geometry(w), table(w), scores, k, sel, mode=mode, seed=seed, err=err)
    return sel


def workspace(w, k=None, num_splits=0):
    k = w.spec.k if k is None else k
    n = vx.vx_workspace_size(geometry(w), w.max_pages, k, num_splits)
    return torch.zeros(n, dtype=torch.uint8, device=w.k_cache.device)  # the persistent step wants it zero-filled


def gpu_decode(w, sel, k=None, num_splits=0, sm_scale=0.0, err=None):
    k = w.spec.k if k is None else k
    out = torch.full((w.batch, w.spec.num_q_heads, w.spec.head_dim_v), float("nan"), dtype=torch.bfloat16,
                     device=w.k_cache.device)
    lse = torch.full((w.batch, w.spec.num_q_heads), float("nan"), dtype=torch.float32, device=w.k_cache.device)
    ws = workspace(w, k, num_splits)
    vx.vx_sparse_decode(geometry(w), table(w), w.q, w.k_cache, w.v_cache, sel, k, out, ws, lse=lse,
                        sm_scale=sm_scale, num_splits=num_splits, err=err)
    return out, lse


def gpu_fused(w, cen, k=None, mode=0, seed=0, num_splits=0, err=None, keep=True, ws=None):
    k = w.spec.k if k is None else k
    dev = w.k_cache.device
    out = torch.empty((w.batch, w.spec.num_q_heads, w.spec.head_dim_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.spec.num_q_heads), dtype=torch.float32, device=dev)
    scores = torch.full((w.batch, w.spec.num_kv_heads, w.max_pages), float("nan"), device=dev) if keep else None
    sel = torch.empty((w.batch, w.spec.num_kv_heads, k), dtype=torch.int32, device=dev) if keep else None
    ws = workspace(w, k, num_splits) if ws is None else ws
    vx.vx_block_topk_decode(geometry(w), table(w), w.q, w.k_cache, w.v_cache, cen, k, out, ws, lse=lse, mode=mode,
                            seed=seed, num_splits=num_splits, scores_out=scores, sel_out=sel, err=err)
    return out, lse, scores, sel


def gpu_persistent(w, cen, k=None, err=None, ws=None):
    """vx_block_topk_decode_persistent; `ws` must have been zero-filled once (workspace() does)."""
    k = w.spec.k if k is None else k
    dev = w.k_cache.device
    out = torch.empty((w.batch, w.spec.num_q_heads, w.spec.head_dim_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.spec.num_q_heads), dtype=torch.float32, device=dev)
    scores = torch.full((w.batch, w.spec.num_kv_heads, w.max_pages), float("nan"), device=dev)
    sel = torch.empty((w.batch, w.spec.num_kv_heads, k), dtype=torch.int32, device=dev)
    ws = workspace(w, k) if ws is None else ws
    vx.vx_block_topk_decode_persistent(geometry(w), table(w), w.q, w.k_cache, w.v_cache, cen, k, out, ws, lse=lse,
                                       scores_out=scores, sel_out=sel, err=err)
    return out, lse, scores, sel


# ------------------------------------------------------------------ oracle side

def host(w):
    return dict(k=synth.bits(w.k_cache), v=None if w.v_cache is None else synth.bits(w.v_cache),
                q=synth.bits(w.q), ptr=w.page_ptr.cpu().numpy(), idx=w.page_indices.cpu().numpy(),
                L=w.seq_lens.cpu().numpy())


def used_pages(h, P):
    n = (h["L"] + P - 1) // P
    return np.unique(np.concatenate([h["idx"][h["ptr"][b]:h["ptr"][b] + n[b]] for b in range(len(n))]))


def valid_scores_mask(L, P, max_pages, hkv):
    n = (np.asarray(L) + P - 1) // P
    m = np.arange(max_pages)[None, None, :] < n[:, None, None]
    return np.broadcast_to(m, (len(n), hkv, max_pages))


def check_scores(gpu, orc, L, P):
    g = gpu.cpu().numpy().astype(np.float64)
    mask = valid_scores_mask(L, P, g.shape[2], g.shape[1])
    assert np.all(np.isfinite(g[mask]))
    rowmax = np.max(np.where(mask, np.abs(orc), 0), axis=2, keepdims=True)
    err = np.where(mask, np.abs(g - orc), 0)
    worst = float(np.max(err / np.maximum(rowmax, 1e-30)))
    assert worst <= SCORE_REL, f"score error {worst:.3e} of the row max"
    return worst


def check_attention(out_gpu, lse_gpu, out_orc, lse_orc):
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - out_orc)
    max_abs = float(err.max())
    rel_l2 = float(np.linalg.norm(o - out_orc) / max(np.linalg.norm(out_orc), 1e-30))
    assert max_abs <= ATT_MAX_ABS, f"max abs error {max_abs:.3e}"
    assert rel_l2 <= ATT_REL_L2, f"relative L2 error {rel_l2:.3e}"
    if lse_gpu is not None:
        l = lse_gpu.cpu().numpy().astype(np.float64)
        fin = np.isfinite(lse_orc)
        assert np.array_equal(np.isfinite(l), fin)
        lerr = float(np.max(np.abs(l[fin] - lse_orc[fin]))) if fin.any() else 0.0
        assert lerr <= LSE_ABS, f"lse error {lerr:.3e}"
    return max_abs, rel_l2


def recall(sel_a, sel_b):
    """mean over rows of |A & B| / |B| (B = exact)."""
    a, b = sel_a.reshape(-1, sel_a.shape[-1]), sel_b.reshape(-1, sel_b.shape[-1])
    vals = []
    for x, y in zip(a, b):
        ys = set(int(v) for v in y if v >= 0)
        if ys:
            vals.append(len(ys & set(int(v) for v in x if v >= 0)) / len(ys))
    return float(np.mean(vals))


def check_attention_pair(out, lse, out_ref, lse_ref):
    """Two GPU results of the same attention, compared with the parity tolerance."""
    return check_attention(out, lse, out_ref.float().cpu().numpy().astype(np.float64),
                           lse_ref.cpu().numpy().astype(np.float64))

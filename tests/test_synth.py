"""The seeded input generator follows the recipe the design notes state: lengths in the stated range,
a pool of ceil(1.125 * pages held) pages (plus the pages appends take later) under a seeded
permutation, no page held by two requests, keys = N(0, 1) + a per-(page, KV head) offset of
standard deviation 0.5, values N(0, 1), queries N(0, 1) + 0.5 x the summed offsets of the request's
planted pages, NaN in every slot no request holds.  CPU, small batches."""
import math

import numpy as np
import pytest
import torch

from paged_block_sparse_kv_b200 import synth


def _np(x):
    return x.float().numpy() if x.dtype == torch.bfloat16 else x.numpy()


@pytest.mark.parametrize("name,batch", [("qwen3_1p7b_gqa_b32", 4), ("long_ctx_128k_b8", 1),
                                        ("mla_576_512_b16", 3), ("cont_batch_b256", 6)])
def test_recipe(name, batch):
    spec = synth.SPECS[name]
    w = synth.make(spec, 5, "cpu", batch=batch)
    P = spec.page_size
    L = w.seq_lens.numpy().astype(np.int64)
    lo, hi = (spec.ctx[1], spec.ctx[1]) if spec.ctx[0] == "fixed" else (spec.ctx[1], spec.ctx[2])
    assert L.min() >= lo and L.max() <= hi
    n0 = -(-L // P)
    n_final = -(-(L + spec.steps) // P)
    assert w.num_pool_pages == math.ceil(1.125 * n0.sum()) + int((n_final - n0).sum())
    ptr, idx = w.page_ptr.numpy(), w.page_indices.numpy()
    held = np.concatenate([idx[ptr[b]:ptr[b] + n0[b]] for b in range(batch)])
    assert len(set(held.tolist())) == len(held) and held.min() >= 0 and held.max() < w.num_pool_pages
    k = _np(w.k_cache)
    # poison: pages nobody holds and the slots past each request's length
    free = np.setdiff1d(np.arange(w.num_pool_pages), held)
    assert np.isnan(k[free]).all()
    for b in range(batch):
        last = idx[ptr[b] + n0[b] - 1]
        assert np.isnan(k[last, :, L[b] - (n0[b] - 1) * P:]).all()
        assert not np.isnan(k[last, :, :L[b] - (n0[b] - 1) * P]).any()
    # keys: N(0, 1) around a per-(page, head) offset of std 0.5
    full = [idx[ptr[b] + j] for b in range(batch) for j in range(n0[b] - 1)]  # whole pages only
    kv = k[full].astype(np.float64)                              # [pages][Hkv][P][D]
    page_mean = kv.mean(axis=2)                                  # ~ offset (+ noise / sqrt(P))
    within = (kv - page_mean[:, :, None, :]).std()  # the page's own mean takes 1/P of the variance
    assert abs(within - math.sqrt(1.0 - 1.0 / P)) < 0.01
    off_var = page_mean.var() - 1.0 / P                          # var(offset) + var(noise mean)
    assert abs(off_var - 0.25) < 0.03
    if not spec.mla_shared_kv:
        v = _np(w.v_cache)[full].astype(np.float64)
        assert abs(v.mean()) < 0.02 and abs(v.std() - 1.0) < 0.02
    # planted pages: n_planted distinct logical pages per request, within its length
    for b in range(batch):
        assert len(w.planted[b]) == min(spec.n_planted, n0[b]) and len(set(w.planted[b])) == len(w.planted[b])
        assert all(0 <= j < n0[b] for j in w.planted[b])


def test_query_carries_the_planted_offsets():
    spec = synth.custom_spec(batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=64, page_size=16,
                             ctx=("list", [4000, 3000]), k=8, n_planted=6)
    w = synth.make(spec, 9, "cpu")
    P = spec.page_size
    q = _np(w.q).astype(np.float64)                              # [B][Hq][D]
    k = _np(w.k_cache).astype(np.float64)
    ptr, idx = w.page_ptr.numpy(), w.page_indices.numpy()
    G = spec.num_q_heads // spec.num_kv_heads
    # estimate each boost from the planted pages' key means (offset + N(0, 1/P) noise) and
    # regress the queries on it: slope var(boost) / (var(boost) + var(noise)) = 0.375 / 0.469
    # for 6 pages of 16 tokens; a query without the boost (or with another page's) gives ~0
    xs, ys = [], []
    for b in range(2):
        pages = idx[ptr[b] + np.array(w.planted[b])]
        est = 0.5 * k[pages].mean(axis=2).sum(axis=0)            # [Hkv][D]
        for g in range(spec.num_q_heads):
            xs.append(est[g // G])
            ys.append(q[b, g])
    x, y = np.concatenate(xs), np.concatenate(ys)
    slope = float((x * y).sum() / (x * x).sum())
    expect = 0.375 / (0.375 + 0.25 * 6 / P)                      # 0.80: boost variance over boost + noise
    assert abs(slope - expect) < 0.2                             # 512 samples; without the boost: ~0
    assert abs((y - slope * x).std() - 1.0) < 0.15              # the rest is the N(0, 1) part

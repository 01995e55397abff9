"""The roofline bytes bench.py divides by, against a token-by-token count on CPU: every page's
centroid row, the K (and V) row of every valid token of every selected page per KV head, and
q / out once per query head."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_block_sparse_kv_b200 import synth  # noqa: E402


def _count(spec, L, sel):
    P = spec.page_size
    cen = kv = 0
    per_tok = spec.head_dim_qk * 2 if spec.mla_shared_kv else (spec.head_dim_qk + spec.head_dim_v) * 2
    for b in range(len(L)):
        n = -(-int(L[b]) // P)
        cen += n * spec.num_kv_heads * spec.head_dim_qk * 2
        for h in range(spec.num_kv_heads):
            for j in sel[b, h]:
                if j < 0:
                    continue
                kv += sum(1 for t in range(j * P, (j + 1) * P) if t < L[b]) * per_tok
    qo = len(L) * spec.num_q_heads * (spec.head_dim_qk + spec.head_dim_v) * 2
    return cen + kv + qo, kv + qo, cen


@pytest.mark.parametrize("mla", [False, True])
def test_step_bytes_match_a_token_count(mla):
    if mla:
        spec = synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
                                 page_size=64, mla_shared_kv=True, ctx=("list", [700, 64, 1]), k=5)
    else:
        spec = synth.custom_spec(batch=4, num_q_heads=8, num_kv_heads=2, head_dim_qk=64, page_size=16,
                                 ctx=("list", [1, 17, 300, 33]), k=6)
    w = synth.make(spec, 3, "cpu")
    L = w.seq_lens.numpy()
    rng = np.random.default_rng(4)
    n = -(-L // spec.page_size)
    sel = np.full((spec.batch, spec.num_kv_heads, spec.k), -1, np.int32)
    for b in range(spec.batch):
        for h in range(spec.num_kv_heads):
            pick = np.sort(rng.permutation(int(n[b]))[:min(spec.k, int(n[b]))])
            sel[b, h, :len(pick)] = pick
    got = bench.step_bytes(w, torch.from_numpy(sel), w.seq_lens, spec.k)
    assert tuple(got) == _count(spec, L, sel)

"""vx_sparse_decode_noalloc, the sparse-decode call for callers that cannot allocate
device memory (an engine that gives all free HBM to its KV pool at start-up, a plugin
interface with no workspace argument, code that must not risk cudaMalloc's device
synchronisation).  Through the C ABI its output must match vx_sparse_decode's, which uses
a caller workspace, within the tolerance of the other parity tests, on two calls in a
row (the second call reuses the scratch the first one left behind).  Collected last on
purpose; it also passes on its own in a fresh process."""
import pytest
import torch

from gpu_cases import check_attention_pair, geometry, gpu_centroids, gpu_decode, gpu_scores, gpu_topk, table
from paged_block_sparse_kv_b200 import synth, vx

pytestmark = pytest.mark.gpu


def _noalloc(w, sel, num_splits=0):
    out = torch.full((w.batch, w.spec.num_q_heads, w.spec.head_dim_v), float("nan"), dtype=torch.bfloat16,
                     device=w.k_cache.device)
    lse = torch.full((w.batch, w.spec.num_q_heads), float("nan"), dtype=torch.float32, device=w.k_cache.device)
    vx.vx_sparse_decode_noalloc(geometry(w), table(w), w.q, w.k_cache, w.v_cache, sel, w.spec.k, out, lse=lse,
                                num_splits=num_splits)
    return out, lse


def test_noalloc_matches_workspace_call_two_calls_in_a_row():
    specs = [
        synth.custom_spec(batch=4, num_q_heads=16, num_kv_heads=8, head_dim_qk=128, page_size=16,
                          ctx=("uniform", 2000, 9000), k=64),
        synth.custom_spec(batch=3, num_q_heads=8, num_kv_heads=2, head_dim_qk=128, page_size=32,
                          ctx=("list", [517, 3000, 64]), k=12),
    ]
    for i, spec in enumerate(specs):  # two calls in a row, different problems
        w = synth.make(spec, 900 + i, "cuda")
        sel = gpu_topk(w, gpu_scores(w, gpu_centroids(w)))
        out_ref, lse_ref = gpu_decode(w, sel)
        out, lse = _noalloc(w, sel)
        torch.cuda.synchronize()
        check_attention_pair(out, lse, out_ref, lse_ref)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 64 requests x 16 query heads on one KV head, 4096 splits: (64 + 4096) partial slots of
    # 16 heads x (128 + 2) floats ~ 34.6 MB, more than the fixed scratch holds
    spec = synth.custom_spec(batch=64, num_q_heads=16, num_kv_heads=1, head_dim_qk=128, page_size=16,
                             ctx=("fixed", 1100), k=64)
    w = synth.make(spec, 7, "cuda")
    sel = torch.zeros((w.batch, spec.num_kv_heads, spec.k), dtype=torch.int32, device="cuda")
    with pytest.raises(vx.VxError) as e:
        _noalloc(w, sel, num_splits=4096)
    assert e.value.status == vx.VX_ERR_WORKSPACE
    assert "vx_sparse_decode_noalloc" in str(e.value)

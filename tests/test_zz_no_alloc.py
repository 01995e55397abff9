"""vx_sparse_decode_noalloc, the sparse-decode call for callers that cannot allocate device
memory (an engine that gives all free HBM to its KV pool at start-up, a plugin interface
with no workspace argument, code that must not risk cudaMalloc's device synchronisation).

Through the C ABI, on two calls in a row (the second call reuses the scratch the first one
left behind), its output must be bit-identical to vx_sparse_decode's with a caller workspace
and the same split count (same kernels, same split plan), and both must match the fp64
oracle within the attention tolerance of the other parity tests.  Collected last on purpose;
it also passes on its own in a fresh process."""
import pytest
import torch

import oracle
from gpu_cases import check_attention, geometry, gpu_centroids, gpu_decode, gpu_scores, gpu_topk, host, table
from paged_block_sparse_kv_b200 import synth, vx

pytestmark = pytest.mark.gpu


def _noalloc(w, sel, num_splits=0):
    out = torch.full((w.batch, w.spec.num_q_heads, w.spec.head_dim_v), float("nan"), dtype=torch.bfloat16,
                     device=w.k_cache.device)
    lse = torch.full((w.batch, w.spec.num_q_heads), float("nan"), dtype=torch.float32, device=w.k_cache.device)
    vx.vx_sparse_decode_noalloc(geometry(w), table(w), w.q, w.k_cache, w.v_cache, sel, w.spec.k, out, lse=lse,
                                num_splits=num_splits)
    return out, lse


def _same_bits(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("num_splits", [0, 7])
def test_noalloc_matches_workspace_call_two_calls_in_a_row(num_splits):
    specs = [
        synth.custom_spec(batch=4, num_q_heads=16, num_kv_heads=8, head_dim_qk=128, page_size=16,
                          ctx=("uniform", 2000, 9000), k=64),
        synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512, page_size=64,
                          mla_shared_kv=True, ctx=("list", [700, 2000, 64]), k=6),
        synth.custom_spec(batch=3, num_q_heads=8, num_kv_heads=2, head_dim_qk=128, page_size=32,
                          ctx=("list", [517, 3000, 64]), k=12),
    ]
    for i, spec in enumerate(specs):  # calls in a row, different problems, one shared scratch
        w = synth.make(spec, 900 + i, "cuda")
        sel = gpu_topk(w, gpu_scores(w, gpu_centroids(w)))
        out_ref, lse_ref = gpu_decode(w, sel, num_splits=num_splits)
        out, lse = _noalloc(w, sel, num_splits=num_splits)
        out2, lse2 = _noalloc(w, sel, num_splits=num_splits)  # again, on what the first call left
        torch.cuda.synchronize()
        for o, l in ((out, lse), (out2, lse2)):
            assert _same_bits(o, out_ref) and _same_bits(l, lse_ref), f"problem {i}: differs from vx_sparse_decode"
        h = host(w)
        o_orc, l_orc = oracle.attend(h["q"], h["k"], h["v"], h["ptr"], h["idx"], h["L"], sel=sel.cpu().numpy(),
                                     mla_shared_kv=spec.mla_shared_kv, head_dim_v=spec.head_dim_v)
        check_attention(out, lse, o_orc, l_orc)


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


def test_noalloc_limit_follows_the_stated_formula():
    # the largest split count whose partials fit: accepted; one more: rejected (GQA, G = 16, Dv = 128)
    spec = synth.custom_spec(batch=64, num_q_heads=16, num_kv_heads=1, head_dim_qk=128, page_size=16,
                             ctx=("fixed", 1100), k=64)
    w = synth.make(spec, 7, "cuda")
    sel = gpu_topk(w, gpu_scores(w, gpu_centroids(w)))
    rows, G, dv = 64, 16, 128

    def need(W):
        s = rows + W
        return ((s * G * dv * 4 + 255) // 256) * 256 + s * G * 2 * 4

    W = max(x for x in range(1, 4096) if need(x) <= vx.NOALLOC_SCRATCH_BYTES)
    assert W < rows * spec.k * (spec.page_size // 16)  # not clamped by the tile count
    out, lse = _noalloc(w, sel, num_splits=W)
    out_ref, lse_ref = gpu_decode(w, sel, num_splits=W)
    torch.cuda.synchronize()
    assert _same_bits(out, out_ref) and _same_bits(lse, lse_ref)
    with pytest.raises(vx.VxError) as e:
        _noalloc(w, sel, num_splits=W + 1)
    assert e.value.status == vx.VX_ERR_WORKSPACE

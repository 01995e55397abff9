"""Prefill write (vx_centroid_update with k_new and first_pos): the new tokens' slots and the
touched pages' centroids, bit for bit against the oracle's prefill write and page means."""
import numpy as np
import pytest
import torch

import oracle
from gpu_cases import err_word, geometry, gpu_centroids, host, table, used_pages
from paged_block_sparse_kv_b200 import synth, vx

pytestmark = pytest.mark.gpu

CASES = {
    # GQA, page 16, head_dim 128: first positions at 0, mid-page, on a page boundary, L - 1, L
    "gqa_d128_p16": (synth.custom_spec(batch=6, num_q_heads=16, num_kv_heads=8, head_dim_qk=128, page_size=16,
                                       ctx=("list", [1, 37, 640, 300, 33, 1000]), k=8), 31,
                     lambda L: np.array([0, 5, 320, 299, 33, 17], np.int32)),
    # GQA, page 64, head_dim 64, group 4
    "gqa_d64_p64": (synth.custom_spec(batch=4, num_q_heads=16, num_kv_heads=4, head_dim_qk=64, page_size=64,
                                      ctx=("list", [200, 64, 129, 4000]), k=8), 32,
                    lambda L: np.array([130, 0, 128, 1000], np.int32)),
    # MLA: one latent+rope pool, no V
    "mla_p64": (synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
                                  page_size=64, mla_shared_kv=True, ctx=("list", [700, 64, 2000]), k=6), 33,
                lambda L: np.array([650, 0, 1], np.int32)),
}


def _prefill(w, fp_np, seed):
    spec = w.spec
    L = w.seq_lens.cpu().numpy()
    n_new = int(sum(int(L[b]) - int(fp_np[b]) for b in range(len(L)) if 0 <= fp_np[b] <= L[b]))
    g = torch.Generator().manual_seed(seed)
    k_new = torch.randn((max(n_new, 1), spec.num_kv_heads, spec.head_dim_qk), generator=g).to(torch.bfloat16)
    v_new = None if spec.mla_shared_kv else torch.randn((max(n_new, 1), spec.num_kv_heads, spec.head_dim_v),
                                                        generator=g).to(torch.bfloat16)
    return n_new, k_new, v_new


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_write_matches_oracle(name):
    spec, seed, fp_of = CASES[name]
    w = synth.make(spec, seed, "cuda")
    h = host(w)
    P = spec.page_size
    fp = fp_of(h["L"])
    n_new, k_new, v_new = _prefill(w, fp, seed)
    err = err_word()
    cen = gpu_centroids(w, err)
    kc = w.k_cache.clone()
    vc = None if spec.mla_shared_kv else w.v_cache.clone()
    fp_d = torch.from_numpy(fp).cuda()
    vx.vx_centroid_update(geometry(w), table(w), kc, cen, v_cache=vc, k_new=k_new.cuda(),
                          v_new=None if v_new is None else v_new.cuda(), first_pos=fp_d, err=err)
    k_o, v_o = oracle.prefill_write(h["k"], h["v"], h["ptr"], h["idx"], h["L"], fp, synth.bits(k_new),
                                    None if v_new is None else synth.bits(v_new), max_len=w.max_pages * P,
                                    mla_shared_kv=spec.mla_shared_kv)
    assert np.array_equal(synth.bits(kc), k_o)  # every slot, the untouched NaN ones included
    if vc is not None:
        assert np.array_equal(synth.bits(vc), v_o)
    _, c16 = oracle.centroids(k_o, h["ptr"], h["idx"], h["L"])
    used = used_pages(h, P)
    assert np.array_equal(synth.bits(cen)[used], c16[used])
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_prefill_bad_first_position_is_reported_and_skipped():
    spec, seed, _ = CASES["gqa_d128_p16"]
    w = synth.make(spec, seed, "cuda")
    h = host(w)
    fp = np.array([0, 5, 700, 299, 33, 17], np.int32)  # request 2: first_pos > seq_len (640)
    n_new, k_new, v_new = _prefill(w, fp, 7)
    err = err_word()
    cen = gpu_centroids(w, err)
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    vx.vx_centroid_update(geometry(w), table(w), kc, cen, v_cache=vc, k_new=k_new.cuda(), v_new=v_new.cuda(),
                          first_pos=torch.from_numpy(fp).cuda(), err=err)
    k_o, v_o = oracle.prefill_write(h["k"], h["v"], h["ptr"], h["idx"], h["L"], fp, synth.bits(k_new),
                                    synth.bits(v_new), max_len=w.max_pages * spec.page_size)
    assert np.array_equal(synth.bits(kc), k_o) and np.array_equal(synth.bits(vc), v_o)
    torch.cuda.synchronize()
    assert int(err.item()) == vx.VX_DATA_BAD_SEQ_LEN


def test_prefill_one_token_per_request_equals_append():
    spec, seed, _ = CASES["gqa_d64_p64"]
    w = synth.make(spec, seed, "cuda")
    L = w.seq_lens
    g = torch.Generator().manual_seed(11)
    k_new = torch.randn((w.batch, spec.num_kv_heads, spec.head_dim_qk), generator=g).to(torch.bfloat16).cuda()
    v_new = torch.randn((w.batch, spec.num_kv_heads, spec.head_dim_v), generator=g).to(torch.bfloat16).cuda()
    outs = []
    for fp in (None, (L - 1).to(torch.int32).contiguous()):
        err = err_word()
        cen = gpu_centroids(w, err)
        kc, vc = w.k_cache.clone(), w.v_cache.clone()
        vx.vx_centroid_update(geometry(w), table(w), kc, cen, v_cache=vc, k_new=k_new, v_new=v_new, first_pos=fp,
                              err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        outs.append((synth.bits(kc), synth.bits(vc), synth.bits(cen)))
    for x, y in zip(*outs):
        assert np.array_equal(x, y)

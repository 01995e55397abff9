"""GPU parity: every step of the hot path through the C ABI against the fp64 oracle on
the same seeded inputs, at sizes the oracle finishes in seconds that still span several
tiles, splits and a ragged tail, plus the method's edge cases."""
import numpy as np
import pytest
import torch

import oracle
from gpu_cases import (check_attention, check_attention_pair, check_scores, err_word, geometry, gpu_centroids,
                       gpu_decode, gpu_fused, gpu_persistent, gpu_scores, gpu_topk, host, recall, table, used_pages, workspace)
from paged_block_sparse_kv_b200 import synth, vx

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_config": (synth.SPECS["tiny_gqa4_d64"], 0),
    "edges_1tok_fullpage_ragged": (synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=8, head_dim_qk=128,
                                                     page_size=16, ctx=("list", [1, 16, 1000]), k=8), 11),
    "g4_page32": (synth.custom_spec(batch=2, num_q_heads=8, num_kv_heads=2, head_dim_qk=128, page_size=32,
                                    ctx=("list", [517, 64]), k=5), 12),
    "g16_d64_page64": (synth.custom_spec(batch=2, num_q_heads=16, num_kv_heads=1, head_dim_qk=64, page_size=64,
                                         ctx=("list", [300, 4097]), k=12), 13),
    "g1_many_rows": (synth.custom_spec(batch=4, num_q_heads=8, num_kv_heads=8, head_dim_qk=128, page_size=16,
                                       ctx=("uniform", 1, 3000), k=16), 14),
    "k_exceeds_pages": (synth.custom_spec(batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=128, page_size=16,
                                          ctx=("list", [40, 90]), k=20), 15),
    "qwen_shape_small_batch": (synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=8, head_dim_qk=128,
                                                 page_size=16, ctx=("uniform", 4096, 9000), k=128, n_planted=8), 16),
    # 81920 tiles, about 69 per warp on 148 SMs: enough that the planned split hands a quarter
    # of them out late, in pieces, from a counter; short contexts leave -1 selection slots
    "late_pieces_b64": (synth.custom_spec(batch=64, num_q_heads=16, num_kv_heads=8, head_dim_qk=128, page_size=16,
                                          ctx=("uniform", 1500, 5000), k=160), 20),
    # few rows of 1025..6144 pages: the 512-thread top-k blocks
    "topk_rows_512": (synth.custom_spec(batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=64, page_size=16,
                                        ctx=("list", [20000, 70000]), k=100), 21),
    "mla_16heads": (synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
                                      page_size=64, mla_shared_kv=True, ctx=("list", [700, 2000, 64]), k=6), 17),
    "mla_5heads_ragged": (synth.custom_spec(batch=2, num_q_heads=5, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
                                            page_size=64, mla_shared_kv=True, ctx=("list", [1, 4000]), k=9), 18),
    "mla_page32": (synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
                                     page_size=32, mla_shared_kv=True, ctx=("list", [33, 900, 32]), k=7), 19),
}


def attend_kw(w):
    return dict(mla_shared_kv=w.spec.mla_shared_kv, head_dim_v=w.spec.head_dim_v)

_cache = {}


def workload(name):
    if name not in _cache:
        spec, seed = CASES[name]
        _cache[name] = synth.make(spec, seed, "cuda")
    return _cache[name]


@pytest.mark.parametrize("name", list(CASES))
def test_step_by_step_parity(name):
    w = workload(name)
    h = host(w)
    P = w.spec.page_size
    err = err_word()
    # a1: centroids, bit-exact with the oracle's correctly rounded mean
    cen = gpu_centroids(w, err)
    _, c16 = oracle.centroids(h["k"], h["ptr"], h["idx"], h["L"])
    used = used_pages(h, P)
    gc = synth.bits(cen)
    assert np.array_equal(gc[used], c16[used]), "centroid mismatch"
    # a2: scores, oracle scoring the same stored centroids
    s = gpu_scores(w, cen, err=err)
    s_orc = oracle.scores(h["q"], h["ptr"], h["idx"], h["L"], P, w.max_pages, w.spec.num_kv_heads,
                          centroids_bf16=gc)
    check_scores(s, s_orc, h["L"], P)
    # a3: exact top-k, bit-exact with the oracle's stable sort on the GPU's own scores
    sel = gpu_topk(w, s, err=err)
    s_gpu = s.cpu().numpy().astype(np.float64)
    sel_orc = oracle.topk_exact(s_gpu, h["L"], P, w.spec.k)
    assert np.array_equal(sel.cpu().numpy(), sel_orc)
    # a4: attention over the GPU's selection
    out, lse = gpu_decode(w, sel, err=err)
    o_orc, l_orc = oracle.attend(h["q"], h["k"], h["v"], h["ptr"], h["idx"], h["L"], sel=sel_orc, **attend_kw(w))
    check_attention(out, lse, o_orc, l_orc)
    # fused entry = the three calls (same split plan -> identical bits)
    out_f, lse_f, s_f, sel_f = gpu_fused(w, cen, err=err)
    assert torch.equal(s_f, s) or np.array_equal(s_f.cpu().numpy(), s.cpu().numpy(), equal_nan=True)
    assert torch.equal(sel_f, sel)
    assert torch.equal(out_f, out) and torch.equal(lse_f, lse)
    if not w.spec.mla_shared_kv:
        # persistent fused step: the same scores and selection bits; its own attention split,
        # so its outputs agree within the attention tolerance
        out_p, lse_p, s_p, sel_p = gpu_persistent(w, cen, err=err)
        assert np.array_equal(s_p.cpu().numpy(), s.cpu().numpy(), equal_nan=True)
        assert torch.equal(sel_p, sel)
        check_attention(out_p, lse_p, o_orc, l_orc)
        check_attention_pair(out_p, lse_p, out, lse)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


@pytest.mark.parametrize("name", ["edges_1tok_fullpage_ragged", "g4_page32", "g16_d64_page64", "tiny_config",
                                  "mla_16heads"])
def test_all_pages_equals_dense_attention(name):
    w = workload(name)
    h = host(w)
    P = w.spec.page_size
    n = (h["L"] + P - 1) // P
    k = int(n.max())
    sel = torch.full((w.batch, w.spec.num_kv_heads, k), -1, dtype=torch.int32)
    for b in range(w.batch):
        sel[b, :, :n[b]] = torch.arange(int(n[b]), dtype=torch.int32)
    out, lse = gpu_decode(w, sel.cuda(), k=k)
    o_orc, l_orc = oracle.attend(h["q"], h["k"], h["v"], h["ptr"], h["idx"], h["L"], **attend_kw(w))  # dense
    check_attention(out, lse, o_orc, l_orc)


@pytest.mark.parametrize("name", ["g1_many_rows", "mla_16heads"])
@pytest.mark.parametrize("splits", [1, 3, 37, 0, 100000])
def test_split_count_invariance(name, splits):
    w = workload(name)
    h = host(w)
    cen = gpu_centroids(w)
    sel = gpu_topk(w, gpu_scores(w, cen))
    out, lse = gpu_decode(w, sel, num_splits=splits)
    o_orc, l_orc = oracle.attend(h["q"], h["k"], h["v"], h["ptr"], h["idx"], h["L"], sel=sel.cpu().numpy(),
                                 **attend_kw(w))
    check_attention(out, lse, o_orc, l_orc)


def test_physical_page_permutation_is_bit_identical():
    w = workload("qwen_shape_small_batch")
    perm = torch.randperm(w.num_pool_pages, generator=torch.Generator().manual_seed(5)).cuda()
    # page p moves to slot perm[p]
    k2 = torch.empty_like(w.k_cache)
    v2 = torch.empty_like(w.v_cache)
    k2[perm] = w.k_cache
    v2[perm] = w.v_cache
    idx2 = perm[w.page_indices.long()].to(torch.int32)
    w2 = synth.Workload(w.spec, w.seed, w.seq_lens, w.page_ptr, idx2, w.row_capacity, w.max_pages,
                        w.num_pool_pages, k2, v2, w.q, w.planted)
    a = gpu_fused(w, gpu_centroids(w))
    b = gpu_fused(w2, gpu_centroids(w2))
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x.view(torch.int32),
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32))


@pytest.mark.parametrize("name", ["qwen_shape_small_batch", "g1_many_rows", "g16_d64_page64", "mla_16heads",
                                  "topk_rows_512"])
def test_approx_topk_bit_exact_on_gpu_scores(name):
    w = workload(name)
    h = host(w)
    s = gpu_scores(w, gpu_centroids(w))
    s32 = s.cpu().numpy()
    for mode, bits in ((1, 12), (2, 10), (3, 8)):
        for seed in (0, 12345):
            sel = gpu_topk(w, s, mode=mode, seed=seed)
            sel_orc = oracle.topk_approx(np.nan_to_num(s32, nan=0.0), h["L"], w.spec.page_size, w.spec.k, seed,
                                         bits=bits)
            assert np.array_equal(sel.cpu().numpy(), sel_orc)
    exact = oracle.topk_exact(s32.astype(np.float64), h["L"], w.spec.page_size, w.spec.k)
    assert recall(sel.cpu().numpy(), exact) > 0.5


@pytest.mark.parametrize("name", ["qwen_shape_small_batch", "mla_16heads", "g16_d64_page64", "edges_1tok_fullpage_ragged",
                                  "late_pieces_b64"])
def test_fused_step_modes_match_separate_calls(name):
    """The fused step in every top-k mode gives the separate calls' scores and selection bit for
    bit (the chained kernels run with programmatic dependent launch)."""
    w = workload(name)
    cen = gpu_centroids(w)
    s = gpu_scores(w, cen)
    for mode in (0, 1, 2, 3):
        for seed in (0, 77):
            err = err_word()
            flags = vx.VX_TABLE_READY if seed else 0  # the flag changes when reads start, not results
            out, lse, s_f, sel_f = gpu_fused(w, cen, mode=mode | flags, seed=seed, err=err)
            assert np.array_equal(s_f.cpu().numpy(), s.cpu().numpy(), equal_nan=True)
            assert torch.equal(sel_f, gpu_topk(w, s, mode=mode, seed=seed))
            # the planned split hands its late pieces to whichever warp is free in the fused step
            # and round robin in the separate call: same pieces, same partial slots, same bits
            out_d, lse_d = gpu_decode(w, sel_f)
            assert torch.equal(out.view(torch.int16), out_d.view(torch.int16)) and torch.equal(lse, lse_d)
            torch.cuda.synchronize()
            assert int(err.item()) == 0
            if mode == 0:
                break


@pytest.mark.parametrize("flags", [0, vx.VX_TABLE_READY])
@pytest.mark.parametrize("name", ["qwen_shape_small_batch", "mla_16heads", "g1_many_rows", "late_pieces_b64"])
def test_fused_steps_on_a_stream_and_in_a_graph(name, flags):
    """Back-to-back fused steps on a created stream (where the kernels' programmatic dependent
    launches take effect) and replayed from a CUDA graph give the default-stream result bit for
    bit, with no device error (a bounded wait that ran out would set VX_DATA_TIMEOUT); with
    VX_TABLE_READY too (each step's scorer then reads the table while the previous step's
    merge runs)."""
    w = workload(name)
    cen = gpu_centroids(w)
    ref = gpu_fused(w, cen)
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    err = err_word()
    bufs = [workspace(w) for _ in range(2)]
    with torch.cuda.stream(st):
        runs = [gpu_fused(w, cen, err=err, ws=bufs[i % 2], mode=flags) for i in range(6)]
    torch.cuda.synchronize()
    outs = []
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        gpu_fused(w, cen, err=err, ws=bufs[0], mode=flags)  # warm-up before capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=st):
            for i in range(4):
                outs.append(gpu_fused(w, cen, err=err, ws=bufs[i % 2], mode=flags))
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for r in runs + outs:
        assert torch.equal(r[0].view(torch.int16), ref[0].view(torch.int16)) and torch.equal(r[1], ref[1])
        assert torch.equal(r[3], ref[3])
    del g


def test_topk_ties_and_signed_zero():
    # crafted rows: all-equal scores pick the lowest pages; -0.0 ties with +0.0
    spec = synth.custom_spec(batch=2, num_q_heads=2, num_kv_heads=2, head_dim_qk=64, page_size=16,
                             ctx=("list", [16 * 300, 16 * 40]), k=10)
    w = synth.make(spec, 3, "cuda")
    s = torch.zeros((2, 2, w.max_pages), dtype=torch.float32)
    s[0, 1, ::2] = -0.0
    s[1, 0, :] = torch.tensor(np.round(np.random.default_rng(0).standard_normal(w.max_pages)), dtype=torch.float32)
    s[1, 1, 7] = 5.0
    sel = gpu_topk(w, s.cuda())
    sel_orc = oracle.topk_exact(s.numpy().astype(np.float64), w.seq_lens.cpu().numpy(), 16, 10)
    assert np.array_equal(sel.cpu().numpy(), sel_orc)
    assert sel[0, 0].tolist() == list(range(10))


def test_append_steps_match_oracle():
    # continuous batching: append one token per request per step, recompute tail centroids
    spec = synth.custom_spec(batch=4, num_q_heads=8, num_kv_heads=4, head_dim_qk=128, page_size=16,
                             ctx=("list", [15, 16, 33, 100]), k=4, steps=18)
    w = synth.make(spec, 21, "cuda")
    geo = geometry(w)
    cen = gpu_centroids(w)
    kc, vc = synth.bits(w.k_cache), synth.bits(w.v_cache)
    ptr, idx = w.page_ptr.cpu().numpy(), w.page_indices.cpu().numpy()
    err = err_word()
    for s in range(spec.steps):
        L = w.seq_lens_at(s)
        vx.vx_centroid_update(geo, table(w, L), w.k_cache, cen, v_cache=w.v_cache, k_new=w.step_k_new[s],
                              v_new=w.step_v_new[s], err=err)
        kc, vc = oracle.append(kc, vc, ptr, idx, L.cpu().numpy(), synth.bits(w.step_k_new[s]),
                               synth.bits(w.step_v_new[s]))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    Lf = w.seq_lens_at(spec.steps - 1).cpu().numpy()
    hh = dict(L=Lf, ptr=ptr, idx=idx)
    used = used_pages(hh, 16)
    gk, gv = synth.bits(w.k_cache), synth.bits(w.v_cache)
    assert np.array_equal(gk[used].view(np.int16), kc[used].view(np.int16))
    assert np.array_equal(gv[used].view(np.int16), vc[used].view(np.int16))
    _, c16 = oracle.centroids(kc, ptr, idx, Lf)
    assert np.array_equal(synth.bits(cen)[used], c16[used])


@pytest.mark.parametrize("mla", [False, True])
def test_appending_step_equals_append_then_fused_call(mla):
    """vx_block_topk_decode_append (append chained into the step) gives the same bits as
    vx_centroid_update's append followed by vx_block_topk_decode, step after step: caches,
    centroids, scores, selection, out and lse."""
    if mla:
        spec = synth.custom_spec(batch=3, num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
                                 page_size=64, mla_shared_kv=True, ctx=("list", [63, 64, 700]), k=5, steps=4)
    else:
        spec = synth.custom_spec(batch=4, num_q_heads=8, num_kv_heads=4, head_dim_qk=128, page_size=16,
                                 ctx=("list", [15, 16, 33, 1000]), k=6, steps=4)
    runs = []
    for fused in (False, True):
        w = synth.make(spec, 41, "cuda")
        geo = geometry(w)
        cen = gpu_centroids(w)
        ws = workspace(w)
        err = err_word()
        outs = []
        for s in range(spec.steps):
            L = w.seq_lens_at(s)
            tab = table(w, L)
            out = torch.empty((w.batch, spec.num_q_heads, spec.head_dim_v), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((w.batch, spec.num_q_heads), dtype=torch.float32, device="cuda")
            sc = torch.full((w.batch, spec.num_kv_heads, w.max_pages), float("nan"), device="cuda")
            sel = torch.empty((w.batch, spec.num_kv_heads, spec.k), dtype=torch.int32, device="cuda")
            v_new = None if w.step_v_new is None else w.step_v_new[s]  # MLA: the value is the latent key
            if fused:  # odd steps with VX_TABLE_READY (same results)
                vx.vx_block_topk_decode_append(geo, tab, w.step_q[s], w.k_cache, w.v_cache, cen, w.step_k_new[s],
                                               v_new, spec.k, out, ws, lse=lse, scores_out=sc, sel_out=sel, err=err,
                                               mode=vx.VX_TABLE_READY if s % 2 else 0)
            else:
                vx.vx_centroid_update(geo, tab, w.k_cache, cen, v_cache=w.v_cache, k_new=w.step_k_new[s],
                                      v_new=v_new, err=err)
                vx.vx_block_topk_decode(geo, tab, w.step_q[s], w.k_cache, w.v_cache, cen, spec.k, out, ws, lse=lse,
                                        scores_out=sc, sel_out=sel, err=err)
            outs.append((out, lse, sc, sel))
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        runs.append((outs, w.k_cache, w.v_cache, cen))
    (o0, k0, v0, c0), (o1, k1, v1, c1) = runs
    assert torch.equal(k0.view(torch.int16), k1.view(torch.int16)) and torch.equal(c0.view(torch.int16),
                                                                                   c1.view(torch.int16))
    if v0 is not None:
        assert torch.equal(v0.view(torch.int16), v1.view(torch.int16))
    for a, b in zip(o0, o1):
        assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)) and torch.equal(a[1], b[1])
        assert np.array_equal(a[2].cpu().numpy(), b[2].cpu().numpy(), equal_nan=True) and torch.equal(a[3], b[3])


def test_bad_page_id_and_length_set_the_error_word():
    w = synth.make(synth.custom_spec(batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=128, page_size=16,
                                     ctx=("list", [100, 200]), k=4), 9, "cuda")
    cen = gpu_centroids(w)
    bad_idx = w.page_indices.clone()
    bad_idx[1] = w.num_pool_pages + 5  # out of the pool
    wb = synth.Workload(w.spec, w.seed, w.seq_lens, w.page_ptr, bad_idx, w.row_capacity, w.max_pages,
                        w.num_pool_pages, w.k_cache, w.v_cache, w.q, w.planted)
    err = err_word()
    out, lse, _, _ = gpu_fused(wb, cen, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & vx.VX_DATA_BAD_PAGE_ID
    bad_len = w.seq_lens.clone()
    bad_len[0] = w.max_pages * 16 + 1
    err2 = err_word()
    sc = torch.zeros((2, 2, w.max_pages), device="cuda")
    vx.vx_score_pages(geometry(w), table(w, bad_len), w.q, cen, sc, err=err2)
    torch.cuda.synchronize()
    assert int(err2.item()) & vx.VX_DATA_BAD_SEQ_LEN
    # the context is still usable
    out_ok, _, _, _ = gpu_fused(w, cen)
    torch.cuda.synchronize()
    assert torch.isfinite(out_ok.float()).all()


@pytest.mark.parametrize("name,dims", [("qwen_shape_small_batch", 64), ("mla_16heads", 512), ("mla_5heads_ragged", 512),
                                       ("mla_page32", 512), ("mla_16heads", 64)])
def test_rope_unaware_score_dims(name, dims):
    """Scores on the first `dims` dims only (MLA: the 512 latent dims without the 64 rope dims, the
    rope-unaware routing of the MLA experiment) against the oracle scoring the same stored
    centroids on the same dims."""
    w = workload(name)
    h = host(w)
    P = w.spec.page_size
    cen = gpu_centroids(w)
    s = gpu_scores(w, cen, score_dims=dims)
    s_orc = oracle.scores(h["q"], h["ptr"], h["idx"], h["L"], P, w.max_pages, w.spec.num_kv_heads,
                          centroids_bf16=synth.bits(cen), score_dims=dims)
    check_scores(s, s_orc, h["L"], P)
    # the cut matters: the full-dims scores differ from these on some page
    s_full = oracle.scores(h["q"], h["ptr"], h["idx"], h["L"], P, w.max_pages, w.spec.num_kv_heads,
                           centroids_bf16=synth.bits(cen))
    fin = np.isfinite(s_full)
    assert np.max(np.abs(s_full[fin] - s_orc[fin])) > 1e-3 * np.max(np.abs(s_full[fin]))


# vx_block_topk_decode_persistent's counters: a fixed region at the head of the workspace
# (4 + 1024 + 2 * 1024 * 16 uint32 words)
FUSED_SYNC_BYTES = (4 + 1024 + 2 * 1024 * 16) * 4


@pytest.mark.parametrize("name", ["qwen_shape_small_batch", "g16_d64_page64", "edges_1tok_fullpage_ragged"])
def test_persistent_step_repeatable_and_leaves_counters_zero(name):
    # every call must leave the counters zero, so back-to-back calls on one workspace give the
    # same bits (the work items are planned from the inputs alone)
    w = workload(name)
    cen = gpu_centroids(w)
    ws = workspace(w)
    err = err_word()
    runs = [gpu_persistent(w, cen, ws=ws, err=err) for _ in range(3)]
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert int(torch.count_nonzero(ws[:FUSED_SYNC_BYTES]).item()) == 0
    for r in runs[1:]:
        for x, y in zip(runs[0], r):
            if x.dtype == torch.bfloat16:
                assert torch.equal(x.view(torch.int16), y.view(torch.int16))
            else:
                assert np.array_equal(x.cpu().numpy(), y.cpu().numpy(), equal_nan=True)


def test_topk_rows_beyond_shared_memory():
    """Rows longer than the top-k kernel's shared-memory key buffer (12,288 pages) read their keys
    from global memory in every pass: exact and both approximate modes against the oracle, with
    heavy ties (scores rounded to a few values)."""
    P = 16
    L = np.array([20000 * P, 13000 * P - 5], np.int32)
    max_pages = 20000
    geo = vx.Geometry(2, 4, 2, 64, 64, P, 0, 40000)
    dev = "cuda"
    rng = np.random.default_rng(21)
    s = np.round(rng.standard_normal((2, 2, max_pages)) * 4).astype(np.float32)  # ~25 distinct values
    s[1, 1, :] = rng.standard_normal(max_pages).astype(np.float32)
    scores = torch.from_numpy(s).to(dev)
    seq = torch.from_numpy(L).to(dev)
    dummy = torch.zeros(4, dtype=torch.int32, device=dev)  # the top-k reads only lengths and scores
    tab = vx.PageTable(dummy, dummy, seq, max_pages)
    k = 700
    err = err_word()
    sel = torch.full((2, 2, k), -7, dtype=torch.int32, device=dev)
    vx.vx_topk_pages(geo, tab, scores, k, sel, mode=0, err=err)
    assert np.array_equal(sel.cpu().numpy(), oracle.topk_exact(s.astype(np.float64), L, P, k))
    for mode, bits in ((1, 12), (2, 10), (3, 8)):
        vx.vx_topk_pages(geo, tab, scores, k, sel, mode=mode, seed=99, err=err)
        assert np.array_equal(sel.cpu().numpy(), oracle.topk_approx(s, L, P, k, 99, bits=bits))
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_largest_batch_step():
    """The whole chained step at the largest batch the library accepts (4,096 requests)."""
    spec = synth.custom_spec(batch=4096, num_q_heads=4, num_kv_heads=2, head_dim_qk=64, page_size=16,
                             ctx=("uniform", 1, 120), k=4)
    w = synth.make(spec, 23, "cuda")
    h = host(w)
    err = err_word()
    cen = gpu_centroids(w, err)
    out, lse, scores, sel = gpu_fused(w, cen, err=err)
    s_gpu = scores.cpu().numpy().astype(np.float64)
    sel_orc = oracle.topk_exact(s_gpu, h["L"], spec.page_size, spec.k)
    assert np.array_equal(sel.cpu().numpy(), sel_orc)
    reqs = [0, 1, 2047, 4094, 4095]
    sub = synth.host_subset(w, reqs)
    o_orc, l_orc = oracle.attend(synth.bits(w.q[reqs]), sub["k_cache"], sub["v_cache"], sub["page_ptr"],
                                 sub["page_indices"], sub["seq_lens"], sel=sel[reqs].cpu().numpy())
    check_attention(out[reqs], lse[reqs], o_orc, l_orc)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_topk_many_short_rows_warp_path():
    """With many rows (>= 4 per SM) exact rows of at most 512 pages are selected by one warp:
    crafted rows with heavy ties, -0.0 and +0.0, lengths 1..512 pages, against the oracle."""
    P, B, hkv, max_pages, k = 16, 512, 2, 512, 40
    rng = np.random.default_rng(31)
    n = rng.integers(1, max_pages + 1, B)
    n[:4] = [1, 40, 41, 512]
    L = (n * P - rng.integers(0, P, B)).clip(1).astype(np.int32)
    s = np.round(rng.standard_normal((B, hkv, max_pages)) * 3).astype(np.float32)
    s[::7, 0, ::3] = -0.0
    s[1::5, 1, :] = rng.standard_normal((len(range(1, B, 5)), max_pages)).astype(np.float32)
    geo = vx.Geometry(B, 4, hkv, 64, 64, P, 0, 40000)
    dummy = torch.zeros(4, dtype=torch.int32, device="cuda")
    tab = vx.PageTable(dummy, dummy, torch.from_numpy(L).cuda(), max_pages)
    err = err_word()
    sel = torch.full((B, hkv, k), -7, dtype=torch.int32, device="cuda")
    vx.vx_topk_pages(geo, tab, torch.from_numpy(s).cuda(), k, sel, mode=0, err=err)
    assert np.array_equal(sel.cpu().numpy(), oracle.topk_exact(s.astype(np.float64), L, P, k))
    torch.cuda.synchronize()
    assert int(err.item()) == 0


@pytest.mark.parametrize("name", ["g1_many_rows", "mla_16heads"])
def test_empty_selection_rows(name):
    """Rows whose selection is entirely empty (all -1) attend to nothing: out = 0, lse = -inf, as
    the oracle gives; the other rows are unaffected."""
    w = workload(name)
    h = host(w)
    sel = gpu_topk(w, gpu_scores(w, gpu_centroids(w)))
    sel[0] = -1            # every KV head of request 0
    sel[1, 0] = -1         # the first KV head of request 1
    err = err_word()
    out, lse = gpu_decode(w, sel, err=err)
    o_orc, l_orc = oracle.attend(h["q"], h["k"], h["v"], h["ptr"], h["idx"], h["L"], sel=sel.cpu().numpy(),
                                 **attend_kw(w))
    G = w.spec.num_q_heads // w.spec.num_kv_heads
    assert torch.equal(out[0], torch.zeros_like(out[0])) and torch.isneginf(lse[0]).all()
    assert torch.equal(out[1, :G], torch.zeros_like(out[1, :G])) and torch.isneginf(lse[1, :G]).all()
    check_attention(out, lse, o_orc, l_orc)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_late_pieces_case_has_late_pieces():
    """The planned split of late_pieces_b64 has late pieces on this GPU (more chunks than warps),
    so the parity cases that use it cover them."""
    w = workload("late_pieces_b64")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles = w.batch * w.spec.num_kv_heads * w.spec.k  # page 16: one tile per selected page
    if tiles // (sms * 8) < 64:
        pytest.skip(f"{sms} SMs: a warp's share of this case is below the 64 tiles that late pieces need")
    assert vx.vx_planned_splits(geometry(w), w.max_pages, w.spec.k) > sms * 8

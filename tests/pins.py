"""Pins of the fp64 oracle to things other than itself.

Each pin is a plain function that raises AssertionError when the oracle disagrees with a
closed form, a brute-force enumeration, a library routine that reduces to the textbook
definition, a published test vector or a hand-worked fixture under tests/golden/.  The
pins are chosen so that a plausible mistake anywhere in the oracle (a dropped term, a
wrong index, a wrong tie rule, a wrong rounding) fails at least one of them;
test_oracle_mutants.py plants such mistakes in copies of the oracle and checks it.

Sources (Vortex paper note): section 系统设计 1 (block top-k: centroid cache, indexer,
top-k, exact attention), 系统设计 2 (vTensor page table), 系统设计 3 (radix top-k with
stochastic early termination and remapping), the MLA experiment section (rope-aware
scoring over latent + rope dims).
"""
import itertools
import math
import os

import numpy as np
import torch

import oracle
from paged_block_sparse_kv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ------------------------------------------------------------------ helpers

def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.strip()
    return out


def _rows(text):
    return [[float(x) for x in r.split()] for r in text.split(";")]


def _bf16_bits(x):
    """float array -> bf16 bits via torch's float32 -> bf16 round-to-nearest-even."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _small(seed=0, **kw):
    spec = synth.custom_spec(**kw)
    return synth.make(spec, seed, "cpu")


def _np(w):
    return dict(k=synth.bits(w.k_cache), v=None if w.v_cache is None else synth.bits(w.v_cache),
                q=synth.bits(w.q), ptr=w.page_ptr.numpy(), idx=w.page_indices.numpy(),
                L=w.seq_lens.numpy())


def _one_page_table(P, L):
    return np.array([0], np.int32), np.array([0], np.int32), np.array([L], np.int32)


# ------------------------------------------------------------------ bf16 conversion

def pin_bf16_narrow_matches_library_rounding():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-38, 38, 4000),
                        rng.standard_normal(200) * 1e-39,  # bf16 subnormals
                        [0.0, -0.0, 1.0, -1.0, 3.0e38]]).astype(np.float32)
    got = oracle.narrow_bf16(x.astype(np.float64))
    want = _bf16_bits(x)
    assert np.array_equal(got, want), "fp32-representable values must round like torch fp32->bf16"


def pin_bf16_narrow_ties_and_double_rounding():
    cases = {1.0 + 2.0 ** -8: 0x3F80,                 # tie -> even (1.0)
             1.0 + 3 * 2.0 ** -8: 0x3F82,             # tie -> even (1 + 2^-6)
             1.0 + 2.0 ** -8 + 2.0 ** -40: 0x3F81,    # just above the tie: up, no float detour
             -(1.0 + 2.0 ** -8): 0xBF80,
             2.0 ** -133: 0x0001,                     # smallest bf16 subnormal
             2.0 ** -134: 0x0000,                     # tie between 0 and 2^-133 -> even (0)
             3.0 * 2.0 ** -134: 0x0002}               # tie -> even (2 * 2^-133)
    got = oracle.narrow_bf16(np.array(list(cases.keys())))
    assert [int(g) for g in got] == list(cases.values()), [hex(int(g)) for g in got]


def pin_bf16_widen_roundtrip():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = allbits[((allbits >> 7) & 0xFF) != 0xFF]
    w = oracle.widen_bf16(finite)
    want = torch.tensor(finite.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(w, want)
    assert np.array_equal(oracle.narrow_bf16(w), finite)


# ------------------------------------------------------------------ centroids

def pin_centroid_golden_partial_page():
    g = _golden("centroid_partial_page.txt")
    P, L = int(g["page_size"]), int(g["seq_len"])
    keys = np.array(_rows(g["keys"]), np.float32)  # [P][D]
    k = _bf16_bits(keys).reshape(1, 1, P, -1)
    ptr, idx, lens = _one_page_table(P, L)
    c64, c16 = oracle.centroids(k, ptr, idx, lens)
    want = np.array([float(x) for x in g["centroid"].split()])
    assert np.array_equal(c64[0, 0], want), c64[0, 0]
    assert np.array_equal(c16[0, 0], _bf16_bits(want))


def pin_centroid_arithmetic_progression():
    # keys a + t * delta: the mean over m tokens is a + (m - 1) / 2 * delta (closed form);
    # integers and small dyadic steps keep every value exact in bf16 and double.
    P, D, Hkv = 16, 8, 2
    a = np.array([[-3, 1, 0, 2, 5, -1, 7, 4], [2, -2, 6, 0, 1, 3, -5, 9]], np.float64)
    delta = np.array([[0.5, -0.25, 1, 2, -1, 0.125, 0, 0.75], [1, 1, -0.5, 0.25, 2, -2, 0.5, 3]])
    for m in (1, 5, 16):
        keys = np.full((1, Hkv, P, D), np.nan)
        for t in range(m):
            keys[0, :, t, :] = a + t * delta
        k = _bf16_bits(keys)
        ptr, idx, lens = _one_page_table(P, m)
        c64, _ = oracle.centroids(k, ptr, idx, lens)
        assert np.array_equal(c64[0], a + (m - 1) / 2 * delta), m


def pin_centroid_sum_invariant():
    # sum_j m_j * centroid_j equals the plain sum of every valid key (numpy gather + sum)
    w = _small(seed=3, batch=3, num_q_heads=4, num_kv_heads=2, head_dim_qk=32, page_size=16,
               ctx=("list", [1, 37, 64]))
    a = _np(w)
    c64, _ = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    kf = oracle.widen_bf16(a["k"])
    P = w.spec.page_size
    for b in range(3):
        L = int(a["L"][b])
        n = (L + P - 1) // P
        phys = a["idx"][a["ptr"][b]:a["ptr"][b] + n]
        lhs = sum(min(P, L - j * P) * c64[phys[j]] for j in range(n))
        toks = np.concatenate([kf[phys[j], :, :min(P, L - j * P), :] for j in range(n)], axis=1)
        rhs = toks.sum(axis=1)
        assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def pin_centroid_stored_is_rounded_mean():
    w = _small(seed=4, batch=2, num_kv_heads=2, num_q_heads=2, head_dim_qk=64, ctx=("list", [50, 16]))
    a = _np(w)
    c64, c16 = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    used = np.unique(np.concatenate([a["idx"][a["ptr"][b]:a["ptr"][b] + (a["L"][b] + 15) // 16]
                                     for b in range(2)]))
    assert np.array_equal(c16[used], oracle.narrow_bf16(c64[used]))
    err = np.abs(oracle.widen_bf16(c16[used]) - c64[used])
    assert np.all(err <= 2.0 ** -8 * np.abs(c64[used]) + 1e-300)


# ------------------------------------------------------------------ scores

def pin_scores_equal_mean_of_token_logits():
    # q . mean_t(K_t) summed over the group == mean_t of the group-summed logits, computed
    # with numpy matmuls over the gathered valid tokens (linearity of the mean).
    w = _small(seed=5, batch=2, num_q_heads=6, num_kv_heads=2, head_dim_qk=48, page_size=16,
               ctx=("list", [70, 33]))
    a = _np(w)
    c64, _ = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    maxp = 5
    s = oracle.scores(a["q"], a["ptr"], a["idx"], a["L"], 16, maxp, 2, centroids_f64=c64)
    qf, kf = oracle.widen_bf16(a["q"]), oracle.widen_bf16(a["k"])
    G = 3
    for b in range(2):
        L = int(a["L"][b])
        for h in range(2):
            for j in range((L + 15) // 16):
                phys = a["idx"][a["ptr"][b] + j]
                m = min(16, L - j * 16)
                logits = qf[b, h * G:(h + 1) * G] @ kf[phys, h, :m, :].T  # [G][m]
                want = logits.sum(0).mean()
                assert abs(s[b, h, j] - want) <= 1e-12 * (1 + abs(want)), (b, h, j)


def pin_scores_one_hot_query():
    # a query that is the unit vector e_d in every head of the group scores G * c[d]
    w = _small(seed=6, batch=1, num_q_heads=8, num_kv_heads=2, head_dim_qk=32, ctx=("list", [40]))
    a = _np(w)
    c64, c16 = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    for d in (0, 7, 31):
        q = np.zeros((1, 8, 32), np.float32)
        q[:, :, d] = 1.0
        s = oracle.scores(_bf16_bits(q), a["ptr"], a["idx"], a["L"], 16, 3, 2, centroids_f64=c64)
        for h in range(2):
            for j in range(3):
                phys = a["idx"][a["ptr"][0] + j]
                assert s[0, h, j] == 4 * c64[phys, h, d]
        s16 = oracle.scores(_bf16_bits(q), a["ptr"], a["idx"], a["L"], 16, 3, 2, centroids_bf16=c16)
        for h in range(2):
            for j in range(3):
                phys = a["idx"][a["ptr"][0] + j]
                assert s16[0, h, j] == 4 * oracle.widen_bf16(c16[phys, h, d:d + 1])[0]


def pin_scores_rope_unaware_dims():
    # score_dims = 512 on a 576-dim key equals the full score with the query's last 64
    # dims zeroed (the MLA rope-unaware variant scores on the latent part only)
    w = _small(seed=7, batch=1, num_q_heads=4, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
               page_size=64, mla_shared_kv=True, ctx=("list", [200]))
    a = _np(w)
    c64, _ = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    s512 = oracle.scores(a["q"], a["ptr"], a["idx"], a["L"], 64, 4, 1, centroids_f64=c64, score_dims=512)
    qz = a["q"].copy()
    qz[:, :, 512:] = 0
    sfull = oracle.scores(qz, a["ptr"], a["idx"], a["L"], 64, 4, 1, centroids_f64=c64)
    assert np.allclose(s512, sfull, rtol=1e-13, atol=1e-12, equal_nan=True)


# ------------------------------------------------------------------ exact top-k

def _valid_topk_set(s, k):
    """The unique set S of min(k, n) pages with: i in S, j not in S => s_i > s_j or
    (s_i == s_j and i < j); found by enumerating every subset."""
    n = len(s)
    keff = min(k, n)
    found = []
    for S in itertools.combinations(range(n), keff):
        Sset = set(S)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j) for i in S for j in range(n) if j not in Sset)
        if ok:
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def pin_topk_brute_force_with_ties():
    rng = np.random.default_rng(8)
    vals = np.array([-1.0, -0.0, 0.0, 1.0, 2.0])
    for n in range(1, 10):
        for _ in range(6):
            s = rng.choice(vals, n)
            for k in (1, 2, max(1, n // 2), n, n + 2):
                row = np.full((1, 1, 12), np.nan)
                row[0, 0, :n] = s
                sel = oracle.topk_exact(row, np.array([n * 4], np.int32), 4, k)[0, 0]
                got = [int(x) for x in sel if x >= 0]
                assert got == _valid_topk_set(list(s), k), (s, k, got)
                assert all(x == -1 for x in sel[min(k, n):])


def pin_topk_golden_ties():
    g = _golden("topk_ties.txt")
    s = np.array([float(x) for x in g["scores"].split()])
    n = len(s)
    for key, val in g.items():
        if not key.startswith("k"):
            continue
        k = int(key[1:])
        row = np.full((1, 1, n), np.nan)
        row[0, 0] = s
        sel = oracle.topk_exact(row, np.array([n], np.int32), 1, k)[0, 0]
        assert [int(x) for x in sel if x >= 0] == [int(x) for x in val.split()], (k, sel)


def pin_topk_matches_lexsort():
    rng = np.random.default_rng(9)
    B, H, maxp, P = 3, 2, 400, 16
    lens = np.array([400 * 16, 17, 123 * 16 - 5], np.int32)
    s = np.round(rng.standard_normal((B, H, maxp)) * 4) / 4  # many ties
    for k in (1, 7, 64, 500):
        sel = oracle.topk_exact(s, lens, P, k)
        for b in range(B):
            n = (int(lens[b]) + P - 1) // P
            for h in range(H):
                order = np.lexsort((np.arange(n), -s[b, h, :n]))[:min(k, n)]
                assert np.array_equal(sel[b, h, :min(k, n)], np.sort(order))


# ------------------------------------------------------------------ approximate top-k

def pin_splitmix64_published_vector():
    # first outputs of SplitMix64 seeded with 0 (published reference sequence)
    assert [oracle.splitmix64(0, i) for i in range(3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def pin_approx_golden_remap():
    for name in ("approx_topk_remap.txt", "approx_topk_remap_scale.txt"):
        g = _golden(name)
        s = np.array([float(x) for x in g["scores"].split()], np.float32)
        n = len(s)
        rows = np.stack([s, s])[None]  # B=1, Hkv=2 -> rows 0 and 1
        sel = oracle.topk_approx(rows, np.array([n], np.int32), 1, int(g["k"]), int(g["seed"]),
                                 bits=int(g["bits"]))
        assert [int(x) for x in sel[0, 0]] == [int(x) for x in g["row0"].split()], name
        assert [int(x) for x in sel[0, 1]] == [int(x) for x in g["row1"].split()], name


def pin_approx_equals_exact_when_buckets_are_singletons():
    # evenly spaced scores with at most one score per code: no boundary bucket to fill,
    # so the one-pass selection is the exact top-k
    for n in (5, 100, 1000):
        s = (np.arange(n, dtype=np.float32) * 3.0 - 7.0)[np.random.default_rng(n).permutation(n)]
        row = s[None, None, :]
        for k in (1, 3, n // 2, n):
            a = oracle.topk_approx(row, np.array([n], np.int32), 1, k, 123)
            e = oracle.topk_exact(row.astype(np.float64), np.array([n], np.int32), 1, k)
            assert np.array_equal(a, e), (n, k)


def pin_approx_one_bucket_guarantee():
    # every chosen score is at least the best unchosen score minus one bucket width
    rng = np.random.default_rng(10)
    B, H, maxp, P, bits = 2, 3, 3000, 16, 12
    lens = np.array([3000 * 16, 700 * 16 - 3], np.int32)
    s = (rng.standard_normal((B, H, maxp)) * 30).astype(np.float32)
    s[0, 0, :50] = 5.0  # a big tie
    for k in (1, 40, 256):
        sel = oracle.topk_approx(s, lens, P, k, 77, bits=bits)
        for b in range(B):
            n = (int(lens[b]) + P - 1) // P
            for h in range(H):
                row = s[b, h, :n].astype(np.float64)
                chosen = [int(x) for x in sel[b, h] if x >= 0]
                assert len(chosen) == min(k, n) == len(set(chosen))
                assert all(0 <= x < n for x in chosen)
                rest = np.setdiff1d(np.arange(n), chosen)
                width = (row.max() - row.min()) / 2 ** bits
                if len(rest):
                    assert row[chosen].min() >= row[rest].max() - width * (1 + 1e-5)


def pin_approx_fill_is_seeded_and_varies():
    # a boundary bucket larger than the slots left: different seeds pick different
    # members, every member can be picked, and one seed always picks the same set
    s = np.zeros((1, 1, 64), np.float32)
    s[0, 0, 60:] = 10.0
    lens = np.array([64], np.int32)
    seen = set()
    picked = set()
    for seed in range(200):
        a = oracle.topk_approx(s, lens, 1, 10, seed)
        b = oracle.topk_approx(s, lens, 1, 10, seed)
        assert np.array_equal(a, b)
        chosen = [int(x) for x in a[0, 0]]
        assert {60, 61, 62, 63} <= set(chosen)
        seen.add(tuple(chosen))
        picked |= set(chosen) - {60, 61, 62, 63}
    assert len(seen) > 20 and picked == set(range(60))


# ------------------------------------------------------------------ attention

def pin_attention_golden_two_tokens():
    g = _golden("attention_two_tokens.txt")
    q = _bf16_bits(np.array([[[float(x) for x in g["q"].split()]]], np.float32))
    keys = _bf16_bits(np.array(_rows(g["keys"]), np.float32)).reshape(1, 1, 2, 2)
    vals = _bf16_bits(np.array(_rows(g["values"]), np.float32)).reshape(1, 1, 2, 2)
    ptr, idx, lens = _one_page_table(2, 2)
    out, lse = oracle.attend(q, keys, vals, ptr, idx, lens, sm_scale=1.0)
    assert np.allclose(out[0, 0], [float(x) for x in g["out"].split()], rtol=1e-14, atol=0)
    assert abs(lse[0, 0] - float(g["lse"])) < 1e-14


def pin_attention_dense_matches_sdpa():
    # dense decode attention equals torch's scaled_dot_product_attention in float64 on the
    # gathered valid tokens (the textbook softmax(q K^T * scale) V)
    w = _small(seed=11, batch=3, num_q_heads=8, num_kv_heads=2, head_dim_qk=64, page_size=16,
               ctx=("list", [1, 45, 160]))
    a = _np(w)
    scale = 0.37
    out, lse = oracle.attend(a["q"], a["k"], a["v"], a["ptr"], a["idx"], a["L"], sm_scale=scale)
    qf, kf, vf = (torch.tensor(oracle.widen_bf16(x)) for x in (a["q"], a["k"], a["v"]))
    for b in range(3):
        L = int(a["L"][b])
        n = (L + 15) // 16
        phys = torch.tensor(a["idx"][a["ptr"][b]:a["ptr"][b] + n].astype(np.int64))
        K = kf[phys].permute(1, 0, 2, 3).reshape(2, n * 16, 64)[:, :L]  # [Hkv][L][D]
        V = vf[phys].permute(1, 0, 2, 3).reshape(2, n * 16, 64)[:, :L]
        Q = qf[b].reshape(2, 4, 64)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)
        assert torch.allclose(torch.tensor(out[b]).reshape(2, 4, 64), ref, rtol=1e-12, atol=1e-12)
        ref_lse = torch.logsumexp(scale * Q @ K.transpose(1, 2), dim=-1).reshape(-1)
        assert torch.allclose(torch.tensor(lse[b]), ref_lse, rtol=1e-12, atol=1e-12)


def pin_attention_constant_keys_and_single_token():
    # equal keys -> uniform weights: out = mean of V, lse = log(T) + scale * q.k
    P, D = 16, 8
    L = 37
    n = 3
    keys = np.full((n, 1, P, D), np.nan, np.float32)
    vals = np.full((n, 1, P, D), np.nan, np.float32)
    rng = np.random.default_rng(12)
    kvec = np.round(rng.standard_normal(D) * 4) / 4
    for t in range(L):
        keys[t // P, 0, t % P] = kvec
        vals[t // P, 0, t % P] = np.round(rng.standard_normal(D) * 8) / 8
    qv = np.round(rng.standard_normal(D) * 4) / 4
    q = _bf16_bits(qv[None, None, :].astype(np.float32))
    ptr, idx, lens = np.array([0], np.int32), np.array([2, 0, 1], np.int32), np.array([L], np.int32)
    # logical page j lives at physical idx[j]; rebuild the pool in that order
    kp = np.empty_like(keys)
    vp = np.empty_like(vals)
    for j in range(n):
        kp[idx[j]] = keys[j]
        vp[idx[j]] = vals[j]
    out, lse = oracle.attend(q, _bf16_bits(kp), _bf16_bits(vp), ptr, idx, lens, sm_scale=0.5)
    tok_v = np.concatenate([vals[j, 0, :min(P, L - j * P)] for j in range(n)]).astype(np.float64)
    assert np.allclose(out[0, 0], tok_v.mean(0), rtol=1e-13, atol=1e-13)
    assert abs(lse[0, 0] - (math.log(L) + 0.5 * float(qv @ kvec))) < 1e-12
    # a single valid token: out is its value row, lse its logit
    out1, lse1 = oracle.attend(q, _bf16_bits(kp), _bf16_bits(vp), ptr, idx, np.array([1], np.int32),
                               sm_scale=0.5)
    assert np.array_equal(out1[0, 0], vals[0, 0, 0].astype(np.float64))
    assert abs(lse1[0, 0] - 0.5 * float(qv @ kvec)) < 1e-13


def pin_attention_selection_semantics():
    # sel listing every page equals the dense path; listing order does not matter;
    # -1 slots are skipped; NaN slots past the length never leak
    w = _small(seed=13, batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=32, page_size=16,
               ctx=("list", [90, 200]))
    a = _np(w)
    d_out, d_lse = oracle.attend(a["q"], a["k"], a["v"], a["ptr"], a["idx"], a["L"])
    assert np.all(np.isfinite(d_out)) and np.all(np.isfinite(d_lse))
    k = 14
    sel = np.full((2, 2, k), -1, np.int32)
    for b in range(2):
        n = (int(a["L"][b]) + 15) // 16
        for h in range(2):
            sel[b, h, :n] = np.random.default_rng(b * 2 + h).permutation(n)
    s_out, s_lse = oracle.attend(a["q"], a["k"], a["v"], a["ptr"], a["idx"], a["L"], sel=sel)
    assert np.allclose(s_out, d_out, rtol=1e-12, atol=1e-12)
    assert np.allclose(s_lse, d_lse, rtol=1e-12, atol=1e-12)
    # a strict subset: equals dense attention restricted to those pages' tokens (sdpa)
    sub = np.full((2, 2, 3), -1, np.int32)
    sub[:, :, 0], sub[:, :, 1] = 0, 4
    o2, l2 = oracle.attend(a["q"], a["k"], a["v"], a["ptr"], a["idx"], a["L"], sel=sub)
    qf, kf, vf = (torch.tensor(oracle.widen_bf16(x)) for x in (a["q"], a["k"], a["v"]))
    for b in range(2):
        L = int(a["L"][b])
        for h in range(2):
            toks = [(j, t) for j in (0, 4) if j * 16 < L for t in range(min(16, L - j * 16))]
            K = torch.stack([kf[int(a["idx"][a["ptr"][b] + j]), h, t] for j, t in toks])
            V = torch.stack([vf[int(a["idx"][a["ptr"][b] + j]), h, t] for j, t in toks])
            Q = qf[b, 2 * h:2 * h + 2]
            ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None],
                                                                   scale=1 / math.sqrt(32))[0]
            assert torch.allclose(torch.tensor(o2[b, 2 * h:2 * h + 2]), ref, rtol=1e-12, atol=1e-12)


def pin_attention_mla_shared_values():
    # with shared K/V the value is the first Dv dims of the key row: same as passing that
    # slice as an explicit value cache
    w = _small(seed=14, batch=2, num_q_heads=4, num_kv_heads=1, head_dim_qk=576, head_dim_v=512,
               page_size=64, mla_shared_kv=True, ctx=("list", [100, 64]))
    a = _np(w)
    o1, l1 = oracle.attend(a["q"], a["k"], None, a["ptr"], a["idx"], a["L"], mla_shared_kv=True,
                           head_dim_v=512)
    v = np.ascontiguousarray(a["k"][..., :512])
    o2, l2 = oracle.attend(a["q"], a["k"], v, a["ptr"], a["idx"], a["L"])
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ------------------------------------------------------------------ page table

def pin_physical_relabel_invariance():
    # moving pages to other physical slots (and the page table with them) changes no
    # score, selection or output: the page table is the only link (vTensor paged layout)
    w = _small(seed=15, batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=32, page_size=16,
               ctx=("list", [100, 61]))
    a = _np(w)
    npool = a["k"].shape[0]
    perm = np.random.default_rng(0).permutation(npool)  # new id of old page p = perm[p]
    k2 = np.empty_like(a["k"]); v2 = np.empty_like(a["v"])
    k2[perm] = a["k"]; v2[perm] = a["v"]
    idx2 = perm[a["idx"]].astype(np.int32)
    c64, c16 = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    c64b, c16b = oracle.centroids(k2, a["ptr"], idx2, a["L"])
    used = a["idx"][:int(sum((a["L"] + 15) // 16))]
    assert np.array_equal(c16b[perm[used]], c16[used])
    r1 = oracle.decode_step(a["q"], a["k"], a["v"], c16, a["ptr"], a["idx"], a["L"], 7, 3)
    r2 = oracle.decode_step(a["q"], k2, v2, c16b, a["ptr"], idx2, a["L"], 7, 3)
    for x, y in zip(r1, r2):
        assert np.array_equal(x, y, equal_nan=True)


def pin_append_running_mean():
    # appending token x to a page with m-1 valid tokens: new_mean * m = old_mean*(m-1) + x
    w = _small(seed=16, batch=3, num_q_heads=4, num_kv_heads=2, head_dim_qk=32, page_size=16,
               ctx=("list", [5, 16, 47]))
    a = _np(w)
    rng = np.random.default_rng(16)
    newL = a["L"] + 1
    # request 1 needs a fresh page: take an unreferenced pool page
    idx = a["idx"].copy()
    ptr = np.array([0, 1, 3], np.int32)
    idx = np.array([a["idx"][0], a["idx"][1], -1, a["idx"][2], a["idx"][3], a["idx"][4]], np.int32)
    used = set(int(x) for x in idx if x >= 0)
    free = [p for p in range(a["k"].shape[0]) if p not in used]
    idx[2] = free[0]
    k_new = _bf16_bits(rng.standard_normal((3, 2, 32)).astype(np.float32))
    v_new = _bf16_bits(rng.standard_normal((3, 2, 32)).astype(np.float32))
    k2, v2 = oracle.append(a["k"], a["v"], ptr, idx, newL, k_new, v_new)
    changed = np.argwhere(np.any(k2.view(np.int16) != a["k"].view(np.int16), axis=-1)
                          | np.any(np.isnan(oracle.widen_bf16(a["k"])) != np.isnan(oracle.widen_bf16(k2)), axis=-1))
    expect = set()
    for b in range(3):
        pos = int(newL[b]) - 1
        phys = int(idx[ptr[b] + pos // 16])
        for h in range(2):
            expect.add((phys, h, pos % 16))
    assert set(map(tuple, changed.tolist())) <= expect
    c_old, _ = oracle.centroids(a["k"], ptr, idx, a["L"])
    c_new, _ = oracle.centroids(k2, ptr, idx, newL)
    kn = oracle.widen_bf16(k_new)
    for b in range(3):
        pos = int(newL[b]) - 1
        phys = int(idx[ptr[b] + pos // 16])
        m = pos % 16 + 1
        old = c_old[phys] if m > 1 else 0.0
        assert np.allclose(c_new[phys] * m, old * (m - 1) + kn[b], rtol=1e-12, atol=1e-12)
        assert np.array_equal(k2[phys, :, pos % 16], k_new[b]) and np.array_equal(v2[phys, :, pos % 16], v_new[b])


def pin_prefill_write_golden_by_hand():
    # 2 requests, page size 4, one KV head, 2 dims.  Request 0: pages [3, 1], 6 tokens, of which
    # positions 2..5 are new; request 1: page [0], 3 tokens, all new.  New rows, packed in request
    # order, hold (r + 1, -(r + 1)) for packed row r.  Old slots of the pool hold 100 + page*10 + slot.
    P, npool = 4, 5
    k = np.zeros((npool, 1, P, 2), np.float32)
    for pg in range(npool):
        for sl in range(P):
            k[pg, 0, sl] = (100 + pg * 10 + sl, 100 + pg * 10 + sl)
    v = -k
    ptr = np.array([0, 2], np.int32)
    idx = np.array([3, 1, 0], np.int32)
    L = np.array([6, 3], np.int32)
    fp = np.array([2, 0], np.int32)
    rows = np.array([[[r + 1.0, -(r + 1.0)]] for r in range(7)], np.float32)  # [7][1][2]
    k2, v2 = oracle.prefill_write(_bf16_bits(k), _bf16_bits(v), ptr, idx, L, fp, _bf16_bits(rows),
                                  _bf16_bits(-rows), max_len=8)
    K = oracle.widen_bf16(k2)[:, 0]
    # expected, written out by hand from the page table
    assert K[3, 0].tolist() == [130.0, 130.0] and K[3, 1].tolist() == [131.0, 131.0]  # old tokens kept
    assert K[3, 2].tolist() == [1.0, -1.0] and K[3, 3].tolist() == [2.0, -2.0]        # positions 2, 3
    assert K[1, 0].tolist() == [3.0, -3.0] and K[1, 1].tolist() == [4.0, -4.0]        # positions 4, 5
    assert K[1, 2].tolist() == [112.0, 112.0] and K[1, 3].tolist() == [113.0, 113.0]  # untouched
    assert K[0, 0].tolist() == [5.0, -5.0] and K[0, 1].tolist() == [6.0, -6.0] and K[0, 2].tolist() == [7.0, -7.0]
    assert K[0, 3].tolist() == [103.0, 103.0] and K[2].tolist() == [[120.0 + i] * 2 for i in range(4)]
    assert np.array_equal(oracle.widen_bf16(v2), -oracle.widen_bf16(k2))
    c64, _ = oracle.centroids(k2, ptr, idx, L)
    assert c64[3, 0].tolist() == [(130 + 131 + 1 + 2) / 4, (130 + 131 - 1 - 2) / 4]
    assert c64[1, 0].tolist() == [3.5, -3.5] and c64[0, 0].tolist() == [6.0, -6.0]


def pin_prefill_write_one_token_is_append():
    # one new token per request (first_pos = seq_len - 1) is the decode append
    w = _small(seed=18, batch=3, num_q_heads=4, num_kv_heads=2, head_dim_qk=32, page_size=16,
               ctx=("list", [5, 16, 47]))
    a = _np(w)
    rng = np.random.default_rng(18)
    k_new = _bf16_bits(rng.standard_normal((3, 2, 32)).astype(np.float32))
    v_new = _bf16_bits(rng.standard_normal((3, 2, 32)).astype(np.float32))
    ka, va = oracle.append(a["k"], a["v"], a["ptr"], a["idx"], a["L"], k_new, v_new)
    kp, vp = oracle.prefill_write(a["k"], a["v"], a["ptr"], a["idx"], a["L"], a["L"] - 1, k_new, v_new,
                                  max_len=16 * 3)
    assert np.array_equal(ka.view(np.int16), kp.view(np.int16)) and np.array_equal(va.view(np.int16), vp.view(np.int16))


def pin_prefill_write_chunks_compose():
    # writing [f, L) at once equals writing [f, mid) with lengths mid, then [mid, L)
    w = _small(seed=19, batch=3, num_q_heads=4, num_kv_heads=2, head_dim_qk=32, page_size=16,
               ctx=("list", [70, 33, 100]))
    a = _np(w)
    f = np.array([0, 20, 37], np.int32)
    mid = np.array([40, 33, 64], np.int32)
    n_all = int((a["L"] - f).sum())
    rng = np.random.default_rng(19)
    k_new = _bf16_bits(rng.standard_normal((n_all, 2, 32)).astype(np.float32))
    v_new = _bf16_bits(rng.standard_normal((n_all, 2, 32)).astype(np.float32))
    k1, v1 = oracle.prefill_write(a["k"], a["v"], a["ptr"], a["idx"], a["L"], f, k_new, v_new, max_len=128)
    starts = np.concatenate([[0], np.cumsum(a["L"] - f)])
    first = np.concatenate([np.arange(starts[b], starts[b] + mid[b] - f[b]) for b in range(3)])
    second = np.concatenate([np.arange(starts[b] + mid[b] - f[b], starts[b + 1]) for b in range(3)])
    k2, v2 = oracle.prefill_write(a["k"], a["v"], a["ptr"], a["idx"], mid, f, k_new[first], v_new[first],
                                  max_len=128)
    k2, v2 = oracle.prefill_write(k2, v2, a["ptr"], a["idx"], a["L"], mid, k_new[second], v_new[second],
                                  max_len=128)
    assert np.array_equal(k1.view(np.int16), k2.view(np.int16)) and np.array_equal(v1.view(np.int16), v2.view(np.int16))
    # and nothing outside the written positions changed
    kw = oracle.widen_bf16(k1)
    k0 = oracle.widen_bf16(a["k"])
    for b in range(3):
        for pos in range(int(a["L"][b])):
            phys = int(a["idx"][a["ptr"][b] + pos // 16])
            if pos < f[b]:
                assert np.array_equal(kw[phys, :, pos % 16], k0[phys, :, pos % 16])


def pin_decode_step_is_the_composition():
    w = _small(seed=17, batch=2, num_q_heads=8, num_kv_heads=2, head_dim_qk=64, page_size=16,
               ctx=("list", [300, 129]))
    a = _np(w)
    _, c16 = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    sc, sel, out, lse = oracle.decode_step(a["q"], a["k"], a["v"], c16, a["ptr"], a["idx"], a["L"], 19, 5)
    sc2 = oracle.scores(a["q"], a["ptr"], a["idx"], a["L"], 16, 19, 2, centroids_bf16=c16)
    assert np.array_equal(sc, sc2, equal_nan=True)
    sel2 = oracle.topk_exact(sc2, a["L"], 16, 5)
    assert np.array_equal(sel, sel2)
    out2, lse2 = oracle.attend(a["q"], a["k"], a["v"], a["ptr"], a["idx"], a["L"], sel=sel2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def pin_planted_pages_are_found():
    # generator sanity (not parity): the planted pages win the exact top-k
    w = synth.make(synth.SPECS["tiny_gqa4_d64"], 0, "cpu")
    a = _np(w)
    _, c16 = oracle.centroids(a["k"], a["ptr"], a["idx"], a["L"])
    _, sel, _, _ = oracle.decode_step(a["q"], a["k"], a["v"], c16, a["ptr"], a["idx"], a["L"],
                                      w.max_pages, w.spec.k)
    assert set(w.planted[0]) <= set(int(x) for x in sel[0, 0])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]

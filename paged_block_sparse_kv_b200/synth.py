"""Seeded synthetic workloads for paged block top-k sparse decode.

This module only draws inputs: it holds none of the method's arithmetic (no centroid,
score, selection or attention), so that the CUDA path and the fp64 oracle can both be
fed from it without sharing any computation.  It imports nothing else from this package.

Recipe (one per named workload, seeded):
  * context lengths: fixed, integer-uniform on [a, b] inclusive, or log-uniform
    floor(exp(U(ln a, ln b))), drawn on a CPU generator so the page table does not depend
    on the device;
  * n_b = ceil(L_b / P) pages per request; the pool holds ceil(1.125 * sum n_b) pages
    (or an explicit size) plus the pages later appends will need; physical ids come
    from a seeded permutation of the pool;
  * per physical page and KV head one offset vector ~ N(0, 0.5^2) (std 0.5);
    keys = N(0, 1) + the page's offset, values ~ N(0, 1); MLA: one latent key row per
    token whose first Dv dims are also its value;
  * per request `n_planted` distinct planted logical pages (shared by all KV heads);
    query head g (KV group h) = N(0, 1) + 0.5 * sum over planted pages of their offset
    for head h;
  * every value is rounded to bf16; pool pages no request references and slots past a
    request's length are NaN, so a wrong gather or a missing mask cannot pass parity.

Large tensors are drawn on `device` with torch's generator for that device (Philox on
CUDA), small metadata on the CPU generator.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch


@dataclass(frozen=True)
class Spec:
    """Shape of one workload family."""
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim_qk: int
    head_dim_v: int
    page_size: int
    mla_shared_kv: bool
    ctx: Tuple  # ("fixed", L) | ("uniform", a, b) | ("loguniform", a, b)
    k: int
    n_planted: int
    pool_pages: Optional[int] = None  # explicit pool size; default ceil(1.125 * used)
    steps: int = 0                    # appending decode steps (continuous batching)
    description: str = ""


# The five workloads the method is measured on, named by what they are.
SPECS = {
    "tiny_gqa4_d64": Spec(
        "tiny_gqa4_d64", 1, 4, 1, 64, 64, 16, False, ("fixed", 1024), 8, 3, pool_pages=128,
        description="1 request, 4 q heads / 1 KV head, d 64, page 16, 1024 tokens in a 128-page pool, k 8"),
    "qwen3_1p7b_gqa_b32": Spec(
        "qwen3_1p7b_gqa_b32", 32, 16, 8, 128, 128, 16, False, ("uniform", 4096, 32768), 128, 8,
        description="Qwen3-1.7B-shaped GQA decode layer: 16 q / 8 KV heads, d 128, page 16, batch 32, "
                    "context U[4096, 32768], k 128 pages"),
    "long_ctx_128k_b8": Spec(
        "long_ctx_128k_b8", 8, 32, 8, 128, 128, 16, False, ("fixed", 131072), 256, 16,
        description="long-context decode: 32 q / 8 KV heads, d 128, page 16, batch 8, 131072 tokens, k 256"),
    "mla_576_512_b16": Spec(
        "mla_576_512_b16", 16, 16, 1, 576, 512, 64, True, ("uniform", 8192, 32768), 32, 4,
        description="MLA geometry decode: 512 latent + 64 rope dims shared by 16 q heads, page 64, "
                    "batch 16, context U[8192, 32768], k 32"),
    "cont_batch_b256": Spec(
        "cont_batch_b256", 256, 32, 8, 128, 128, 16, False, ("loguniform", 1024, 65536), 64, 8,
        steps=100,
        description="continuous-batching step loop: 32 q / 8 KV heads, d 128, page 16, batch 256, "
                    "context log-U[1024, 65536], one appended token per request per step, 100 steps, "
                    "k min(64, pages)"),
}


@dataclass
class Workload:
    spec: Spec
    seed: int
    seq_lens: torch.Tensor       # int32 [B]   lengths at step 0 (before any append)
    page_ptr: torch.Tensor       # int32 [B]   row starts in page_indices
    page_indices: torch.Tensor   # int32 [cap] physical ids; rows have room for the appends
    row_capacity: torch.Tensor   # int32 [B]   entries reserved per row
    max_pages: int               # pages of the longest row over all steps
    num_pool_pages: int
    k_cache: torch.Tensor        # bf16 [Npool][Hkv][P][Dqk]
    v_cache: Optional[torch.Tensor]  # bf16 [Npool][Hkv][P][Dv]; None when V is part of K
    q: torch.Tensor              # bf16 [B][Hq][Dqk]
    planted: List[List[int]]     # planted logical pages per request
    # continuous batching: per-step inputs (empty when spec.steps == 0)
    step_q: Optional[torch.Tensor] = None      # bf16 [S][B][Hq][Dqk]
    step_k_new: Optional[torch.Tensor] = None  # bf16 [S][B][Hkv][Dqk]
    step_v_new: Optional[torch.Tensor] = None  # bf16 [S][B][Hkv][Dv]
    extra: dict = field(default_factory=dict)

    @property
    def batch(self):
        return self.spec.batch

    def seq_lens_at(self, step: int) -> torch.Tensor:
        """Lengths after `step + 1` appends (step -1 = the initial lengths)."""
        return self.seq_lens + (step + 1)

    def to(self, device) -> "Workload":
        def mv(t):
            return None if t is None else t.to(device)
        return Workload(self.spec, self.seed, mv(self.seq_lens), mv(self.page_ptr), mv(self.page_indices),
                        mv(self.row_capacity), self.max_pages, self.num_pool_pages, mv(self.k_cache),
                        mv(self.v_cache), mv(self.q), self.planted, mv(self.step_q), mv(self.step_k_new),
                        mv(self.step_v_new), dict(self.extra))


def custom_spec(name="custom", batch=2, num_q_heads=4, num_kv_heads=2, head_dim_qk=64, head_dim_v=None,
                page_size=16, mla_shared_kv=False, ctx=("uniform", 1, 200), k=4, n_planted=2,
                pool_pages=None, steps=0) -> Spec:
    """A small workload of any supported geometry (for parity and edge cases)."""
    return Spec(name, batch, num_q_heads, num_kv_heads, head_dim_qk,
                head_dim_qk if head_dim_v is None else head_dim_v, page_size, mla_shared_kv, tuple(ctx), k,
                n_planted, pool_pages, steps)


def _draw_lengths(spec: Spec, gen: torch.Generator, batch: int) -> torch.Tensor:
    kind = spec.ctx[0]
    if kind == "fixed":
        return torch.full((batch,), int(spec.ctx[1]), dtype=torch.int64)
    if kind == "uniform":
        a, b = int(spec.ctx[1]), int(spec.ctx[2])
        return torch.randint(a, b + 1, (batch,), generator=gen, dtype=torch.int64)
    if kind == "loguniform":
        a, b = int(spec.ctx[1]), int(spec.ctx[2])
        u = torch.rand(batch, generator=gen, dtype=torch.float64)
        x = torch.floor(torch.exp(math.log(a) + u * (math.log(b) - math.log(a))))
        return x.clamp(a, b).to(torch.int64)
    if kind == "list":
        return torch.tensor(list(spec.ctx[1]), dtype=torch.int64)
    raise ValueError(kind)


def make(spec: Spec, seed: int, device="cpu", batch: Optional[int] = None,
         lengths: Optional[List[int]] = None, chunk_pages: int = 8192) -> Workload:
    """Draw one workload.  `batch` overrides spec.batch; `lengths` fixes the contexts."""
    device = torch.device(device)
    B = spec.batch if batch is None else batch
    P, Hkv, Hq = spec.page_size, spec.num_kv_heads, spec.num_q_heads
    Dqk, Dv = spec.head_dim_qk, spec.head_dim_v
    meta = torch.Generator("cpu").manual_seed(seed)
    dev = torch.Generator(device).manual_seed(seed * 7919 + 17)

    L0 = torch.tensor(lengths, dtype=torch.int64) if lengths is not None else _draw_lengths(spec, meta, B)
    assert len(L0) == B and int(L0.min()) >= 0
    n0 = (L0 + P - 1) // P
    n_final = (L0 + spec.steps + P - 1) // P
    used = int(n0.sum())
    grow = int((n_final - n0).sum())
    pool = spec.pool_pages if spec.pool_pages is not None else int(math.ceil(1.125 * used)) + grow
    if pool < used + grow:
        raise ValueError("pool too small for the workload")

    perm = torch.randperm(pool, generator=meta).to(torch.int64)
    cap = n_final.clone()
    page_ptr = torch.zeros(B, dtype=torch.int64)
    if B > 1:
        page_ptr[1:] = torch.cumsum(cap, 0)[:-1]
    page_indices = torch.full((max(int(cap.sum()), 1),), -1, dtype=torch.int64)
    nxt = 0
    for b in range(B):  # pages held at step 0
        nb = int(n0[b])
        page_indices[int(page_ptr[b]):int(page_ptr[b]) + nb] = perm[nxt:nxt + nb]
        nxt += nb
    for s in range(spec.steps):  # fresh pages, in the order the appends need them
        for b in range(B):
            pos = int(L0[b]) + s  # position of the token appended at step s
            if pos % P == 0:
                page_indices[int(page_ptr[b]) + pos // P] = perm[nxt]
                nxt += 1

    planted = []
    for b in range(B):
        nb = int(n0[b])
        m = min(spec.n_planted, nb)
        planted.append(sorted(torch.randperm(nb, generator=meta)[:m].tolist()) if nb > 0 else [])

    # offsets per physical page and KV head, std 0.5
    offsets = torch.randn((pool, Hkv, Dqk), generator=dev, device=device, dtype=torch.float32) * 0.5

    k_cache = torch.empty((pool, Hkv, P, Dqk), dtype=torch.bfloat16, device=device)
    for c0 in range(0, pool, chunk_pages):
        c1 = min(pool, c0 + chunk_pages)
        x = torch.randn((c1 - c0, Hkv, P, Dqk), generator=dev, device=device, dtype=torch.float32)
        x += offsets[c0:c1, :, None, :]
        k_cache[c0:c1] = x.to(torch.bfloat16)
    v_cache = None
    if not spec.mla_shared_kv:
        v_cache = torch.empty((pool, Hkv, P, Dv), dtype=torch.bfloat16, device=device)
        for c0 in range(0, pool, chunk_pages):
            c1 = min(pool, c0 + chunk_pages)
            v_cache[c0:c1] = torch.randn((c1 - c0, Hkv, P, Dv), generator=dev, device=device,
                                         dtype=torch.float32).to(torch.bfloat16)

    # NaN poison: unreferenced pages (including pages that appends will take later) and
    # slots past each request's length.
    held = torch.zeros(pool, dtype=torch.bool)
    for b in range(B):
        nb = int(n0[b])
        held[page_indices[int(page_ptr[b]):int(page_ptr[b]) + nb]] = True
    held_d = held.to(device)
    k_cache[~held_d] = float("nan")
    if v_cache is not None:
        v_cache[~held_d] = float("nan")
    for b in range(B):
        L, nb = int(L0[b]), int(n0[b])
        if nb > 0 and L % P != 0:
            phys = int(page_indices[int(page_ptr[b]) + nb - 1])
            k_cache[phys, :, L % P:, :] = float("nan")
            if v_cache is not None:
                v_cache[phys, :, L % P:, :] = float("nan")

    def draw_query(gen_shape_batch):
        qf = torch.randn((B, Hq, Dqk), generator=dev, device=device, dtype=torch.float32)
        G = Hq // Hkv
        for b in range(B):
            if not planted[b]:
                continue
            rows = page_indices[int(page_ptr[b]) + torch.tensor(planted[b], dtype=torch.int64)]
            boost = 0.5 * offsets[rows.to(device)].sum(0)  # [Hkv][Dqk]
            qf[b] += boost.repeat_interleave(G, dim=0)
        return qf.to(torch.bfloat16)

    q = draw_query(None)

    step_q = step_k = step_v = None
    if spec.steps > 0:
        S = spec.steps
        step_q = torch.empty((S, B, Hq, Dqk), dtype=torch.bfloat16, device=device)
        step_k = torch.empty((S, B, Hkv, Dqk), dtype=torch.bfloat16, device=device)
        step_v = None if spec.mla_shared_kv else torch.empty((S, B, Hkv, Dv), dtype=torch.bfloat16,
                                                             device=device)
        for s in range(S):
            step_q[s] = draw_query(None)
            pos = L0 + s
            rows = page_indices[page_ptr + pos // P].to(device)
            kn = torch.randn((B, Hkv, Dqk), generator=dev, device=device, dtype=torch.float32)
            step_k[s] = (kn + offsets[rows]).to(torch.bfloat16)
            if step_v is not None:
                step_v[s] = torch.randn((B, Hkv, Dv), generator=dev, device=device,
                                        dtype=torch.float32).to(torch.bfloat16)

    return Workload(
        spec=spec, seed=seed,
        seq_lens=L0.to(torch.int32).to(device),
        page_ptr=page_ptr.to(torch.int32).to(device),
        page_indices=page_indices.to(torch.int32).to(device),
        row_capacity=cap.to(torch.int32).to(device),
        max_pages=max(int(n_final.max()) if B > 0 else 1, 1),
        num_pool_pages=pool,
        k_cache=k_cache, v_cache=v_cache, q=q, planted=planted,
        step_q=step_q, step_k_new=step_k, step_v_new=step_v,
    )


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


def host_subset(w: Workload, requests: List[int], seq_lens: Optional[torch.Tensor] = None,
                k_cache: Optional[torch.Tensor] = None, v_cache: Optional[torch.Tensor] = None):
    """Host copy of only the pages some of the requests hold, renumbered compactly.

    Returns a dict of numpy arrays (k_cache/v_cache as uint16 bits, page table int32)
    plus `phys` (new page -> original physical id).  Plumbing only: a gather of pages.
    """
    import numpy as np
    L = (w.seq_lens if seq_lens is None else seq_lens).cpu().to(torch.int64)
    ptr = w.page_ptr.cpu().to(torch.int64)
    idx = w.page_indices.cpu().to(torch.int64)
    P = w.spec.page_size
    kc = w.k_cache if k_cache is None else k_cache
    vc = w.v_cache if v_cache is None else v_cache
    phys, rows, lens = [], [], []
    for b in requests:
        nb = int((L[b] + P - 1) // P)
        ids = idx[int(ptr[b]):int(ptr[b]) + nb]
        rows.append(list(range(len(phys), len(phys) + nb)))
        phys.extend(ids.tolist())
        lens.append(int(L[b]))
    phys_t = torch.tensor(phys, dtype=torch.int64)
    dev = kc.device
    out = {
        "k_cache": bits(kc[phys_t.to(dev)]),
        "v_cache": None if vc is None else bits(vc[phys_t.to(dev)]),
        "page_ptr": np.array([r[0] if r else 0 for r in rows], dtype=np.int32),
        "page_indices": np.arange(len(phys), dtype=np.int32),
        "seq_lens": np.array(lens, dtype=np.int32),
        "phys": np.array(phys, dtype=np.int64),
    }
    if len(out["page_indices"]) == 0:
        out["page_indices"] = np.zeros(1, np.int32)
    # rows are consecutive: page_ptr[b] = first compact page of request b
    starts, acc = [], 0
    for r in rows:
        starts.append(acc)
        acc += len(r)
    out["page_ptr"] = np.array(starts, dtype=np.int32)
    return out

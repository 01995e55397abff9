"""Benchmark: block top-k sparse attention decode over a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--mode exact|approx|approx1024|approx256]
    python bench.py --impl reference ...     # the fp64 CPU oracle on the host cores

A step is one decode step of one layer: score every page of every request from the
cached centroids, select the top-k pages per (request, KV head), attend exactly over
them (split-K + log-sum-exp merge); the continuous-batching workload first appends one
token per request and updates the tail page's centroid.  `value` is query tokens/s per
layer (batch / step time) summed over ranks.  Consecutive timed steps cycle through
independent copies of the inputs (separate page pools, caches, centroids and queries)
so that no step finds its working set in L2; steps are replayed from CUDA graphs and
timed with CUDA events on the launching stream.

Multi-GPU: every rank runs its own independent batch (weak scaling, no collective on
the data path); timings are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-decode query tokens/s per layer; achieved HBM GB/s vs B200 peak"
UNIT = "query tokens/s"
L2_BYTES = 126 * 1024 * 1024
DEFAULT_CONFIG = "qwen3_1p7b_gqa_b32"

# DRAM traffic of the dominant kernel from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum),
# as a multiple of the algorithmic bytes of the captured launch, per (kernel source, workload); valid only
# for the kernel source it was taken on (sha256 of the file), otherwise the bench reports null.
DECODE_TRAFFIC = [
    {"file": "csrc/k_decode.cu", "sha256": "836824bf1089964ce4de52184d5e180253562ffb75dbade3387bb195cbaeab2f",
     "ratio": (268.934912 + 3.29856 + 268.955392 + 0.409856) / (2 * 268.511488), "workload": "qwen3_1p7b_gqa_b32",
     "note": "two consecutive launches of the full workload (2 input copies), 1-pass dram__bytes capture"},
    {"file": "csrc/k_decode.cu", "sha256": "836824bf1089964ce4de52184d5e180253562ffb75dbade3387bb195cbaeab2f",
     "ratio": (67.366656 + 0.883456 + 67.365888 + 0.361984) / (2 * 67.1744), "workload": "long_ctx_128k_b8",
     "note": "captured at batch 4 (67.2 MB per launch, two launches), scaled to the full launch by its bytes"},
    {"file": "csrc/k_decode.cu", "sha256": "836824bf1089964ce4de52184d5e180253562ffb75dbade3387bb195cbaeab2f",
     "ratio": (674.105088 + 8.291072 + 674.06336 + 5.162496) / (2 * 672.470302), "workload": "cont_batch_b256",
     "note": "captured at batch 160 (672.5 MB per launch, two steps; the split with late pieces, as at batch 256), "
             "scaled to the full launch by its bytes"},
    {"file": "csrc/k_decode_mla.cu", "sha256": "22e81ccb531f4f8aa2fb7013d797d94d058073446b7d6bf9de54dc1da54b31da",
     "ratio": (38.15936 + 0.050944 + 38.155264 + 0.000256) / (2 * 38.264896), "workload": "mla_576_512_b16",
     "note": "two consecutive launches of the full workload (2 input copies, the planned 128-CTA split), "
             "1-pass dram__bytes capture"},
]


def measured_traffic(kernel_file, workload, algorithmic_bytes):
    import hashlib
    path = os.path.join(ROOT, "paged_block_sparse_kv_b200", kernel_file)
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(path, "rb").read()).hexdigest()
    for entry in DECODE_TRAFFIC:
        if entry["file"] == kernel_file and entry["workload"] == workload and entry["sha256"] == sha:
            return int(entry["ratio"] * algorithmic_bytes)
    return None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs of the job; more than 1 needs one process per GPU (torchrun sets WORLD_SIZE)")
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="vx", choices=["vx", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--mode", default="exact", choices=["exact", "approx", "approx1024", "approx256"],
                    help="top-k mode: exact, or approximate with 4096, 1024 or 256 codes")
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--no-table-ready", action="store_true",
                    help="call the chained step without VX_TABLE_READY (every read waits for the previous kernel)")
    ap.add_argument("--score-dims", type=int, default=0,
                    help="dims of the key scored against the centroids (0: all; 512 on MLA: rope-unaware)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (small profiling cases only)")
    ap.add_argument("--copies", type=int, default=0,
                    help="independent input copies to rotate (0: enough for > 3x L2); fewer only for ncu "
                         "captures, which flush the caches before each captured launch themselves")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--persistent", action="store_true",
                    help="time vx_block_topk_decode_persistent (one persistent kernel) instead of the chained call")
    ap.add_argument("--prefill-write", action="store_true",
                    help="time the prefill write instead (vx_centroid_update with first_pos = 0: every token of the "
                         "workload's contexts into its page slot, with the page centroids) and print its own line")
    ap.add_argument("--breakdown", action="store_true",
                    help="also time the score, top-k and decode calls separately (CUDA events, graphs)")
    return ap.parse_args()


# ------------------------------------------------------------------ peaks / clocks

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, enabled=True):
        self.gpu_id, self.enabled, self.proc, self.lines = gpu_id, enabled, None, []

    def __enter__(self):
        if self.enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                     "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1].split()[0]))
                mx.append(float(f[2].split()[0]))
            except Exception:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ roofline bytes

def step_bytes(w, sel, seq_lens, k):
    """Algorithmic HBM bytes of one step: centroid reads + selected valid K/V tokens + q + out.

    Returns (total, decode_part, centroid_part)."""
    import numpy as np
    s = w.spec
    L = seq_lens.cpu().numpy().astype(np.int64)
    P = s.page_size
    n = (L + P - 1) // P
    cen = int(n.sum()) * s.num_kv_heads * s.head_dim_qk * 2
    sel_h = sel.cpu().numpy()
    tok = 0
    for b in range(len(L)):
        rows = sel_h[b]
        valid = rows[rows >= 0].astype(np.int64)
        m = np.minimum(P, L[b] - valid * P)
        tok += int(m.sum())  # summed over the KV heads
    per_tok = s.head_dim_qk * 2 if s.mla_shared_kv else (s.head_dim_qk + s.head_dim_v) * 2
    kv = tok * per_tok
    qo = len(L) * s.num_q_heads * (s.head_dim_qk + s.head_dim_v) * 2
    return cen + kv + qo, kv + qo, cen


# ------------------------------------------------------------------ multi-rank helpers
# (weak scaling: every rank runs its own independent batch; the only collectives are a
# barrier and the max of the timings)

def rank_seed(config, rank):
    """Seed of rank `rank`'s synthetic workload: independent draws per rank."""
    from paged_block_sparse_kv_b200 import synth
    return 1000 * list(synth.SPECS).index(config) + 17 * rank


def max_over_ranks(ms, world, device):
    """The slowest rank's time (every rank must call it, in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(batch_per_rank, ms_per_step, world):
    """Query tokens per second of the whole job: every rank's batch, at the slowest rank's step time."""
    return batch_per_rank / (ms_per_step * 1e-3) * world


# ------------------------------------------------------------------ our arm

def progress(rank, t0, what, errs=None):
    """One line per bench phase on stderr (rank 0): wall seconds since start and, when given,
    the device error words so far."""
    if rank == 0:
        extra = "" if errs is None else f" device errors {errs}"
        print(f"[bench] {time.time() - t0:7.1f} s  {what}{extra}", file=sys.stderr, flush=True)


def run_vx(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    t_start = time.time()

    from paged_block_sparse_kv_b200 import synth, vx

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    spec = synth.SPECS[args.config]
    if args.batch:
        spec = synth.Spec(**{**spec.__dict__, "batch": args.batch})
    mode = {"exact": 0, "approx": 1, "approx1024": 2, "approx256": 3}[args.mode]
    # the chained steps' mode: the page tables and lengths here are set up before the timed
    # region (or copied in by the e2e leg's own H2D copies), never written by the kernel
    # right before a call, so the scorer may read them while that kernel finishes
    step_mode = mode if args.no_table_ready else mode | vx.VX_TABLE_READY
    k = spec.k
    B = spec.batch

    def geom(w):
        return vx.Geometry(w.batch, spec.num_q_heads, spec.num_kv_heads, spec.head_dim_qk, spec.head_dim_v,
                           spec.page_size, spec.mla_shared_kv, w.num_pool_pages)

    seed0 = rank_seed(args.config, rank)

    def buffers(w, geo):
        out = torch.empty((B, spec.num_q_heads, spec.head_dim_v), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, spec.num_q_heads), dtype=torch.float32, device=dev)
        scores = torch.empty((B, spec.num_kv_heads, w.max_pages), dtype=torch.float32, device=dev)
        sel = torch.empty((B, spec.num_kv_heads, k), dtype=torch.int32, device=dev)
        ws = torch.zeros(vx.vx_workspace_size(geo, w.max_pages, k, args.splits), dtype=torch.uint8, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        return dict(out=out, lse=lse, scores=scores, sel=sel, ws=ws, err=err)

    def rebuild_centroids(w, geo, tab):
        cen = torch.zeros((w.num_pool_pages, spec.num_kv_heads, spec.head_dim_qk), dtype=torch.bfloat16, device=dev)
        vx.vx_centroid_update(geo, tab, w.k_cache, cen, v_cache=w.v_cache)
        return cen

    def fused(c):
        if args.persistent:
            if c["append"]:
                vx.vx_centroid_update(c["geo"], c["tab"], c["w"].k_cache, c["cen"], v_cache=c["w"].v_cache,
                                      k_new=c["k_new"], v_new=c["v_new"], err=c["err"])
            vx.vx_block_topk_decode_persistent(c["geo"], c["tab"], c["q"], c["w"].k_cache, c["w"].v_cache, c["cen"],
                                               k, c["out"], c["ws"], lse=c["lse"], scores_out=c["scores"],
                                               sel_out=c["sel"], err=c["err"])
            return
        if c["append"]:  # one call: the append, then the chained step
            vx.vx_block_topk_decode_append(c["geo"], c["tab"], c["q"], c["w"].k_cache, c["w"].v_cache, c["cen"],
                                           c["k_new"], c["v_new"], k, c["out"], c["ws"], lse=c["lse"], mode=step_mode,
                                           seed=0, num_splits=args.splits, score_dims=args.score_dims,
                                           scores_out=c["scores"], sel_out=c["sel"], err=c["err"])
            return
        vx.vx_block_topk_decode(c["geo"], c["tab"], c["q"], c["w"].k_cache, c["w"].v_cache, c["cen"], k, c["out"],
                                c["ws"], lse=c["lse"], mode=step_mode, seed=0, num_splits=args.splits,
                                score_dims=args.score_dims, scores_out=c["scores"], sel_out=c["sel"], err=c["err"])

    st = []
    if spec.steps == 0:
        # independent input copies, rotated so no step finds its inputs in L2
        w = synth.make(spec, seed0, dev)
        geo = geom(w)
        tab = vx.PageTable(w.page_ptr, w.page_indices, w.seq_lens, w.max_pages)
        st.append(dict(w=w, geo=geo, tab=tab, cen=rebuild_centroids(w, geo, tab), q=w.q, append=False,
                       seq_lens=w.seq_lens, **buffers(w, geo)))
        fused(st[0])
        torch.cuda.synchronize()
        progress(rank, t_start, "first step", [int(st[0]["err"].item())])
        total0 = step_bytes(w, st[0]["sel"], w.seq_lens, k)[0]
        # the other copies' bytes between two uses of one copy exceed 3x L2
        n_copies = args.copies or max(2, math.floor(3 * L2_BYTES / max(total0, 1)) + 2)
        for i in range(1, n_copies):
            w = synth.make(spec, seed0 + i, dev)
            geo = geom(w)
            tab = vx.PageTable(w.page_ptr, w.page_indices, w.seq_lens, w.max_pages)
            st.append(dict(w=w, geo=geo, tab=tab, cen=rebuild_centroids(w, geo, tab), q=w.q, append=False,
                           seq_lens=w.seq_lens, **buffers(w, geo)))
        l2_note = "inputs rotate over {n} independent copies, {mb:.0f} MB between reuses " + (
            "(> 3x L2)" if (n_copies - 1) * total0 > 3 * L2_BYTES else "(fewer than 3x L2: profiling run only)")
    else:
        # continuous batching: one workload, `steps` consecutive decode steps, each appending
        # one token per request before it decodes (replays rewrite the same slots)
        w = synth.make(spec, seed0, dev)
        geo = geom(w)
        lens = torch.stack([w.seq_lens_at(s_) for s_ in range(spec.steps)]).contiguous()
        cen = rebuild_centroids(w, geo, vx.PageTable(w.page_ptr, w.page_indices, w.seq_lens, w.max_pages))
        shared = buffers(w, geo)
        for s_ in range(spec.steps):
            tab = vx.PageTable(w.page_ptr, w.page_indices, lens[s_], w.max_pages)
            ctx = dict(w=w, geo=geo, tab=tab, cen=cen, q=w.step_q[s_], append=True, k_new=w.step_k_new[s_],
                       v_new=w.step_v_new[s_], seq_lens=lens[s_], **shared)
            ctx["sel"] = torch.empty_like(shared["sel"])
            st.append(ctx)
        l2_note = "{n} consecutive appending decode steps over one {mb:.0f} MB-per-step working set (> L2)"
    # kernels per step: the centroid append (continuous batching), then the fused call's own
    # (scores, top-k, attention, merge; the persistent entry is one kernel)
    launches_per_step = (1 if args.persistent else 4) + (1 if st[0]["append"] else 0)
    progress(rank, t_start, f"{len(st)} input copies ready")
    for c in st:
        fused(c)
    torch.cuda.synchronize()
    progress(rank, t_start, "one step per copy", sorted(set(int(c["err"].item()) for c in st)))
    per_copy = [step_bytes(c["w"], c["sel"], c["seq_lens"], k) for c in st]

    stream = torch.cuda.Stream(device=dev)
    def capture(n_steps, start, fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(n_steps):
                    fn(st[(start + i) % len(st)])
        return g

    def timed_replay(fn, steps, warmup, chunk=500):
        # warm-up (eager) then graphs of `chunk` steps; exactly `steps` timed steps
        with torch.cuda.stream(stream):
            for i in range(warmup):
                fn(st[i % len(st)])
        torch.cuda.synchronize()
        c = min(chunk, steps)
        c -= c % len(st) if c >= len(st) else 0
        c = max(c, 1)
        full, rem = divmod(steps, c)
        g_full = capture(c, 0, fn)
        g_rem = capture(rem, 0, fn) if rem else None
        torch.cuda.synchronize()
        g_full.replay()  # one untimed replay primes the graph
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(full):
                g_full.replay()
            if g_rem is not None:
                g_rem.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        return ms, (g_full, c)

    gpu_id = _gpu_id(local_rank)
    with ClockSampler(gpu_id, enabled=not args.no_clocks and rank == 0) as clk:
        ms_total, (g_full, chunk) = timed_replay(fused, args.steps, args.warmup)
        progress(rank, t_start, f"timed steps: {ms_total / args.steps * 1e3:.2f} us per step")
        # keep the GPU in the same steady state for >= 1 s so the sampler sees it
        t_end = time.time() + 1.0
        while time.time() < t_end:
            with torch.cuda.stream(stream):
                g_full.replay()
            torch.cuda.synchronize()
    clocks = clk.summary()

    # per-step distribution of the appending loop (mean and median over its steps): one graph per
    # step, replayed back to back with an event between steps (so no overlap across steps)
    progress(rank, t_start, "clock sampling done")
    per_step = None
    if spec.steps:
        import numpy as np
        gs = [capture(1, i, fused) for i in range(len(st))]
        torch.cuda.synchronize()
        n_ps = 2 * len(st)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ps + 1)]
        with torch.cuda.stream(stream):
            for i in range(n_ps):
                evs[i].record(stream)
                gs[i % len(st)].replay()
            evs[n_ps].record(stream)
        torch.cuda.synchronize()
        ts = [evs[i].elapsed_time(evs[i + 1]) * 1e3 for i in range(n_ps)]
        per_step = {"mean_us": round(float(np.mean(ts)), 2), "p50_us": round(float(np.median(ts)), 2),
                    "steps": n_ps, "method": "one CUDA graph per step, replayed back to back, events between steps"}
        del gs

    ms_step = ms_total / args.steps
    mean_bytes = sum(p[0] for p in per_copy) / len(per_copy)
    tok_s = job_throughput(B, ms_step, world)
    peak, peak_kind = peaks()
    step_gbs = mean_bytes / (ms_step * 1e-3) / 1e9

    # dominant kernel: the sparse decode call (gather-attention kernel + its merge), timed alone
    def decode_only(c):
        vx.vx_sparse_decode(c["geo"], c["tab"], c["q"], c["w"].k_cache, c["w"].v_cache, c["sel"], k, c["out"],
                            c["ws"], lse=c["lse"], num_splits=args.splits, err=c["err"])
    dec_steps = max(len(st), min(args.steps, 1000))
    ms_dec, _ = timed_replay(decode_only, dec_steps, 3)
    progress(rank, t_start, f"sparse decode call: {ms_dec / dec_steps * 1e3:.2f} us")
    ms_dec_launch = ms_dec / dec_steps
    dec_bytes = sum(p[1] for p in per_copy) / len(per_copy)
    dec_gbs = dec_bytes / (ms_dec_launch * 1e-3) / 1e9

    breakdown = None
    if args.breakdown:
        def score_only(c):
            vx.vx_score_pages(c["geo"], c["tab"], c["q"], c["cen"], c["scores"], err=c["err"])

        def topk_only(c):
            vx.vx_topk_pages(c["geo"], c["tab"], c["scores"], k, c["sel"], mode=mode, seed=0, err=c["err"])

        def chain(c):  # the same step as three separate calls (no programmatic dependent launch)
            score_only(c)
            topk_only(c)
            decode_only(c)

        nb = max(len(st), min(args.steps, 1000))
        breakdown = {}
        for name, fn in (("score", score_only), ("topk", topk_only), ("decode_merge", decode_only),
                         ("chain", chain)):
            ms_b, _ = timed_replay(fn, nb, 3)
            breakdown[name + "_us"] = round(ms_b / nb * 1e3, 3)
            progress(rank, t_start, f"breakdown {name}: {breakdown[name + '_us']} us")
        if spec.steps:
            def append_only(c):
                vx.vx_centroid_update(c["geo"], c["tab"], c["w"].k_cache, c["cen"], v_cache=c["w"].v_cache,
                                      k_new=c["k_new"], v_new=c["v_new"], err=c["err"])
            ms_b, _ = timed_replay(append_only, nb, 3)
            breakdown["append_us"] = round(ms_b / nb * 1e3, 3)
        breakdown["step_us"] = round(ms_step * 1e3, 3)

    # end to end through the public call with host buffers.  Every step copies that step's
    # inputs (query, page table, lengths; the appended K/V rows when the step appends) from one
    # packed pinned host buffer to the device in one H2D copy, makes the call, and reads out
    # and lse back in one D2H copy into pinned memory.  Buffer sets alternate and the
    # copies run on two more streams, so step i+1's H2D and step i-1's D2H overlap step i's
    # kernels (the call's own stream order is unchanged); the steps are replayed from CUDA
    # graphs like the device-timed leg.
    def packed(tensors):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.zeros(n, dtype=torch.uint8, device=dev)
        views = []
        for t, o in zip(tensors, offs):
            v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
            v.copy_(t)
            views.append(v)
        return buf, views

    # one buffer set per input copy (the same copies the device-timed leg rotates over, so no
    # step finds its cache pages in L2), at least two so consecutive steps never share buffers
    sets = []
    for j in range(max(2, min(len(st), 8))):
        c = st[j % len(st)]
        w = c["w"]
        ins = [c["q"], w.page_ptr, w.page_indices, c["seq_lens"]]
        if c["append"]:
            ins += [c["k_new"], c["v_new"]]
        d_in, v_in = packed(ins)
        d_out, (v_out, v_lse) = packed([c["out"], c["lse"]])
        ce = dict(c, q=v_in[0], seq_lens=v_in[3], out=v_out, lse=v_lse,
                  tab=vx.PageTable(v_in[1], v_in[2], v_in[3], w.max_pages))
        if c["append"]:
            ce["k_new"], ce["v_new"] = v_in[4], v_in[5]
        sets.append(dict(d_in=d_in, d_out=d_out, ctx=ce, h_in=d_in.cpu().pin_memory(),
                         h_out=torch.empty(d_out.shape, dtype=torch.uint8).pin_memory(),
                         ev_in=torch.cuda.Event(), ev_comp=torch.cuda.Event(), ev_done=torch.cuda.Event()))
    nsets = len(sets)
    h2d = sum(S["d_in"].numel() for S in sets) / nsets
    d2h = sum(S["d_out"].numel() for S in sets) / nsets
    in_stream, out_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_steps_on(n):  # n steps; the copy streams fork from and join `stream`
        in_stream.wait_stream(stream)
        out_stream.wait_stream(stream)
        for i in range(n):
            S = sets[i % nsets]
            with torch.cuda.stream(in_stream):
                if i >= nsets:
                    in_stream.wait_event(S["ev_done"])  # the set's previous call and D2H are done
                S["d_in"].copy_(S["h_in"], non_blocking=True)
                S["ev_in"].record(in_stream)
            stream.wait_event(S["ev_in"])
            fused(S["ctx"])
            S["ev_comp"].record(stream)
            with torch.cuda.stream(out_stream):
                out_stream.wait_event(S["ev_comp"])
                S["h_out"].copy_(S["d_out"], non_blocking=True)
                S["ev_done"].record(out_stream)
        stream.wait_stream(in_stream)
        stream.wait_stream(out_stream)

    e2e_steps = max(1, args.e2e_steps)
    with torch.cuda.stream(stream):
        e2e_steps_on(2 * nsets)
    torch.cuda.synchronize()
    chunk_e = min(e2e_steps, 100)
    g_e = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g_e, stream=stream):
            e2e_steps_on(chunk_e)
    # warm-up: one untimed window of back-to-back replays, exactly like the timed one.  The
    # first such window of a process runs about 1.7 ms slower in all (measured: 88.8 against
    # 80.2 us per step over 200 steps, every later window 80.1-80.3), whatever the number of
    # single synchronised replays before it; the device-only legs show no such step.
    reps = max(1, e2e_steps // chunk_e)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g_e.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(reps):
            g_e.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1) / (reps * chunk_e), world, dev)
    del g_e
    # the outputs that came back are the call's (a bad copy path would not match)
    for S in sets:
        assert torch.equal(S["h_out"].to(dev), S["d_out"]), "e2e: the D2H copy does not hold the call's outputs"

    errs = [int(c["err"].item()) for c in st]
    progress(rank, t_start, f"e2e: {ms_e2e * 1e3:.2f} us per step", sorted(set(errs)))
    # the device-timed steps once more, after the other legs (a drift here is the GPU's state,
    # e.g. its clocks after seconds of load, not the e2e copies)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g_full.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    progress(rank, t_start, f"device steps again after e2e: {e0.elapsed_time(e1) / chunk * 1e3:.2f} us per step")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(st[0]["w"], st[0]["cen"], k, st[0]["seq_lens"], st[0]["q"])

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(tok_s, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.config + (f" (batch overridden to {B})" if args.batch else ""), "batch": B, "num_q_heads": spec.num_q_heads,
                       "num_kv_heads": spec.num_kv_heads, "head_dim_qk": spec.head_dim_qk,
                       "head_dim_v": spec.head_dim_v, "page_size": spec.page_size, "k_pages": k,
                       "context": list(spec.ctx), "topk_mode": args.mode, "splits": args.splits or "planned",
                       "score_dims": args.score_dims or spec.head_dim_qk,
                       "table_ready": not (args.no_table_ready or args.persistent),
                       "entry": "vx_block_topk_decode_persistent" if args.persistent else (
                           "vx_block_topk_decode_append" if st[0]["append"] else "vx_block_topk_decode"),
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": l2_note.format(n=len(st), mb=mean_bytes * max(1, len(st) - 1) / 1e6)},
            "hbm": {"roofline_bytes_per_step": int(mean_bytes), "achieved_gbs": round(step_gbs, 1),
                    "peak_gbs": peak, "frac": round(step_gbs / peak, 4), "peak_kind": peak_kind,
                    "centroid_bytes": int(sum(p[2] for p in per_copy) / len(per_copy))},
            "roofline": {"bound": "hbm", "kernel": "sparse decode (gather-attention + merge)",
                         "achieved": round(dec_gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(dec_gbs / peak, 4),
                         "traffic": measured_traffic("csrc/k_decode_mla.cu" if spec.mla_shared_kv else
                                                     "csrc/k_decode.cu", args.config, dec_bytes),
                         "bytes_per_launch": int(dec_bytes), "us_per_launch": round(ms_dec_launch * 1e3, 3),
                         "peak_kind": peak_kind},
            "e2e": {"value": round(job_throughput(B, ms_e2e, world), 1), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms_e2e, 4),
                    "method": "per step: one H2D of the packed inputs from pinned memory, the public call, one "
                              "D2H of out+lse into pinned memory; copies on their own streams overlapping the "
                              "neighbouring steps' kernels (two buffer sets); CUDA-graph replay, CUDA events"},
            "gpu_launches": launches_per_step * args.steps,
            "breakdown": breakdown,
            "clocks": clocks,
            "device_errors": errs,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if per_step is not None:
            line["per_step"] = per_step
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _gpu_id(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",")]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------------ oracle (CPU) timing

def cpu_baseline(w, cen, k, seq_lens, q, budget_s=15.0):
    """The oracle, as it stands, on the host cores over a bounded sample of the workload:
    the first requests of one step, repeated for about `budget_s` seconds."""
    import torch

    import oracle
    from paged_block_sparse_kv_b200 import synth
    reqs = list(range(min(4, w.batch)))
    h = synth.host_subset(w, reqs, seq_lens=seq_lens)
    cen_h = synth.bits(cen[torch.as_tensor(h["phys"], dtype=torch.int64, device=cen.device)])
    P = w.spec.page_size
    maxp = int(((h["seq_lens"] + P - 1) // P).max())
    args = (synth.bits(q[:len(reqs)]), h["k_cache"], h["v_cache"], cen_h, h["page_ptr"], h["page_indices"],
            h["seq_lens"], maxp, k)
    kw = dict(mla_shared_kv=w.spec.mla_shared_kv, head_dim_v=w.spec.head_dim_v)
    t0 = time.perf_counter()
    oracle.decode_step(*args, **kw)
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.decode_step(*args, **kw)
    dt = time.perf_counter() - t0
    cores = oracle.num_threads()
    # the same call on one core: the first request only, a few seconds
    args1 = (args[0][:1], h["k_cache"], h["v_cache"], cen_h, h["page_ptr"][:1], h["page_indices"], h["seq_lens"][:1],
             maxp, k)
    prev = oracle.set_num_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.decode_step(*args1, **kw)
        one1 = time.perf_counter() - t0
        reps1 = max(1, int(budget_s / 3 / max(one1, 1e-6)))
        t0 = time.perf_counter()
        for _ in range(reps1):
            oracle.decode_step(*args1, **kw)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(prev)
    return {"value": round(len(reqs) * reps / dt, 3), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{len(reqs)} of {w.batch} requests x {reps} decode steps (score + exact top-k + "
                      f"attention, fp64), {dt:.1f} s",
            "single_thread": {"value": round(reps1 / dt1, 3), "unit": UNIT, "cores": 1,
                              "sample": f"1 of {w.batch} requests x {reps1} decode steps, {dt1:.1f} s"}}


def run_reference(args, rank, world, budget_s=150.0):
    """The fp64 oracle, as it stands, timed on the host cores: each step is a bounded sample
    of the workload (2 requests; fewer KV heads when K + W steps of that would not fit in
    about `budget_s` seconds)."""
    if rank != 0:
        return
    import numpy as np

    import oracle
    from paged_block_sparse_kv_b200 import synth
    spec = synth.SPECS[args.config]
    n_req = min(spec.batch, 2)  # requests drawn for the sample (the workload's first two)
    w = synth.make(synth.Spec(**{**spec.__dict__, "steps": 0}), rank_seed(args.config, 0), "cpu", batch=n_req)
    h = synth.host_subset(w, list(range(n_req)))
    _, cen16 = oracle.centroids(h["k_cache"], h["page_ptr"], h["page_indices"], h["seq_lens"])
    maxp = int(((h["seq_lens"] + spec.page_size - 1) // spec.page_size).max())
    q = synth.bits(w.q)
    G = spec.num_q_heads // spec.num_kv_heads

    def call(hk):
        v = None if h["v_cache"] is None else np.ascontiguousarray(h["v_cache"][:, :hk])
        return oracle.decode_step(np.ascontiguousarray(q[:, :hk * G]), np.ascontiguousarray(h["k_cache"][:, :hk]), v,
                                  np.ascontiguousarray(cen16[:, :hk]), h["page_ptr"], h["page_indices"],
                                  h["seq_lens"], maxp, spec.k, mla_shared_kv=spec.mla_shared_kv,
                                  head_dim_v=spec.head_dim_v)

    t0 = time.perf_counter()
    call(spec.num_kv_heads)
    one = time.perf_counter() - t0
    per_step = budget_s / max(1, args.steps + args.warmup)
    hk = spec.num_kv_heads if one <= per_step else max(1, int(spec.num_kv_heads * per_step / one))
    for _ in range(args.warmup):
        call(hk)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call(hk)
    dt = time.perf_counter() - t0
    req_per_step = n_req * hk / spec.num_kv_heads
    value = req_per_step * args.steps / dt
    sample = (f"{n_req} of {spec.batch} requests, {hk} of {spec.num_kv_heads} KV heads per step "
              f"(score + exact top-k + attention, fp64)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.config, "k_pages": spec.k, "sample": sample},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill_write(args, rank, world, local_rank):
    """Whole-context prefill write of the workload's requests: read the packed new K/V once,
    write them into their slots and the page centroids; HBM-bound, reported against the copy peak."""
    import torch

    import torch.distributed as dist

    from paged_block_sparse_kv_b200 import synth, vx
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    spec = synth.SPECS[args.config]
    spec = synth.Spec(**{**spec.__dict__, "steps": 0, **({"batch": args.batch} if args.batch else {})})
    w = synth.make(spec, rank_seed(args.config, rank), dev)
    geo = vx.Geometry(w.batch, spec.num_q_heads, spec.num_kv_heads, spec.head_dim_qk, spec.head_dim_v,
                      spec.page_size, spec.mla_shared_kv, w.num_pool_pages)
    tab = vx.PageTable(w.page_ptr, w.page_indices, w.seq_lens, w.max_pages)
    n_tok = int(w.seq_lens.sum())
    g = torch.Generator(device=dev).manual_seed(5)
    k_new = torch.randn((n_tok, spec.num_kv_heads, spec.head_dim_qk), generator=g, device=dev).to(torch.bfloat16)
    v_new = None if spec.mla_shared_kv else torch.randn((n_tok, spec.num_kv_heads, spec.head_dim_v), generator=g,
                                                        device=dev).to(torch.bfloat16)
    cen = torch.zeros((w.num_pool_pages, spec.num_kv_heads, spec.head_dim_qk), dtype=torch.bfloat16, device=dev)
    fp = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def call():
        vx.vx_centroid_update(geo, tab, w.k_cache, cen, v_cache=w.v_cache, k_new=k_new, v_new=v_new, first_pos=fp,
                              err=err, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(1, min(args.steps, 50))
    with ClockSampler(_gpu_id(local_rank), not args.no_clocks) as clk:
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                call()  # 2.4+ GB per call at the default workload: nothing stays in L2 between calls
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error word {int(err.item())}"
    kv_row = spec.num_kv_heads * (spec.head_dim_qk + (0 if spec.mla_shared_kv else spec.head_dim_v)) * 2
    pages = int(((w.seq_lens + spec.page_size - 1) // spec.page_size).sum())
    algo = 2 * n_tok * kv_row + pages * spec.num_kv_heads * spec.head_dim_qk * 2  # read + write, centroids
    # the ranks draw their own contexts, so the job's bytes are the sum over ranks
    algo_job = algo
    if world > 1:
        t = torch.tensor([float(algo)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        algo_job = float(t.item())
    peak, peak_kind = peaks()
    gbs = algo / (ms * 1e-3) / 1e9
    if rank == 0:
        print(json.dumps({"metric": "prefill write (KV slots + page centroids) GB/s",
                          "value": round(algo_job / (ms * 1e-3) / 1e9, 1),
                          "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": max(3, args.warmup),
                          "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
                          "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": args.config + (f" (batch overridden to {w.batch})" if args.batch else ""),
                                     "tokens": n_tok, "pages": pages,
                                     "bytes_per_call": algo, "entry": "vx_centroid_update (first_pos = 0)"},
                          "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                                       "frac": round(gbs / peak, 4), "peak_kind": peak_kind},
                          "gpu_launches": steps, "clocks": clk.summary()}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def check_world(gpus, world):
    """--gpus must match the processes launched: one per GPU, WORLD_SIZE set by torchrun."""
    if gpus != world:
        raise SystemExit(f"bench.py: --gpus {gpus} but {world} process(es) launched; for N > 1 GPUs launch "
                         f"one process per GPU with torchrun --nproc-per-node N")


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    check_world(args.gpus, world)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.prefill_write:
        run_prefill_write(args, rank, world, local_rank)
        return
    run_vx(args, rank, world, local_rank)


if __name__ == "__main__":
    main()

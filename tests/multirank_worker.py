"""Worker body of test_multirank_host.py: one gloo rank on CPU calling the multi-rank helpers
that bench.py uses (kept in its own module so spawned processes can import it)."""
import contextlib
import datetime
import io
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_rank(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank r's own step time
        slowest = bench.max_over_ranks(ms, world, "cpu")
        e2e = bench.max_over_ranks(2.0 * ms, world, "cpu")  # a second reduction, same order on every rank
        seed = bench.rank_seed("qwen3_1p7b_gqa_b32", rank)
        tput = bench.job_throughput(32, slowest, world)
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            ret = bench.run_reference(None, rank, world) if rank != 0 else None  # other ranks: no work
        dist.barrier()
        queue.put((rank, slowest, e2e, seed, tput, ret, out.getvalue()))
    finally:
        dist.destroy_process_group()

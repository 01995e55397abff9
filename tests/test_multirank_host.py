"""The N > 1 path of bench.py on CPU: two gloo ranks (127.0.0.1) run the helpers the GPU bench
uses.  Every rank ends with the slowest rank's time, ranks draw independent workloads (weak
scaling: no data-path collective), the job throughput counts every rank's batch at that time,
and the reference arm does no work on ranks other than 0."""
import multiprocessing as mp
import socket

import multirank_worker


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_share_the_slowest_time():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=multirank_worker.run_rank, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        rank, slowest, e2e, seed, tput, ret, out = queue.get(timeout=120)
        results[rank] = (slowest, e2e, seed, tput, ret, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0][0] == results[1][0] == 15.0          # max over ranks of 10 and 15 ms
    assert results[0][1] == results[1][1] == 30.0          # second reduction, same order
    assert results[0][2] != results[1][2]                  # independent draws per rank
    assert abs(results[0][3] - 32 * 2 / 15e-3) < 1e-6      # both ranks' batches at the slowest time
    assert results[1][4] is None and results[1][5] == ""   # reference arm: rank 1 does nothing

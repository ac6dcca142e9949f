"""The N > 1 host path of bench.py on CPU: two gloo ranks (no GPU).

With several GPUs every rank streams its own replica of the workload; the only
cross-rank traffic is the barrier around the timed region and the max over ranks of the
elapsed time, which is what rank 0 reports.  Here two processes rendezvous on
127.0.0.1 over gloo and exercise exactly those calls.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    r, w, local = bench.dist_setup(world)
    bench.barrier(w)
    got = bench.max_over_ranks(1.5 + r, w)       # elapsed ms of each rank
    bench.barrier(w)
    ref = bench.run_reference(None, None, r, w) if r != 0 else "rank0"
    bench._teardown(w)
    queue.put((r, w, local, got, ref))


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_elapsed_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1]
    assert all(o[1] == 2 for o in out)
    assert all(o[3] == 2.5 for o in out)          # both ranks see the slowest rank's time
    assert out[1][4] is None                       # the reference arm runs on rank 0 only

"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks timing reduction, barriers, and that only rank 0 runs and
prints the reference arm.  The data path has no collective ("replicas
only"), so this is all the multi-rank logic there is."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import bench
    w, r, _ = bench.dist_setup()
    try:
        mx = bench.max_over_ranks(1.5 + r, w, torch.device("cpu"))
        bench.barrier(w)

        class A:
            steps, warmup, workload, reference_seconds = 2, 1, "square4096", 0.5
        line = bench.run_reference(A(), w, r)
        q.put((r, w, mx, None if line is None else line["impl"]))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0] == (0, 2, 2.5, "reference")      # max over ranks; rank 0 runs the reference arm
    assert res[1] == (1, 2, 2.5, None)             # other ranks do no work

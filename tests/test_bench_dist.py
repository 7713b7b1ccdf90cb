"""The multi-rank timing reduction of bench.py on two gloo ranks (CPU): every rank ends with the
maximum of the per-rank times, as the benchmark's max-over-ranks rule requires."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import sys

    import torch.distributed as dist

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = [1.25, 3.5][rank]
    got = bench.reduce_max(local, dist, "cpu")
    out[rank] = got
    dist.destroy_process_group()


def test_reduce_max_two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 3.5 and out[1] == 3.5


def test_reduce_max_single_process():
    import bench

    assert bench.reduce_max(2.0, None, "cpu") == 2.0

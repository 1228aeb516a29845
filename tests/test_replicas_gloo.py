"""The N > 1 host path of bench.py: step times reduced with a max over ranks, whole-job counts
with a sum over ranks (gloo, world size 2, CPU)."""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", init_method="env://", rank=rank, world_size=world)
    ws, r, local = bench._dist_env()
    assert (ws, r, local) == (world, rank, rank)
    got = bench.max_over_ranks([10.0 + rank, 3.0 - rank])
    total = bench.sum_over_ranks([1.0 + rank, 100.0])
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, (got, total)))


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == ([11.0, 3.0], [3.0, 200.0])


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.sum_over_ranks([1.5, 2.5]) == [1.5, 2.5]

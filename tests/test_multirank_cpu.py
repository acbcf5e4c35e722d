"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): every rank gets
the max elapsed time and its own batch; no data-path collective exists."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from sparse_rank_approximation_b200.workloads import make_inputs, small_workload
    got = bench.max_over_ranks(10.0 * (rank + 1))
    x = make_inputs(small_workload(N=64, H=1), seed=bench.rank_seed(rank))["Q"]
    dist.barrier()
    q.put((rank, got, float(x.sum())))
    dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]
    assert res[0][2] != res[1][2]

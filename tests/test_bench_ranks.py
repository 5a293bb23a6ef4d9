"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): each rank
runs its own independently seeded stream, the job time is the max over ranks
and the job value counts every rank's units."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from windowed_memory_attention_b200 import inputs
    elapsed = [120.0, 150.0][rank]
    t = bench.max_over_ranks(elapsed, world)
    w = bench.rank_workload(rank, layers=1).with_(M=8, H=2)
    k0 = inputs.draw(w, 0, "k")
    gathered = [torch.zeros_like(k0) for _ in range(world)]
    dist.all_gather(gathered, k0)
    q.put((rank, t, bench.job_value(10 * 24, world, t), w.seed0,
           bool(torch.equal(gathered[0], gathered[1]))))
    dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_streams():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value, seed0, same in res:
        assert t == 150.0                      # the slower rank sets the job time
        assert value == pytest.approx(2 * 240 / 0.150)
        assert seed0 == rank
        assert not same                        # the two ranks stream different data

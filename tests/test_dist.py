"""Multi-process host logic of bench.py on CPU (gloo, world size 2): each
replica times its own work; the job reports the max over ranks; barriers and
the reference arm's rank-0-only rule hold."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    bench.barrier(world)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    seeds = [None] * world
    dist.all_gather_object(seeds, bench.rank_seed(rank))
    out.put((rank, t, seeds))
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_and_distinct_streams_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, seeds in res:
        assert t == 15.0                        # the slowest rank sets the job time
        assert len(set(seeds)) == world         # each replica decodes its own stream


def test_reference_arm_prints_on_rank0_only(monkeypatch):
    import bench
    args = type("A", (), {"steps": 1, "warmup": 0, "rate": None, "ref_budget": 1.0})()
    res, show = bench.run_reference(args, bench.wl.CONFIGS[0], 2, 1, 1)
    assert res is None and show is False

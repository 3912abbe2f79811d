"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): the
slowest rank's time is what every rank reports, and whole-job throughput is
the units all ranks processed over that time (weak scaling, no data-path
collective)."""
import os
import socket

import pytest
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
    try:
        import bench
        my_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        value = bench.aggregate_throughput(1e9, ms, world)
        q.put((rank, ms, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate():
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
    for rank, ms, value in res:
        assert ms == 15.0                              # every rank reports the slowest rank
        assert value == pytest.approx(2 * 1e9 / 15e-3)  # all ranks' units over that time


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.aggregate_throughput(2.0, 1000.0, 1) == pytest.approx(2.0)


def _spawned_target(args):
    """A rank started by bench.spawn_ranks: joins a gloo group from the
    environment the launcher set and reports what it sees."""
    dist.init_process_group("gloo")
    try:
        import bench
        rank, world = dist.get_rank(), dist.get_world_size()
        ms = bench.max_over_ranks(20.0 + rank, dist, torch.device("cpu"))
        with open(os.path.join(args["dir"], f"rank{rank}.txt"), "w") as f:
            f.write(f"{rank} {world} {os.environ['LOCAL_RANK']} {ms}")
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_spawn_ranks_starts_one_process_per_rank(tmp_path):
    """The launch path bench.py takes for --gpus N outside torchrun."""
    import bench
    rc = bench.spawn_ranks(2, _spawned_target, {"dir": str(tmp_path)}, timeout_s=180)
    assert rc == 0
    got = sorted(open(tmp_path / f"rank{r}.txt").read().split() for r in range(2))
    assert got == [["0", "2", "0", "21.0"], ["1", "2", "1", "21.0"]]

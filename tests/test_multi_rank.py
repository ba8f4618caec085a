"""The N-GPU bench path is N independent replicas; its only cross-rank steps are the barrier
around the timed region and the max over ranks of the measured time.  Both run here as two
gloo ranks on the CPU (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        bench.barrier(world)
        mine = 1.5 + 2.0 * rank  # rank-specific "elapsed ms"
        results[rank] = bench.max_over_ranks(mine, world)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0, 0], codes
        assert dict(results) == {0: 3.5, 1: 3.5}


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(4.25, 1) == 4.25
    bench.barrier(1)  # no process group needed

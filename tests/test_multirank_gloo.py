"""The multi-process plumbing bench.py uses under torchrun, on CPU with the
gloo backend and two ranks: every rank runs its own replica (tokens add up
over ranks), the step time is the max over ranks, and the barrier holds."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 10.0 + 5.0 * rank
    total = bench.max_over_ranks(local_ms, world)
    bench.barrier(world)
    tokens = sum(bench.shard_tokens(4096, world))
    out[rank] = (total, tokens)
    dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        total, tokens = out[r]
        assert total == pytest.approx(15.0)      # the slowest rank's device time
        assert tokens == 2 * 4096                # weak scaling: a replica per rank

"""The N > 1 host path of the benchmark (independent replicas) exercised as
world_size-2 gloo process groups on CPU: barrier, max-over-ranks timing and
the whole-job throughput aggregate."""
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


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from video_vae_causal_implicit_b200 import replicas
    replicas.init("gloo", timeout_s=60)
    assert replicas.world() == world
    replicas.barrier()
    local_s = 0.010 * (rank + 1)          # rank 1 is the slowest
    slowest = replicas.max_over_ranks(local_s)
    thr = replicas.aggregate_throughput(100.0, local_s)
    seeds = replicas.replica_seed(7, rank)
    q.put((rank, slowest, thr, seeds))
    replicas.shutdown()


def test_two_rank_replicas_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, slowest, thr, seed in res:
        assert slowest == pytest.approx(0.020)
        assert thr == pytest.approx(2 * 100.0 / 0.020)
    assert res[0][3] != res[1][3]


def test_single_process_needs_no_group():
    from video_vae_causal_implicit_b200 import replicas
    assert replicas.world() == 1
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.aggregate_throughput(10.0, 2.0) == 5.0

"""Multi-process host logic of the benchmark on CPU (gloo, world size 2): the
timing reduction takes the slowest rank, and replicas draw distinct batches."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from mla_latent_space_lca_b200.inputs import make_decode_inputs
        t = bench.max_over_ranks(1.0 + 2.5 * rank, world)
        inp = make_decode_inputs(1, 64, seed=bench.replica_seed(rank))
        q.put((rank, t, float(inp.cache.float().sum())))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 2000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] == res[1][1] == pytest.approx(3.5)   # the slowest rank's value on both
    assert res[0][2] != res[1][2]                          # different batches per replica


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.0, 1) == 2.0

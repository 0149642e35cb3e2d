"""Multi-process host logic on CPU (gloo, world sizes 2 and 3): the timing
reduction takes the slowest rank, replicas draw distinct batches, and the
decode split along the cache gathers and merges every rank's shard record,
and a prefill split over query blocks reassembles the whole prefill (the
oracle stands in for the kernels)."""
import math
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
        from benchmarks import common
        from mla_latent_space_lca_b200.inputs import make_decode_inputs
        t = common.max_over_ranks(1.0 + 2.5 * rank, world)
        inp = make_decode_inputs(1, 64, seed=common.replica_seed(rank))
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
    from benchmarks import common
    assert common.max_over_ranks(2.0, 1) == 2.0


# ------------------------------------------------ decode split along the cache
def _oracle_shard_fn(cache_shard, q_recent, q, L, row0, g=16, w=1024, scale=None, ws=None):
    """Stand-in for lca_decode_shard on CPU: the oracle run on this rank's
    rows alone, packed into the library's shard record (o, then lse2)."""
    import numpy as np
    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits
    Ls = cache_shard.shape[1]
    w_loc = w if row0 + Ls == L else 0          # only the last shard holds the window
    o, lse, _ = oracle.lca_decode_shard(bf16_bits(cache_shard), bf16_bits(q_recent), bf16_bits(q),
                                        g, w_loc, scale, 0, Ls)
    rec = np.concatenate([o.ravel(), (lse / math.log(2.0)).ravel()])
    return torch.from_numpy(rec.astype(np.float32))


def _oracle_combine_fn(parts, w_uv, B, out=None):
    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits
    n = parts.shape[0]
    o = parts[:, : B * 16 * 512].double().numpy().reshape(n, B, 16, 512)
    lse = parts[:, B * 16 * 512:].double().numpy().reshape(n, B, 16) * math.log(2.0)
    return torch.from_numpy(oracle.combine_shards(o, lse, bf16_bits(w_uv))[1])


def _split_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mla_latent_space_lca_b200.inputs import make_decode_inputs
        from mla_latent_space_lca_b200.split_l import shard_bounds, split_l_decode
        inp = make_decode_inputs(2, 256 + 16 * 9 + 5, w=256, seed=41)
        row0, row1 = shard_bounds(inp.L, world, 16, 256)[rank]
        out = split_l_decode(inp.cache[:, row0:row1].contiguous(), inp.q_recent, inp.q, inp.w_uv,
                             inp.L, row0, w=256, scale=inp.scale, shard_fn=_oracle_shard_fn,
                             combine_fn=_oracle_combine_fn)
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_l_decode_gathers_and_merges_shards(world):
    """Each rank decodes its own rows of the cache, the shard records are
    all-gathered, and every rank's merge equals the unsplit decode."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() + world) % 2000
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = make_decode_inputs(2, 256 + 16 * 9 + 5, w=256, seed=41)
    _, ref, _ = oracle.lca_decode(bf16_bits(inp.cache), bf16_bits(inp.q_recent), bf16_bits(inp.q),
                                  bf16_bits(inp.w_uv), 16, 256, inp.scale)
    for _, out in res:   # float32 records: agreement to fp32 rounding
        np.testing.assert_allclose(out, ref, rtol=0, atol=2e-6)


def test_shard_bounds():
    sys.path.insert(0, ROOT)
    from mla_latent_space_lca_b200.split_l import shard_bounds
    for L, n, g, w in [(1 << 20, 8, 16, 1024), (4096 + 21, 3, 16, 1024), (1024 + 48, 4, 16, 1024),
                       (81, 5, 16, 0), (80, 5, 16, 0), (32768, 1, 16, 1024), (131072, 7, 16, 1024)]:
        b = shard_bounds(L, n, g, w)
        m = max(0, (L - w) // g)
        assert len(b) == n and b[0][0] == 0 and b[-1][1] == L
        for (a0, a1), (c0, _) in zip(b[:-1], b[1:]):
            assert a1 == c0 and a1 % g == 0 and a1 <= m * g   # whole groups, window in the last
        assert all(r1 > r0 for r0, r1 in b)
        rows = [r1 - r0 for r0, r1 in b]
        if m * g >= (n - 1) * (L // n):                       # balanced when the history allows
            assert max(rows) - min(rows) <= 2 * g
    assert shard_bounds(1 << 20, 8)[3] == (3 << 17, 4 << 17)
    with pytest.raises(ValueError):
        shard_bounds(1024 + 32, 4)      # two groups, four shards
    with pytest.raises(ValueError):
        shard_bounds(80, 6, 16, 0)      # five groups and no window row for a sixth shard


# ------------------------------------------------ prefill split over query blocks
def test_prefill_block_ranges():
    sys.path.insert(0, ROOT)
    from mla_latent_space_lca_b200.split_blocks import block_flops, prefill_block_ranges
    for L, n, w in [(131072, 8, 1024), (16384, 4, 1024), (2048, 3, 256), (4096 + 7, 5, 100), (64, 4, 0)]:
        r = prefill_block_ranges(L, n, w=w)
        assert len(r) == n and r[0][0] == 0 and sum(ql for _, ql in r) == 16 * (L // 16)
        for (s0, l0), (s1, _) in zip(r[:-1], r[1:]):
            assert s0 + l0 == s1 and l0 > 0 and s0 % 16 == 0 and l0 % 16 == 0
        work = [sum(block_flops(k, w=w) for k in range(s // 16, (s + ql) // 16)) for s, ql in r]
        if L // 16 >= 64 * n:      # enough blocks: balanced to a block's work
            assert max(work) - min(work) <= 2 * max(block_flops(k, w=w) for k in range(L // 16))
    with pytest.raises(ValueError):
        prefill_block_ranges(48, 4)


def _prefill_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from mla_latent_space_lca_b200.inputs import bf16_bits, make_prefill_inputs
        from mla_latent_space_lca_b200.split_blocks import prefill_block_ranges
        inp = make_prefill_inputs(1, 384, w=64, seed=51)
        qs, ql = prefill_block_ranges(384, world, w=64)[rank]
        _, out, _ = oracle.lca_prefill(bf16_bits(inp.cache), bf16_bits(inp.q), bf16_bits(inp.w_uv), qs, ql,
                                       16, 64, inp.scale, want_olat=False)
        rows = [None] * world
        dist.all_gather_object(rows, (qs, out))
        q.put((rank, rows))
    finally:
        dist.destroy_process_group()


def test_split_prefill_ranges_reassemble_the_full_prefill():
    """Each rank prefills its work-balanced range of query blocks (the oracle
    stands in for the kernels); the gathered rows equal one prefill of the
    whole prompt."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits, make_prefill_inputs
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 33500 + os.getpid() % 2000
    procs = [ctx.Process(target=_prefill_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = make_prefill_inputs(1, 384, w=64, seed=51)
    _, full, _ = oracle.lca_prefill(bf16_bits(inp.cache), bf16_bits(inp.q), bf16_bits(inp.w_uv), 0, 384,
                                    16, 64, inp.scale, want_olat=False)
    for _, rows in res:
        got = np.concatenate([out for _, out in sorted(rows, key=lambda x: x[0])], axis=1)
        np.testing.assert_allclose(got, full, rtol=0, atol=1e-12)

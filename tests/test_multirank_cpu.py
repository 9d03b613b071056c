"""The bench's N > 1 path on the CPU: two gloo ranks, each an independent shard.

Every rank builds its own block pool for the same schedule (replicas only: no
data-path collective), runs decode-step bookkeeping through libkvp's host
allocator, checks it against the oracle's, and combines its timing numbers with
the bench's max / sum reductions.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, q):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import paged_kv_cache_319_b200 as kvp
        from oracle.block_manager import BlockManager
        import workloads

        wl = workloads.opt13b(num_seqs=8, max_len=300)
        g = wl.geometry
        ctx = np.asarray(wl.info["context_lens"])
        pool = kvp.BlockPool(wl.num_blocks, g.block_size, g.num_kv_heads, g.head_dim, g.dtype,
                             wl.free_order)
        ora = BlockManager(wl.num_blocks, g.block_size, wl.free_order)
        seqs = np.array([pool.create() for _ in ctx], dtype=np.int64)
        oseqs = [ora.create() for _ in ctx]
        for s, o, L in zip(seqs, oseqs, ctx):
            assert pool.append(int(s), int(L) - 3) == ora.append(o, int(L) - 3)
        mb = int(-(-(ctx.max() + 3) // g.block_size))
        step_bytes = 0
        for _ in range(3):
            slots = pool.append_batch(seqs, 1)
            want = [ora.append(o, 1)[0] for o in oseqs]
            assert slots.tolist() == want
            tables, lens = pool.build_batch(seqs, mb)
            ot, ol = ora.build_batch(oseqs, mb)
            assert tables.tolist() == ot and lens.tolist() == ol
            step_bytes += bench.algorithmic_bytes(lens, g)
        total = bench.dist_sum(float(step_bytes), world)
        worst = bench.dist_max(float(rank + 1), world)
        seed = bench.shard_value_seed(wl.value_seed, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        q.put((rank, step_bytes, total, worst, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_independent_shards():
    world = 2
    port = free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    per_rank = [r[1] for r in results]
    assert per_rank[0] == per_rank[1] > 0                  # same schedule on both shards
    assert all(r[2] == sum(per_rank) for r in results)     # sum over ranks
    assert all(r[3] == world for r in results)             # max over ranks
    seeds = results[0][4]
    assert len(set(seeds)) == world                        # independent values per shard


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse

    import bench

    args = argparse.Namespace(workload="opt13b", warmup=3, steps=1, ref_seqs_per_step=1)
    bench.run_reference(args, world=2, rank=1)             # no work, no output
    assert capsys.readouterr().out == ""

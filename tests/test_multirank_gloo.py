"""World-size-2 checks of the multi-rank host logic on CPU (gloo).

1. Each rank of `bench.py --gpus N` takes its own tensor of the workload
   (weak scaling, no data exchange): shapes agree, contents differ, and
   rank 0 keeps the workload's own tensor.
2. The timing reduction is a max over ranks.
3. Row-sharding one tensor needs exactly one exchange, a max all-reduce of
   the tensor amax: per-rank amax -> all-reduce(MAX) -> per-rank NVFP4
   quantisation and scale search with that amax reproduce the unsharded
   result bit for bit.  The orchestration is bench.py's own (`shard_rows`
   for the row ranges, `sharded_step` for the order amax -> all-reduce ->
   the rest, as `bench.py --shard rows` runs it with fp4_tensor_amax and the
   fp4_*_with_amax entry points); the per-rank arithmetic here is the
   oracle's, standing in for the device calls.
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        import bench
        import oracle
        import workloads
        dist.init_process_group("gloo", rank=rank, world_size=world)
        # 1. per-rank tensors
        w = workloads.for_rank(workloads.with_shape(workloads.WEIGHT_4K, 64, 256), rank)
        x = workloads.generate(w)
        shapes = [None] * world
        dist.all_gather_object(shapes, (tuple(x.shape), float(x.float().sum())))
        # 2. max over ranks
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank], "cpu", world)
        # 3. row-sharded NVFP4 and scale search with one amax all-reduce,
        # through bench.py's orchestration
        full = workloads.generate(workloads.with_shape(workloads.ACT_8K, 97, 512))
        r0, r1 = bench.shard_rows(97, world, rank)
        local = workloads.as_oracle_array(full[r0:r1])
        calls = []

        def local_amax():
            calls.append("amax")
            return torch.tensor([oracle.tensor_amax(local)], dtype=torch.float32)

        def all_reduce_max(a):
            calls.append("all_reduce")
            dist.all_reduce(a, op=dist.ReduceOp.MAX)

        def rest(a):
            calls.append("rest")
            g = oracle.nv_global_scale(a.item())
            p, s = oracle.nvfp4_quantize_with_g(local, g)
            sp, ss, _ = oracle.nvfp4_scale_search_with_g(local, g)
            return p, s, g, sp, ss

        out = bench.sharded_step(local_amax, all_reduce_max, rest)
        assert calls == ["amax", "all_reduce", "rest"]
        parts = [None] * world
        dist.all_gather_object(parts, (r0, r1) + tuple(out))
        q.put((rank, shapes, got, parts if rank == 0 else None))
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e), None))


def test_two_ranks_gloo():
    import oracle
    import workloads
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, shapes, got, parts = q.get(timeout=240)
        assert shapes != "error", got
        res[r] = (shapes, got, parts)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shapes, got, parts = res[0]
    assert shapes[0][0] == shapes[1][0] and shapes[0][1] != shapes[1][1]
    w0 = workloads.with_shape(workloads.WEIGHT_4K, 64, 256)
    assert shapes[0][1] == float(workloads.generate(w0).float().sum())
    assert got == [2.0, 5.0] and res[1][1] == [2.0, 5.0]
    full = workloads.as_oracle_array(workloads.generate(workloads.with_shape(workloads.ACT_8K, 97, 512)))
    p, s, g = oracle.nvfp4_quantize(full)
    sp, ss, sg, _ = oracle.nvfp4_scale_search(full)
    # the shards tile the rows in order, the first one a row longer
    assert [pt[:2] for pt in parts] == [(0, 49), (49, 97)]
    assert parts[0][4] == parts[1][4] == g == sg
    assert np.array_equal(np.concatenate([parts[0][2], parts[1][2]]), p)
    assert np.array_equal(np.concatenate([parts[0][3], parts[1][3]]), s)
    assert np.array_equal(np.concatenate([parts[0][5], parts[1][5]]), sp)
    assert np.array_equal(np.concatenate([parts[0][6], parts[1][6]]), ss)
    # shard_rows tiles any row count for any world size
    import bench
    for rows in (0, 1, 7, 96, 97):
        for world in (1, 2, 3, 8):
            rs = [bench.shard_rows(rows, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            assert max(b - a for a, b in rs) - min(b - a for a, b in rs) <= 1

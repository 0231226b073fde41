"""Multi-process checks of the sharded path on CPU (gloo, world size 2).

Tokens are routed independently, so a batch split across ranks (each rank running
the layer on its own tokens with replicated weights) must reproduce the unsplit
layer; and the bench's step time is the max over ranks.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from oracle import moe_oracle as O
        from workloads import make_inputs, small

        inp = {k: v.double().numpy() for k, v in
               make_inputs(small("dist", T=50, d=32, h=48, seed=3), "cpu").items()}
        shard = np.array_split(np.arange(50), world)[rank]
        y_local = O.moe_layer(inp["x"][shard], inp["Wg"], inp["W1"], inp["W3"], inp["W2"])["y"]
        parts = [None] * world
        dist.all_gather_object(parts, y_local)
        m = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        if rank == 0:
            full = O.moe_layer(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"])["y"]
            q.put((np.max(np.abs(np.concatenate(parts) - full)), m))
        else:
            q.put((None, m))
    finally:
        dist.destroy_process_group()


def _bench_worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import bench
        from workloads import make_inputs, small

        r, w = bench.init_dist("gloo")  # the bench's own set-up path
        wl = small("replica", T=24, d=32, h=48, seed=9)
        inp = bench.rank_inputs(wl, r, w, "cpu")
        parts = [None] * w
        dist.all_gather_object(parts, {k: v.float().numpy() for k, v in inp.items()})
        m = bench.max_over_ranks(0.25 * (r + 1), w)
        bench.barrier(w)
        if r == 0:
            ref = {k: v.float().numpy() for k, v in make_inputs(wl, "cpu").items()}
            same_w = all(np.array_equal(p[k], ref[k]) for p in parts
                         for k in ("Wg", "W1", "W3", "W2"))
            x0_is_ref = np.array_equal(parts[0]["x"], ref["x"])
            x_differ = not np.array_equal(parts[0]["x"], parts[1]["x"])
            q.put((same_w, x0_is_ref, x_differ, m, r, w))
        else:
            q.put((True, True, True, m, r, w))
    except Exception as exc:
        q.put(repr(exc))
        raise
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_bench_replica_setup_on_two_ranks():
    """bench.py's replica path on two gloo ranks: init from the torchrun environment,
    every rank draws its own batch while the weights stay identical (rank 0's batch is
    the workload's own), and the step time is the max over ranks."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(isinstance(r, tuple) for r in res), res
    assert all(p.exitcode == 0 for p in procs)
    for same_w, x0_is_ref, x_differ, m, r, w in res:
        assert same_w and x0_is_ref and x_differ
        assert m == 0.5 and w == world


def test_token_shards_reproduce_the_full_batch_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    diffs = [r[0] for r in results if r[0] is not None]
    assert len(diffs) == 1 and diffs[0] <= 1e-12  # each token's output is independent
    assert all(r[1] == 3.0 for r in results)    # max over ranks of (1.5, 3.0)

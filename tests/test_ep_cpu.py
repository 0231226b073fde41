"""Expert parallelism on CPU: the transfer plan, and a world-size-2 gloo run of the
row exchange with the fp64 oracle standing in for the expert kernels.

Each rank routes and groups its own tokens, exchanges row counts, sends every
(destination, local expert) slice to its rank, runs its local experts on what arrives,
sends the outputs back and combines; the concatenated outputs must equal the
single-process layer over all tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plan_tiles_both_buffers():
    from sparse_mixture_experts_26_b200.ep import plan_transfers
    rng = np.random.default_rng(0)
    for N, El in ((1, 1), (2, 2), (4, 2), (3, 3), (8, 1)):
        send = rng.integers(0, 5, size=(N, El)).tolist()
        recv = rng.integers(0, 5, size=(N, El)).tolist()
        for rank in range(N):
            p = plan_transfers(send, recv, rank)
            # send slices tile the grouped rows in (destination, local expert) order
            at = 0
            for (dst, j, s, n), (dst2, j2) in zip(p.sends, [(a, b) for a in range(N)
                                                            for b in range(El)]):
                assert (dst, j) == (dst2, j2) and s == at and n == send[dst][j]
                at += n
            # receive slices tile the buffer: local expert major, sources in rank order
            at = 0
            for (src, j, s, n), (j2, src2) in zip(p.recvs, [(b, a) for b in range(El)
                                                            for a in range(N)]):
                assert (src, j) == (src2, j2) and s == at and n == recv[src][j]
                at += n
            assert at == p.received == p.local_offsets[-1]
            for j in range(El):
                assert p.local_offsets[j + 1] - p.local_offsets[j] == sum(
                    recv[s][j] for s in range(N))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, E, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import moe_oracle as O
        from sparse_mixture_experts_26_b200.ep import (exchange_counts, plan_transfers,
                                                       run_transfers)
        from workloads import make_inputs, small

        T_all = 57
        inp = {k: v.double().numpy() for k, v in
               make_inputs(small("ep", T=T_all, d=16, h=24, E=E, seed=11,
                                 kind="skew" if E == 8 else "plain"), "cpu").items()}
        El = E // world
        shard = np.array_split(np.arange(T_all), world)[rank]  # unequal shard sizes
        x = inp["x"][shard]
        logits = O.router_logits(x, inp["Wg"])
        idx = O.top2_select(logits)
        w = O.gate_weights(logits, idx)
        offsets, perm_token, inv_perm = O.permutation(idx, E)
        x_perm = torch.from_numpy(O.gather_rows(x, perm_token))
        counts = torch.from_numpy(np.diff(offsets).astype(np.int64)).view(world, El)
        recv_counts = exchange_counts(counts)
        plan = plan_transfers(counts.tolist(), recv_counts.tolist(), rank)
        x_recv = torch.zeros(plan.received, x.shape[1], dtype=torch.float64)
        run_transfers(plan, rank, x_perm, x_recv)
        # the local experts (the oracle stands in for the expert kernels)
        Y_recv = torch.zeros_like(x_recv)
        for j in range(El):
            lo, hi = plan.local_offsets[j], plan.local_offsets[j + 1]
            if hi > lo:
                e = rank * El + j
                Y_recv[lo:hi] = torch.from_numpy(O.expert_swiglu(
                    x_recv[lo:hi].numpy(), inp["W1"][e], inp["W3"][e], inp["W2"][e]))
        Y_perm = torch.zeros(x_perm.shape, dtype=torch.float64)
        run_transfers(plan, rank, Y_recv, Y_perm, reverse=True)
        y = O.combine(Y_perm.numpy(), inv_perm, w)
        parts = [None] * world
        dist.all_gather_object(parts, y)
        if rank == 0:
            full = O.moe_layer(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"])["y"]
            q.put(float(np.max(np.abs(np.concatenate(parts) - full))))
        else:
            q.put(0.0)
    except Exception as exc:  # report instead of leaving the parent waiting
        q.put(repr(exc))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("E", [2, 4, 8])
def test_two_ranks_reproduce_the_whole_layer(E):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, E, q)) for r in range(world)]
    for p in procs:
        p.start()
    errs = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(isinstance(e, float) for e in errs), errs
    assert all(p.exitcode == 0 for p in procs)
    assert max(errs) <= 1e-12, errs


class OracleSteps:
    """The four layer steps written with the fp64 oracle, on CPU tensors, standing in
    for libmoe's kernels so that ExpertParallelMoE.forward's own planning and transfer
    code runs on gloo ranks.  Outputs are stored in the tensors' dtypes (float32)."""

    @staticmethod
    def route(x, Wg, idx, w):
        from oracle import moe_oracle as O
        logits = O.router_logits(x.double().numpy(), Wg.double().numpy())
        i = O.top2_select(logits)
        idx.copy_(torch.from_numpy(i))
        w.copy_(torch.from_numpy(O.gate_weights_f32(logits, i)))

    @staticmethod
    def permute(idx, x, offsets, perm_token, inv_perm, x_perm, ws, E):
        from oracle import moe_oracle as O
        off, pt, inv = O.permutation(idx.numpy(), E)
        offsets.copy_(torch.from_numpy(off))
        perm_token.copy_(torch.from_numpy(pt))
        inv_perm.copy_(torch.from_numpy(inv))
        x_perm.copy_(torch.from_numpy(O.gather_rows(x.numpy(), pt)))

    @staticmethod
    def expert_ffn(x_rows, offsets, W1, W3, W2, Y, ws):
        from oracle import moe_oracle as O
        off = offsets.numpy()
        n = int(off[-1])  # a padding row past the last group belongs to no expert
        Y[:n] = torch.from_numpy(O.expert_ffn_grouped(
            x_rows[:n].double().numpy(), off, W1.double().numpy(), W3.double().numpy(),
            W2.double().numpy())).to(Y.dtype)

    @staticmethod
    def combine(Y, inv_perm, w, y):
        from oracle import moe_oracle as O
        y.copy_(torch.from_numpy(O.combine(Y.double().numpy(), inv_perm.numpy(),
                                           w.double().numpy())).to(y.dtype))


def _forward_worker(rank, world, port, E, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import moe_oracle as O
        from sparse_mixture_experts_26_b200.ep import ExpertParallelMoE
        from tests.test_ep_cpu import OracleSteps
        from workloads import make_inputs, small

        T_all = 61
        inp = make_inputs(small("epf", T=T_all, d=16, h=24, E=E, seed=19, dtype="f32",
                                kind="skew" if E == 8 else "plain"), "cpu")
        El = E // world
        shard = np.array_split(np.arange(T_all), world)[rank]
        layer = ExpertParallelMoE(inp["Wg"], inp["W1"][rank * El:(rank + 1) * El].contiguous(),
                                  inp["W3"][rank * El:(rank + 1) * El].contiguous(),
                                  inp["W2"][rank * El:(rank + 1) * El].contiguous(),
                                  steps=OracleSteps)
        routing = {}
        y = layer.forward(inp["x"][shard].contiguous(), routing).double().numpy()
        parts = [None] * world
        dist.all_gather_object(parts, (y, routing["idx"].numpy()))
        if rank == 0:
            c = {k: v.double().numpy() for k, v in inp.items()}
            ref = O.moe_layer(c["x"], c["Wg"], c["W1"], c["W3"], c["W2"])
            y_all = np.concatenate([p[0] for p in parts])
            idx_all = np.concatenate([p[1] for p in parts])
            same_idx = bool((idx_all == ref["idx"]).all())
            err = float(np.linalg.norm(y_all - ref["y"]) / np.linalg.norm(ref["y"]))
            q.put((same_idx, err))
        else:
            q.put((True, 0.0))
    except Exception as exc:  # report instead of leaving the parent waiting
        q.put(repr(exc))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("E", [2, 8])
def test_two_ranks_drive_expert_parallel_forward(E):
    """ExpertParallelMoE.forward end to end on two gloo ranks (count exchange, plan,
    dispatch, local experts, return, combine), with the oracle's steps injected in
    place of the kernels: routing is bit-exact and y matches the whole-batch oracle
    to float32 rounding (the steps store w, Y and y in float32)."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_forward_worker, args=(r, world, port, E, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(isinstance(r, tuple) for r in res), res
    assert all(p.exitcode == 0 for p in procs)
    assert all(r[0] for r in res)
    assert max(r[1] for r in res) <= 1e-6, res

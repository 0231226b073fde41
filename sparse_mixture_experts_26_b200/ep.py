"""Expert parallelism: each rank holds E / N of the experts, and every (token, slot) row
travels to the rank of its expert and back.

notion notes "Mixtral of Experts", "Expert Parallelism": tokens are routed to the
device that holds the chosen expert and its output is returned to the token's
original location; ml-canon "52 Mixtral", "Questions worth asking", and crackai
"Mixtral of Experts", "Key Takeaways": that exchange is an all-to-all.

Experts are numbered so that rank r owns experts [r * El, (r + 1) * El), El = E / N.
One layer call on every rank:

1. route and group the rank's own tokens by expert (libmoe ``moe_route``,
   ``moe_permute``): the grouped rows are then ordered by destination rank, then by
   the destination's local expert;
2. exchange the row counts: rank r learns, for each source rank s and local expert j,
   how many rows s sends for expert r * El + j (``exchange_counts``);
3. dispatch: every (destination, local expert) slice of the grouped rows goes to its
   rank, where it lands in the local expert's region, sources in rank order, so each
   local expert's rows arrive contiguous (``plan_transfers`` + ``run_transfers``);
4. run the local experts on the received rows (libmoe ``moe_expert_ffn``);
5. return the fp32 expert outputs along the same transfers reversed;
6. weight and add each token's two outputs in its original order (``moe_combine``).

The transfers use ``torch.distributed`` point-to-point operations issued as one
batch (NCCL on GPUs; gloo works for the host-side tests), with a rank's rows for its
own experts copied locally.  Steps 2-5 need the per-expert row counts on the host,
so a layer call synchronises once after the permutation.  The arithmetic of every
step runs in libmoe's kernels; this module only plans and moves rows.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

__all__ = ["TransferPlan", "plan_transfers", "exchange_counts", "run_transfers",
           "LibmoeSteps", "ExpertParallelMoE"]


@dataclass
class TransferPlan:
    """Row slices of one dispatch (the return runs the same slices reversed).

    ``sends``: (peer, local expert j, start, rows) slices of the grouped rows;
    ``recvs``: (peer, local expert j, start, rows) slices of the receive buffer;
    ``local_offsets``: El + 1 group offsets of the received rows, by local expert;
    ``received``: total rows received.
    """
    sends: list
    recvs: list
    local_offsets: list
    received: int


def plan_transfers(send_counts, recv_counts, rank: int) -> TransferPlan:
    """Plan a dispatch from row counts (plain integers, host side).

    ``send_counts[dst][j]``: rows this rank sends for expert dst * El + j, which are
    consecutive in its grouped rows in (dst, j) order; ``recv_counts[src][j]``: rows it
    receives from rank src for its local expert j.  The receive buffer holds local
    expert 0's rows from source 0, 1, ..., then local expert 1's, and so on.
    """
    N = len(send_counts)
    El = len(send_counts[0]) if N else 0
    sends, start = [], 0
    for dst in range(N):
        for j in range(El):
            n = int(send_counts[dst][j])
            sends.append((dst, j, start, n))
            start += n
    local_offsets, total = [0], 0
    for j in range(El):
        total += sum(int(recv_counts[src][j]) for src in range(N))
        local_offsets.append(total)
    recvs = []
    for j in range(El):
        at = local_offsets[j]
        for src in range(N):
            n = int(recv_counts[src][j])
            recvs.append((src, j, at, n))
            at += n
    return TransferPlan(sends=sends, recvs=recvs, local_offsets=local_offsets, received=total)


def exchange_counts(send_counts: torch.Tensor, group=None) -> torch.Tensor:
    """All-to-all of the [N, El] row-count matrix: row dst goes to rank dst; the result's
    row src holds what rank src sends to this rank.  Counts live on the host (int64)."""
    send = send_counts.to(torch.int64).contiguous()
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return send.clone()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv


def run_transfers(plan: TransferPlan, rank: int, src_rows: torch.Tensor,
                  dst_rows: torch.Tensor, reverse: bool = False, group=None) -> None:
    """Move rows along ``plan``: forward, ``src_rows`` are the grouped rows and
    ``dst_rows`` the receive buffer; with ``reverse``, ``src_rows`` is the receive-side
    buffer and ``dst_rows`` the grouped layout.  Slices for this rank itself are copied
    locally; all others go out as one batch of point-to-point operations."""
    # pair each send slice (dst, j) with the matching receive slice on the peer:
    # forward, this rank's send (dst, j) lands in dst's recv (me, j); its recv (src, j)
    # comes from src's send (me, j).
    sends = {(p, j): (s, n) for p, j, s, n in plan.sends}
    recvs = {(p, j): (s, n) for p, j, s, n in plan.recvs}
    out_slices, in_slices = (recvs, sends) if reverse else (sends, recvs)
    ops = []
    for (peer, j), (s, n) in sorted(out_slices.items()):
        if n == 0:
            continue
        if peer == rank:
            d0, dn = in_slices[(rank, j)]
            assert dn == n, "local slice sizes disagree"
            dst_rows[d0:d0 + n].copy_(src_rows[s:s + n])
        else:
            ops.append(dist.P2POp(dist.isend, src_rows[s:s + n], peer, group=group))
    for (peer, j), (s, n) in sorted(in_slices.items()):
        if n == 0 or peer == rank:
            continue
        ops.append(dist.P2POp(dist.irecv, dst_rows[s:s + n], peer, group=group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


class LibmoeSteps:
    """The four layer steps an expert-parallel call runs, as libmoe's kernels."""

    @staticmethod
    def route(x, Wg, idx, w):
        from . import moe_route
        moe_route(x, Wg, idx, w)

    @staticmethod
    def permute(idx, x, offsets, perm_token, inv_perm, x_perm, ws, E):
        from . import moe_permute
        moe_permute(idx, x, offsets, perm_token, inv_perm, x_perm, ws, E)

    @staticmethod
    def expert_ffn(x_rows, offsets, W1, W3, W2, Y, ws):
        from . import moe_expert_ffn
        moe_expert_ffn(x_rows, offsets, W1, W3, W2, Y, ws)

    @staticmethod
    def combine(Y, inv_perm, w, y):
        from . import moe_combine
        moe_combine(Y, inv_perm, w, y)


class ExpertParallelMoE:
    """One layer with its experts spread over the ranks of ``group``.

    Every rank passes the full router ``Wg [d, E]`` and the weights of its own experts
    (``W1_local, W3_local [El, h, d]``, ``W2_local [El, d, h]``; rank r holds experts
    r * El .. r * El + El - 1).  bf16 layers (the libmoe expert kernels); CUDA tensors.
    ``steps`` replaces the four layer steps (route, permute, expert_ffn, combine;
    default: libmoe's kernels) -- a test hook, so that the planning and transfer code
    can be driven on CPU ranks with reference steps in place of the kernels.
    """

    def __init__(self, Wg, W1_local, W3_local, W2_local, group=None, steps=None):
        from . import alloc_workspace  # noqa: F401  (the package loads libmoe)
        self.steps = LibmoeSteps if steps is None else steps
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.Wg, self.W1, self.W3, self.W2 = Wg, W1_local, W3_local, W2_local
        self.E = Wg.shape[1]
        self.El, self.h, self.d = W1_local.shape
        if self.E != self.El * self.world:
            raise ValueError(f"{self.E} experts do not split into {self.world} x {self.El}")
        self._ws = {}

    def _workspace(self, T: int, x: torch.Tensor) -> torch.Tensor:
        from . import moe_workspace_bytes
        need = moe_workspace_bytes(T, self.d, self.h, self.E, 2, x.dtype)
        ws = self._ws.get("ws")
        if ws is None or ws.numel() < need:
            ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
            self._ws["ws"] = ws
        return ws

    def forward(self, x: torch.Tensor, routing: dict | None = None) -> torch.Tensor:
        """The layer on this rank's tokens ``x [T, d]``; returns ``y [T, d]``.  If a dict
        is passed as ``routing``, it receives this rank's ``idx``, ``w``, ``offsets``,
        ``perm_token`` and ``inv_perm``."""
        st = self.steps
        T, d = x.shape
        dev = x.device
        E, El, N = self.E, self.El, self.world
        idx = torch.empty(T, 2, dtype=torch.int32, device=dev)
        w = torch.empty(T, 2, dtype=torch.float32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm_token = torch.empty(2 * T, dtype=torch.int32, device=dev)
        inv_perm = torch.empty(T, 2, dtype=torch.int32, device=dev)
        x_perm = torch.empty(2 * T, d, dtype=x.dtype, device=dev)
        ws = self._workspace(max(T, 1), x)
        if T > 0:
            st.route(x, self.Wg, idx, w)
        st.permute(idx, x, offsets, perm_token, inv_perm, x_perm, ws, E)
        counts = (offsets[1:] - offsets[:-1]).to(torch.int64).cpu().view(N, El)
        recv_counts = exchange_counts(counts, self.group)
        plan = plan_transfers(counts.tolist(), recv_counts.tolist(), self.rank)
        # the expert FFN takes an even row count; a padding row belongs to no group
        rows = plan.received + (plan.received & 1)
        x_recv = torch.empty(rows, d, dtype=x.dtype, device=dev)
        run_transfers(plan, self.rank, x_perm, x_recv, group=self.group)
        Y_recv = torch.empty(rows, d, dtype=torch.float32, device=dev)
        if plan.received > 0:
            local_off = torch.tensor(plan.local_offsets, dtype=torch.int32, device=dev)
            st.expert_ffn(x_recv, local_off, self.W1, self.W3, self.W2, Y_recv,
                          self._ffn_workspace(rows, x))
        Y_perm = torch.empty(2 * T, d, dtype=torch.float32, device=dev)
        run_transfers(plan, self.rank, Y_recv, Y_perm, reverse=True, group=self.group)
        y = torch.empty_like(x)
        if T > 0:
            st.combine(Y_perm, inv_perm, w, y)
        if routing is not None:
            routing.update(idx=idx, w=w, offsets=offsets, perm_token=perm_token,
                           inv_perm=inv_perm)
        return y

    def _ffn_workspace(self, rows: int, x: torch.Tensor) -> torch.Tensor:
        """Workspace for the local expert FFN over `rows` (even) received rows: rows / 2
        plays the part of T in the size formula, El that of E."""
        from . import moe_expert_ffn_workspace_bytes
        need = moe_expert_ffn_workspace_bytes(rows, self.d, self.h, self.El, x.dtype)
        ws = self._ws.get("ffn")
        if ws is None or ws.numel() < need:
            ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
            self._ws["ffn"] = ws
        return ws

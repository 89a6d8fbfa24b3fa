"""One rank of a real expert-parallel group: the per-rank form of `Buffer`.

On R GPUs each rank holds only its own router output (MoonEP README,
"dispatch fwd": `tokens_per_expert` is the rank's local count), and the
dispatched buffers of the R ranks live on R devices.  The planner needs, besides
the rank's picks, every rank's counts: one all-gather of R x E int32
(`gather_counts`), after which every rank derives the same layout and writes
the slots of its own picks (`moonep_plan_rank`).  Dispatch and combine address
the R ranks' buffers through a table of their device pointers
(`moonep_dispatch_rank`, `moonep_combine_rank`); the weight prefetch reads
each slot's expert from its home rank, and the grad reduction of a home rank
reads and zeroes the slots of every rank (`moonep_prefetch_weight_rank`,
`moonep_reduce_grad_rank`).

`RankBuffer` takes those buffers as a list of R entries: tensors, or device
pointers of the peers' memory.  With one process per rank, `IpcPeers` maps
the other ranks' buffers into this process (CUDA IPC, through the library's
moonep_ipc_export / moonep_ipc_import) and gives the tables; the ranks may
share one GPU or sit on several GPUs of a node.  Within one process, R
separate local allocations stand in for the ranks.  Argument marshalling
only: every step runs in the library's kernels, and the gathers are
torch.distributed collectives of the caller's process group.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moonep


def gather_counts(tokens_per_expert: torch.Tensor, group=None) -> torch.Tensor:
    """[R, E] int32: row q = rank q's tokens_per_expert [E], in group rank
    order, identical on every rank (one all-gather)."""
    if tokens_per_expert.dim() != 1 or tokens_per_expert.dtype != torch.int32:
        raise ValueError("tokens_per_expert: expected an [E] int32 tensor")
    world = dist.get_world_size(group)
    rows = [torch.empty_like(tokens_per_expert) for _ in range(world)]
    dist.all_gather(rows, tokens_per_expert.contiguous(), group=group)
    return torch.stack(rows)


class IpcPeers:
    """This rank's tensors, shared with the other ranks of `group` (one
    process per rank).  Every rank exports the allocation behind each of its
    tensors, the exports are all-gathered over the group (pickled bytes: a
    gloo group, or any group that can gather objects), and every rank maps
    the others' into this process.  `table(i)` lists tensor i of every rank,
    in group rank order: this rank's own tensor at its own index, the peers'
    as device pointers.  Tensor i must have the same shape and dtype on every
    rank.  `close()` releases the mappings once no kernel uses them."""

    def __init__(self, tensors, group=None):
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.tensors = list(tensors)
        mine = [moonep.moonep_ipc_export(t) for t in self.tensors]
        every = [None] * self.world
        dist.all_gather_object(every, mine, group=group)
        self._imports = []
        self.rows = []
        for q in range(self.world):
            if q == self.rank:
                self.rows.append(list(self.tensors))
                continue
            if len(every[q]) != len(self.tensors):
                raise ValueError(f"rank {q} shared {len(every[q])} tensors, this rank {len(self.tensors)}")
            row = []
            for blob in every[q]:
                ptr = moonep.moonep_ipc_import(blob)
                self._imports.append(ptr)
                row.append(ptr)
            self.rows.append(row)

    def table(self, i: int):
        """Tensor i of every rank, in rank order (tensors or device pointers)."""
        return [self.rows[q][i] for q in range(self.world)]

    def close(self) -> None:
        for ptr in self._imports:
            moonep.moonep_ipc_close(ptr)
        self._imports = []


class RankBuffer:
    """Rank `rank` of an EP group of `num_ep_ranks`: S tokens, hidden size H,
    top-K over E experts, B prefetch slots.

    `hidden_nvs`: the R ranks' dispatched buffers, a list of R [NvS, H] bf16
    tensors or device pointers (entry `rank` is this rank's own; e.g.
    `IpcPeers.table`); `route_weights_nvs` the same for the [NvS] fp32
    weights, or None.  NvS is `self.nvs`, known before any buffer exists
    (`RankBuffer.nvs_of`)."""

    def __init__(self, S: int, H: int, K: int, E: int, num_ep_ranks: int, rank: int, hidden_nvs,
                 route_weights_nvs=None, token_padding: int = 128, B: int | None = None,
                 mode: int = moonep.TRAINING, num_sms: int | None = None):
        if not 0 <= rank < num_ep_ranks:
            raise ValueError(f"rank {rank} outside [0, {num_ep_ranks})")
        self.handle = moonep.moonep_create(S, H, K, E, num_ep_ranks, B, token_padding, num_sms or 0, mode)
        self.rank, self.R = rank, num_ep_ranks
        self.S, self.H, self.K, self.E, self.B = S, H, K, E, self.handle.B
        self.nvs = self.handle.nvs
        # checked and marshalled once: the per-layer calls pass the tables
        self.hidden_nvs = moonep.PeerTable(hidden_nvs, (self.nvs, H), torch.bfloat16, "hidden_nvs[q]")
        self.route_weights_nvs = None if route_weights_nvs is None else moonep.PeerTable(
            route_weights_nvs, (self.nvs,), torch.float32, "route_weights_nvs[q]")

    @staticmethod
    def nvs_of(S: int, K: int, E: int, num_ep_ranks: int, token_padding: int = 128) -> int:
        """Slots of one rank's buffer, as moonep_nvs computes them."""
        G, tp = E // num_ep_ranks, token_padding
        n = S * K + 2 * G * (tp - 1)
        return (n + tp - 1) // tp * tp

    def plan(self, topk, tokens_per_expert=None, *, counts_all=None, group=None) -> moonep.Plan:
        """This rank's plan from its picks topk [S,K] and the gathered counts:
        `counts_all` [R,E] when the caller has it, else gathered here from
        `tokens_per_expert` [E] over `group`."""
        if counts_all is None:
            if tokens_per_expert is None:
                raise ValueError("plan needs tokens_per_expert or counts_all")
            counts_all = gather_counts(tokens_per_expert, group)
        return moonep.moonep_plan_rank(self.handle, self.rank, topk, counts_all)

    def dispatch(self, plan: moonep.Plan, hidden, route_weights=None):
        """Scatter this rank's rows hidden [S,H] (route_weights [S,K]) into
        the R ranks' buffers.  The receivers may read their buffer once every
        rank's dispatch has completed (a barrier of the caller's group)."""
        w_nvs = self.route_weights_nvs if route_weights is not None else None
        moonep.moonep_dispatch_rank(self.handle, plan, hidden, route_weights, self.hidden_nvs, w_nvs)

    def combine(self, plan: moonep.Plan, expert_out_nvs=None, weighted: bool = True, out=None):
        """out [S,H] = bf16(sum_k w_k * y[slot of (t,k)]) over this rank's
        tokens, reading `expert_out_nvs` (the R ranks' [NvS,H] outputs: a list
        or a moonep.PeerTable; None reads the dispatch buffers themselves)
        and, when weighted, the route weights that dispatch placed.  Returns
        (out, gathered_weights [S,K] or None)."""
        w_nvs = self.route_weights_nvs if weighted else None
        if weighted and w_nvs is None:
            raise ValueError("weighted combine needs route_weights_nvs")
        y = self.hidden_nvs if expert_out_nvs is None else expert_out_nvs
        return moonep.moonep_combine_rank(self.handle, plan, y, w_nvs, out)

    def prefetch_weight(self, plan: moonep.Plan, home_weights, pools) -> None:
        """pools[p] [B,H,H'] bf16 (this rank's slots) <- each slot's expert,
        read from its home rank: home_weights[p][q] is rank q's [G,H,H'] bf16
        home experts of projection p."""
        moonep.moonep_prefetch_weight_rank(self.handle, plan, self.rank, home_weights, pools)

    def reduce_grad(self, plan: moonep.Plan, grads, reduce_buffers) -> None:
        """grads[p] [G,H,H'] fp32 (this rank's home experts) += every rank's
        slots holding them, in (rank, slot) order; those slots are zeroed.
        reduce_buffers[p][q] is rank q's [B,H,H'] fp32 slots."""
        moonep.moonep_reduce_grad_rank(self.handle, plan, self.rank, grads, reduce_buffers)

    def destroy(self) -> None:
        if self.handle is not None:
            self.handle.close()
            self.handle = None

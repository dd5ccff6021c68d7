"""Expert-parallel routed MoE FFN layer over G ranks (one process per GPU).

Rank g owns experts ``[g*E/G, (g+1)*E/G)``.  One layer step on every rank:

1. ``dispatch``: the routed rows sorted by owner rank (stable in the routed
   row r = t*top_k + j), their input rows packed, with their local expert ids,
   and the per-owner row counts (the library's ``moe_ep_dispatch``);
2. the counts, then the rows and ids, go to their owners (all-to-all);
3. ``experts``: each owner runs its experts on the rows it received, giving
   the unweighted per-slot rows d (the library's ``moe_ffn_slots``, slotted
   layout, one slot per row);
4. d goes back to the home ranks (the reverse all-to-all);
5. ``combine``: ``y[t] = sum_j fl(w[t,j] * d[t,j])`` in slot order (the
   library's ``moe_ep_combine``) -- the same arithmetic as the single-rank
   layer's weighted epilogue and ordered combine, so the bits agree whenever
   the owners run the kernels the single-rank call would run on those rows.

The exchange is the only step outside the library: ``TorchComm`` uses
``torch.distributed.all_to_all_single`` (NCCL between GPUs); ``SelfComm`` is
the single-rank case.  The device steps
come from an ``ops`` object; ``CudaEpOps`` binds them to the library, and
there is no other implementation in the package (no fallback: a missing
library raises).  The pages run every expert on one device; this split is
not on them.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (SHARED_PER_TOKEN, SLOTTED, moe_ep_combine, moe_ep_dispatch, moe_ffn_slots,
               moe_ffn_workspace)


@dataclass
class EpPlan:
    """One step's dispatch result on one rank."""
    send_x: torch.Tensor        # [R, hidden] bf16 rows in send order
    send_expert: torch.Tensor   # [R] int32 local expert id of each sent row
    send_counts: list           # host ints: rows for each rank
    state: object               # what the combine needs (the dispatch workspace)


class CudaEpOps:
    """The device steps of an expert-parallel layer, on this library's kernels."""

    def dispatch(self, x, ids, n_experts: int, n_ranks: int, layout: int) -> EpPlan:
        send_x, send_expert, counts, ws = moe_ep_dispatch(x, ids, n_experts, n_ranks, layout)
        # the split sizes of the all-to-all are host values
        return EpPlan(send_x, send_expert, [int(c) for c in counts.cpu().tolist()], ws)

    def experts(self, recv_x, recv_expert, W_gate, W_up, W_down):
        n = recv_x.shape[0]
        if n == 0:
            return torch.empty((0, W_down.shape[1]), dtype=torch.float32, device=recv_x.device)
        E_loc, inter, hidden = W_gate.shape
        ws = torch.empty(moe_ffn_workspace(n, hidden, inter, 1, E_loc, SLOTTED),
                         dtype=torch.uint8, device=recv_x.device)
        d = moe_ffn_slots(recv_x.view(n, 1, hidden), recv_expert.view(n, 1), W_gate, W_up, W_down,
                          layout=SLOTTED, ws=ws)
        return d.view(n, hidden)

    def combine(self, d_back, weights, n_ranks: int, plan: EpPlan):
        return moe_ep_combine(d_back, weights, n_ranks, plan.state)

    def empty_rows(self, like, rows: int):
        return torch.empty((rows,) + tuple(like.shape[1:]), dtype=like.dtype, device=like.device)


class TorchComm:
    """All-to-all over a torch.distributed process group (NCCL between GPUs,
    gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def exchange_counts(self, send_counts: list, device) -> list:
        """send_counts[g] rows go to rank g; returns the rows each rank sends here."""
        s = torch.tensor(send_counts, dtype=torch.int64, device=device)
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        return [int(v) for v in r.cpu().tolist()]

    def all_to_all(self, out, inp, out_splits: list, in_splits: list):
        self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        return out


class SelfComm:
    """The exchange of a single rank (G = 1): every row stays here."""
    rank = 0
    world = 1

    def exchange_counts(self, send_counts: list, device) -> list:
        return list(send_counts)

    def all_to_all(self, out, inp, out_splits: list, in_splits: list):
        out.copy_(inp)
        return out


def ep_moe_forward(x, ids, weights, W_gate_local, W_up_local, W_down_local, n_experts: int,
                   comm, layout: int = SHARED_PER_TOKEN, ops=None):
    """One expert-parallel layer step on this rank: returns y [m, hidden] f32
    for this rank's m tokens.  ``W_*_local`` are this rank's E/G experts
    (rank g: experts g*E/G ... (g+1)*E/G - 1 of the full stack)."""
    ops = CudaEpOps() if ops is None else ops
    G = comm.world
    if n_experts % G:
        raise ValueError(f"n_experts ({n_experts}) must be a multiple of the world size ({G})")
    if W_gate_local.shape[0] != n_experts // G:
        raise ValueError("W_gate_local must hold n_experts / world_size experts")
    plan = ops.dispatch(x, ids, n_experts, G, layout)
    recv_counts = comm.exchange_counts(plan.send_counts, plan.send_expert.device)
    n_recv = sum(recv_counts)
    recv_x = comm.all_to_all(ops.empty_rows(plan.send_x, n_recv), plan.send_x, recv_counts,
                             plan.send_counts)
    recv_expert = comm.all_to_all(ops.empty_rows(plan.send_expert, n_recv), plan.send_expert,
                                  recv_counts, plan.send_counts)
    d = ops.experts(recv_x, recv_expert, W_gate_local, W_up_local, W_down_local)
    d_back = comm.all_to_all(ops.empty_rows(d, sum(plan.send_counts)), d, plan.send_counts,
                             recv_counts)
    return ops.combine(d_back, weights, G, plan)

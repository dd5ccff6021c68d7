"""Test-side pieces of the expert-parallel tests (test infrastructure).

``NumpyEpOps`` runs the device steps of an expert-parallel layer step on the
CPU from their plain definitions -- a stable sort of the routed rows by owner
rank, the oracle's f64 SwiGLU expert per received row (rounded once to f32),
and the weighted slot-order f32 sum -- so that multi-process CPU ranks (gloo)
can drive the same orchestration code (``ep.ep_moe_forward``) as the GPU.
``LoopbackComm`` exchanges rows between G ranks emulated as threads of one
process (one GPU): a barrier, then each rank gathers the slices addressed to
it; no kernel ever waits on another.
"""
import threading

import numpy as np
import torch

from mixture_experts_routed_sigmoid_b200.ep import EpPlan


class NumpyEpOps:
    def __init__(self, oracle_mod):
        self.oracle = oracle_mod

    def dispatch(self, x, ids, n_experts, n_ranks, layout):
        idsn = ids.numpy().astype(np.int64)
        m, top_k = idsn.shape
        hidden = x.shape[-1]
        per = n_experts // n_ranks
        flat = idsn.reshape(-1)
        owner = flat // per
        perm = np.argsort(owner, kind="stable")
        src = perm if layout else perm // top_k
        send_x = x.reshape(-1, hidden)[torch.from_numpy(src)].contiguous()
        send_e = (flat[perm] - owner[perm] * per).astype(np.int32)
        counts = np.bincount(owner, minlength=n_ranks).astype(np.int64)
        inv = np.empty(len(perm), np.int64)
        inv[perm] = np.arange(len(perm))
        return EpPlan(send_x, torch.from_numpy(send_e), counts.tolist(), inv)

    def experts(self, recv_x, recv_expert, W_gate, W_up, W_down):
        n, hidden = recv_x.shape
        if n == 0:
            return torch.empty((0, hidden), dtype=torch.float32)
        bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
        d = self.oracle.ffn(bits(recv_x).reshape(n, 1, hidden),
                            recv_expert.numpy().reshape(n, 1), np.ones((n, 1), np.float32),
                            bits(W_gate), bits(W_up), bits(W_down), layout=1)
        return torch.from_numpy(d.astype(np.float32))

    def combine(self, d_back, weights, n_ranks, plan):
        d = d_back.numpy()
        w = weights.numpy()
        m, top_k = w.shape
        y = np.zeros((m, d.shape[1]), np.float32)
        for t in range(m):
            acc = None
            for j in range(top_k):
                q = np.float32(w[t, j]) * d[plan.state[t * top_k + j]]
                acc = q if acc is None else (acc + q).astype(np.float32)
            y[t] = acc
        return torch.from_numpy(y)

    def empty_rows(self, like, rows):
        return torch.empty((rows,) + tuple(like.shape[1:]), dtype=like.dtype)


class LoopbackComm:
    """One of G ranks emulated as threads sharing a ``LoopbackHub``."""

    def __init__(self, hub, rank):
        self.hub = hub
        self.rank = rank
        self.world = hub.world

    def exchange_counts(self, send_counts, device):
        got = self.hub.swap(self.rank, list(send_counts))
        return [got[src][self.rank] for src in range(self.world)]

    def all_to_all(self, out, inp, out_splits, in_splits):
        got = self.hub.swap(self.rank, (inp, list(in_splits)))
        parts = []
        for src in range(self.world):
            t, splits = got[src]
            start = sum(splits[:self.rank])
            parts.append(t[start:start + splits[self.rank]])
        assert out.shape[0] == sum(out_splits)
        if out.shape[0]:
            torch.cat(parts, out=out)
        return out


class LoopbackHub:
    def __init__(self, world):
        self.world = world
        self.slots = [None] * world
        self.barrier = threading.Barrier(world, timeout=120)

    def swap(self, rank, value):
        self.slots[rank] = value
        self.barrier.wait()
        got = list(self.slots)
        self.barrier.wait()
        return got

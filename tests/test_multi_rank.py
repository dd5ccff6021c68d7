"""The benchmark's multi-rank plumbing on CPU with two gloo ranks.

The layer shards by tokens with no exchange step, so with N GPUs every rank
runs its own replica; ranks only meet for the barrier, the max over ranks of
the step time, and rank 0 printing the line.  These tests run that plumbing
as two spawned gloo processes (no GPU).
"""
import datetime
import os
import socket
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import moe_inputs

        # each rank timed its own replica; the slowest rank defines the step
        my_ms = 2.0 + rank  # rank 1 is slower
        ms = bench.reduce_max(my_ms, world, torch.device("cpu"))
        e2e = bench.reduce_max(3.0 - rank, world, torch.device("cpu"))
        dist.barrier()
        out = {"rank": rank, "ms": ms, "e2e": e2e}
        if rank == 0:
            cfg = moe_inputs.PREFILL
            res = {"peaks": bench.load_peaks(), "stage_ms": [0.02, 0.02, 1.0, 0.8, 0.1],
                   "step_quantiles": {"p25": 1.9, "p50": 2.0, "p75": 2.1}, "n_active": 256,
                   "clocks": None, "decode": None}
            args = types.SimpleNamespace(steps=5, warmup=3)
            line = bench.compose_line(args, cfg, world, res, ms, e2e)
            out["value"] = line["value"]
            out["n_gpus"] = line["n_gpus"]
            out["tokens_per_s"] = line["tokens_per_s"]
            out["scaling"] = line["scaling"]
        # the reference arm does its work on rank 0 only
        ref_args = types.SimpleNamespace(steps=1, warmup=0, seed=0)
        if rank != 0:
            assert bench.run_reference(ref_args, rank, world) is None
        q.put(out)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time_and_aggregate_throughput():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = {r["rank"]: r for r in results}
    # both ranks agree on the max over ranks
    assert by_rank[0]["ms"] == by_rank[1]["ms"] == 3.0
    assert by_rank[0]["e2e"] == by_rank[1]["e2e"] == 3.0
    # whole-job throughput: both replicas' routed FLOPs over the slowest rank's time
    import bench
    import moe_inputs
    flops = bench.prefill_flops(moe_inputs.PREFILL)
    assert by_rank[0]["value"] == pytest.approx(2 * flops / 3.0e-3 / 1e12)
    assert by_rank[0]["tokens_per_s"] == pytest.approx(2 * 4096 / 3.0e-3)
    assert by_rank[0]["n_gpus"] == 2 and by_rank[0]["scaling"] == "weak"

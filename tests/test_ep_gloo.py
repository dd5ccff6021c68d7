"""Expert-parallel orchestration on CPU ranks (gloo, world sizes 2 and 4).

Each rank routes its own tokens; the layer step (``ep.ep_moe_forward``) sorts
the routed rows by owner rank, exchanges them with ``all_to_all_single``,
runs the owner's experts, returns the per-slot rows and combines them on the
home rank.  The device steps here are the plain CPU definitions
(``ep_reference.NumpyEpOps``); the orchestration and the exchange are the
product's.  Every rank's output must equal, bit for bit, the single-rank step
over all experts on the same tokens, and match the oracle's layer.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import moe_inputs

E, HIDDEN, INTER, TOP_K = 8, 16, 8, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_inputs(case, rank):
    """Tokens of one rank (the weights are shared by all ranks)."""
    g = moe_inputs.generator(100 + rank)
    m = case["m"][rank % len(case["m"])] + (rank // len(case["m"]))
    layout = case.get("layout", 0)
    x = moe_inputs.bf16_normal((m * TOP_K if layout else m, HIDDEN), 1.0, g)
    if layout:
        x = x.view(m, TOP_K, HIDDEN)
    if case.get("ids") == "rank0_experts":      # every row goes to rank 0's experts
        ids = moe_inputs.uniform_distinct_ids(m, E // 2, TOP_K, g)
    elif case.get("ids") == "repeat":           # MayRepeat: every slot of t picks t mod E
        ids = moe_inputs.may_repeat_ids(m, E, TOP_K)
    else:
        ids = moe_inputs.uniform_distinct_ids(m, E, TOP_K, g)
    w = torch.rand((m, TOP_K), generator=g)
    return x, ids, w


def _weights():
    g = moe_inputs.generator(7)
    return (moe_inputs.bf16_normal((E, INTER, HIDDEN), 0.2, g),
            moe_inputs.bf16_normal((E, INTER, HIDDEN), 0.2, g),
            moe_inputs.bf16_normal((E, HIDDEN, INTER), 0.2, g))


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    import oracle
    from ep_reference import NumpyEpOps
    from mixture_experts_routed_sigmoid_b200.ep import SelfComm, TorchComm, ep_moe_forward

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ops = NumpyEpOps(oracle.default())
        Wg, Wu, Wd = _weights()
        per = E // world
        loc = slice(rank * per, (rank + 1) * per)
        for name, case in CASES.items():  # every rank takes the cases in the same order
            x, ids, w = _rank_inputs(case, rank)
            layout = case.get("layout", 0)
            y = ep_moe_forward(x, ids, w, Wg[loc].contiguous(), Wu[loc].contiguous(),
                               Wd[loc].contiguous(), E, TorchComm(), layout=layout, ops=ops)
            y1 = ep_moe_forward(x, ids, w, Wg, Wu, Wd, E, SelfComm(), layout=layout, ops=ops)
            np.save(os.path.join(out_dir, f"{name}_y{rank}.npy"), y.numpy())
            np.save(os.path.join(out_dir, f"{name}_y1_{rank}.npy"), y1.numpy())
    finally:
        dist.destroy_process_group()


CASES = {
    "uniform": {"m": [6, 5]},
    "one_rank_empty": {"m": [7, 0]},
    "all_rows_to_rank0": {"m": [4, 6], "ids": "rank0_experts"},
    "slotted": {"m": [5, 3], "layout": 1},
    "may_repeat": {"m": [9, 4], "ids": "repeat"},
}


@pytest.fixture(scope="module")
def gloo_results(tmp_path_factory):
    out = tmp_path_factory.mktemp("ep_gloo")
    for world in (2, 4):
        d = out / f"w{world}"
        d.mkdir()
        mp.spawn(_worker, args=(world, _free_port(), str(d)), nprocs=world, join=True)
    return out


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("name", list(CASES))
def test_gloo_ranks_match_one_rank_bit_for_bit(oracle_mod, gloo_results, name, world):
    """Two and four ranks (E/G = 4 and 2 experts each); with four ranks the
    case's per-rank token counts repeat, one token more per repetition."""
    case = CASES[name]
    bits = moe_inputs.bf16_bits
    Wg, Wu, Wd = _weights()
    res = gloo_results / f"w{world}"
    for rank in range(world):
        y = np.load(res / f"{name}_y{rank}.npy")
        y1 = np.load(res / f"{name}_y1_{rank}.npy")
        x, ids, w = _rank_inputs(case, rank)
        m = x.shape[0]
        assert y.shape == (m, HIDDEN)
        assert np.array_equal(y.view(np.int32), y1.view(np.int32)), rank
        if m:
            want = oracle_mod.ffn(bits(x), ids.numpy(), w.numpy(), bits(Wg), bits(Wu), bits(Wd),
                                  layout=case.get("layout", 0))
            np.testing.assert_allclose(y, want, rtol=1e-5, atol=1e-5 * np.abs(want).max())

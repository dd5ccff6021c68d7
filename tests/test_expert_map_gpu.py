"""GPU expert map vs the oracle: counts, offsets, perm, inv_perm bit-exact."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import host

pytestmark = pytest.mark.gpu


def _compare(oracle_mod, ids, E):
    got = moe.moe_expert_map(ids.cuda(), E)
    torch.cuda.synchronize()
    want = oracle_mod.expert_map(host(ids), E)
    for g, w, name in zip(got, want, ("counts", "offsets", "perm", "inv_perm")):
        assert np.array_equal(host(g), w), name


@pytest.mark.parametrize("m,E,top_k", [(1, 1, 1), (4, 8, 2), (9, 8, 6), (8, 256, 8),
                                       (300, 7, 3), (257, 1024, 8), (4096, 256, 8),
                                       (16384, 128, 8), (5000, 3, 3)])
def test_map_uniform_ids(oracle_mod, m, E, top_k):
    g = moe_inputs.generator(m + E)
    _compare(oracle_mod, moe_inputs.uniform_distinct_ids(m, E, top_k, g), E)


@pytest.mark.parametrize("m,E,top_k", [(4096, 256, 8), (777, 16, 4)])
def test_map_profiles(oracle_mod, m, E, top_k):
    _compare(oracle_mod, moe_inputs.skewed_ids(m, top_k), E)
    _compare(oracle_mod, moe_inputs.balanced_ids(m, E, top_k), E)


def test_map_repeated_ids(oracle_mod):
    g = moe_inputs.generator(3)
    ids = torch.randint(0, 5, (3000, 4), generator=g, dtype=torch.int32)
    _compare(oracle_mod, ids, 5)


def test_map_bad_id_sets_status():
    ids = torch.tensor([[0, 1], [7, 2]], dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_expert_map_workspace(2, 2, 4), dtype=torch.uint8, device="cuda")
    moe.moe_expert_map(ids, 4, ws=ws)
    assert moe.moe_check_status(ws) == 6  # MOE_ERR_DEVICE_BAD_ID
    ok = torch.tensor([[0, 1], [3, 2]], dtype=torch.int32, device="cuda")
    moe.moe_expert_map(ok, 4, ws=ws)
    assert moe.moe_check_status(ws) == 0  # every call clears the status word

"""GPU routing kernel vs the oracle: ids bit-exact, weights within 1e-6."""
import math

import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import WEIGHT_REL_TOL, host
from test_oracle import ROUTE_CASES

pytestmark = pytest.mark.gpu


def _compare(oracle_mod, logits, bias, top_k):
    lg = logits.cuda()
    b = None if bias is None else bias.cuda()
    scores = torch.empty_like(lg)
    ids, w = moe.moe_route_topk(lg, b, top_k, scores=scores)
    torch.cuda.synchronize()
    oid, ow, os_ = oracle_mod.route(host(logits), None if bias is None else host(bias), top_k)
    assert np.array_equal(host(ids), oid)
    np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)
    # the f32 score is sigmoid in double rounded once; allow one f32 ulp for
    # the two libraries' double exp
    gs = host(scores)
    nan = np.isnan(os_)
    assert np.array_equal(np.isnan(gs), nan)
    d = np.abs(gs.view(np.int32).astype(np.int64) - os_.view(np.int32))
    assert np.all(d[~nan] <= 1)


@pytest.mark.parametrize("m,E,top_k", [(1, 1, 1), (7, 5, 3), (33, 37, 4), (256, 64, 8),
                                       (100, 100, 32), (64, 1000, 8), (40, 1024, 32),
                                       (4096, 256, 8), (16384, 128, 8), (50, 384, 8),
                                       (10, 512, 16), (9, 33, 32)])
def test_route_matches_oracle(oracle_mod, m, E, top_k):
    g = moe_inputs.generator(m * 31 + E)
    logits = torch.randn((m, E), generator=g)
    bias = moe_inputs.uniform_bias(E, 0.1, g)
    _compare(oracle_mod, logits, bias, top_k)
    _compare(oracle_mod, logits, None, top_k)


def test_route_ties_and_coarse_values(oracle_mod):
    g = moe_inputs.generator(5)
    logits = (torch.randint(-3, 4, (512, 48), generator=g) * 0.5).float()
    bias = (torch.randint(-2, 3, (48,), generator=g) * 0.05).float()
    _compare(oracle_mod, logits, bias, 8)
    _compare(oracle_mod, torch.zeros((8, 64)), torch.zeros(64), 16)  # all tied


def test_route_special_values(oracle_mod):
    logits = torch.tensor([[float("nan"), 0.0, -200.0, 200.0, float("inf"), float("-inf"), 1.0, 2.0]])
    bias = torch.tensor([0.0, 0.0, 0.6, 0.0, 0.0, 0.0, -0.0, 0.0])
    _compare(oracle_mod, logits, bias, 5)


@pytest.mark.parametrize("case", ROUTE_CASES, ids=[c["name"] for c in ROUTE_CASES])
def test_route_closed_form_cases(case):
    logits = torch.tensor([case["logits"]], dtype=torch.float32, device="cuda")
    bias = torch.tensor(case["bias"], dtype=torch.float32, device="cuda")
    ids, w = moe.moe_route_topk(logits, bias, case["top_k"])
    assert host(ids)[0].tolist() == case["ids"]
    np.testing.assert_allclose(host(w)[0], case["weights"], rtol=1e-6, atol=1e-7)


def test_route_weights_forced(oracle_mod):
    g = moe_inputs.generator(9)
    m, E, top_k = 4096, 256, 8
    logits = torch.randn((m, E), generator=g)
    for ids in (moe_inputs.skewed_ids(m, top_k), moe_inputs.balanced_ids(m, E, top_k),
                moe_inputs.uniform_distinct_ids(m, E, top_k, g)):
        w = moe.moe_route_weights(logits.cuda(), ids.cuda())
        ow = oracle_mod.route_weights(host(logits), host(ids))
        np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)


def test_route_weights_bad_id_gives_nan():
    logits = torch.zeros((2, 4), device="cuda")
    ids = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")
    w = host(moe.moe_route_weights(logits, ids))
    assert np.allclose(w[0], [0.5, 0.5]) and np.isnan(w[1]).all()


def test_route_empty():
    ids, w = moe.moe_route_topk(torch.zeros((0, 8), device="cuda"), None, 2)
    assert ids.shape == (0, 2) and w.shape == (0, 2)

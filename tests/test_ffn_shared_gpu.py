"""GPU routed FFN plus the sigmoid-gated shared expert vs the oracle, across
the four path pairs (routed part streaming or grouped by m*top_k, shared part
streaming or grouped by m), ragged widths, a single token, the prefill layer
(sampled rows), and a bad id."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import (OUTPUT_REL_TOL, assert_overwritten_and_guarded, bits, host, poisoned_f32,
                     rel, sample_tokens)

pytestmark = pytest.mark.gpu

SH_KEYS = ("w_sh", "W_sh_gate", "W_sh_up", "W_sh_down")


def _layer(m, hidden, inter, inter_sh, E, top_k, seed, w_std=0.05):
    cfg = moe_inputs.FfnConfig("case", m, hidden, inter, E, top_k, w_std=w_std)
    inp = moe_inputs.ffn_inputs(cfg, seed=seed, device="cuda")
    inp.update(moe_inputs.shared_expert_inputs(hidden, inter_sh, seed, "cuda", w_std=w_std,
                                               gate_std=w_std))
    ids, w = moe.moe_route_topk(inp["logits"], inp["bias"], top_k)
    return inp, ids, w


def _want(oracle_mod, inp, ids, w, tokens=None):
    return oracle_mod.ffn_shared(bits(inp["x"]), host(ids), host(w), bits(inp["W_gate"]),
                                 bits(inp["W_up"]), bits(inp["W_down"]),
                                 *[bits(inp[k]) for k in SH_KEYS], tokens=tokens)


def _run(inp, ids, w, y=None):
    return moe.moe_ffn_forward_shared(inp["x"], ids, w, inp["W_gate"], inp["W_up"],
                                      inp["W_down"], *[inp[k] for k in SH_KEYS], y=y)


@pytest.mark.parametrize("m,hidden,inter,inter_sh,E,top_k", [
    (8, 256, 128, 192, 16, 8),      # routed streams (64 rows), shared streams
    (40, 256, 128, 96, 16, 8),      # routed grouped (320 rows), shared streams
    (300, 136, 200, 72, 5, 2),      # both grouped; widths off the tile grids
    (1, 512, 256, 512, 16, 8),      # a single token
    (129, 64, 64, 1032, 4, 1),      # shared grouped with a ragged last tile, top_k = 1
])
def test_shared_matches_oracle(oracle_mod, m, hidden, inter, inter_sh, E, top_k):
    inp, ids, w = _layer(m, hidden, inter, inter_sh, E, top_k, seed=m + inter_sh)
    buf, y = poisoned_f32((m, hidden))
    _run(inp, ids, w, y=y)
    torch.cuda.synchronize()
    assert_overwritten_and_guarded(buf, m * hidden)
    r = rel(host(y), _want(oracle_mod, inp, ids, w))
    assert r <= OUTPUT_REL_TOL, r


def test_shared_prefill_layer_sampled(oracle_mod):
    """The prefill layer (4096 tokens, hidden 4096, 256 experts of 1536, top-8)
    with a 1024-wide shared expert; sampled rows."""
    cfg = moe_inputs.PREFILL
    inp = moe_inputs.ffn_inputs(cfg, seed=0, device="cuda")
    inp.update(moe_inputs.shared_expert_inputs(cfg.hidden, 1024, 0, "cuda"))
    ids, w = moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k)
    y = _run(inp, ids, w)
    torch.cuda.synchronize()
    tokens = sample_tokens(cfg.m, 16, seed=5)
    got = host(y)
    assert np.isfinite(got).all()
    assert rel(got[tokens], _want(oracle_mod, inp, ids, w, tokens=tokens)) <= OUTPUT_REL_TOL
    # repeat call: same bits
    y2 = host(_run(inp, ids, w))
    assert np.array_equal(y2.view(np.int32), got.view(np.int32))


def test_zero_shared_down_gives_routed_bits():
    """W_sh_down = 0 adds exact zeros after the routed sum: the bits equal
    moe_ffn_forward's."""
    inp, ids, w = _layer(300, 128, 64, 64, 8, 2, seed=3)
    inp["W_sh_down"] = torch.zeros_like(inp["W_sh_down"])
    a = host(_run(inp, ids, w))
    b = host(moe.moe_ffn_forward(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"]))
    assert np.array_equal(a.view(np.int32), b.view(np.int32))


def test_shared_bad_id_reports_and_leaves_output():
    inp, ids, w = _layer(200, 64, 64, 64, 4, 2, seed=4)
    ids[7, 1] = 9
    ws = torch.empty(moe.moe_ffn_shared_workspace(200, 64, 64, 64, 2, 4), dtype=torch.uint8,
                     device="cuda")
    buf, y = poisoned_f32((200, 64))
    moe.moe_ffn_forward_shared(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"],
                               *[inp[k] for k in SH_KEYS], y=y, ws=ws)
    assert moe.moe_check_status(ws) == 6
    assert (buf.view(torch.int32).cpu().numpy() == 0x7FC000C7).all()

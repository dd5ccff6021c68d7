"""Decode-size FFN (m*top_k <= 128: the weight-streaming kernels) vs the
oracle on every row, on the prefill layer's weights, next to the first shape
past the threshold (which runs the grouped GEMMs)."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, WEIGHT_REL_TOL, bits, host, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    cfg = moe_inputs.PREFILL
    inp = moe_inputs.ffn_inputs(cfg, seed=3, device="cuda", m=40)
    host_bits = {k: bits(inp[k]) for k in ("W_gate", "W_up", "W_down")}
    return cfg, inp, host_bits


def _oracle_routing(oracle_mod, logits, bias, top_k, ids, w):
    """The oracle's own (ids, weights) for these logits; the GPU's must match
    (ids bit for bit, weights to 1e-6).  bias None: the ids were fixed by the
    caller and only the weights are the oracle's."""
    if bias is None:
        oid, ow = host(ids), oracle_mod.route_weights(host(logits), host(ids))
    else:
        oid, ow, _ = oracle_mod.route(host(logits), host(bias), top_k)
    assert np.array_equal(host(ids), oid)
    np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)
    return oid, ow


def _check(oracle_mod, layer, m, ids=None, w=None):
    cfg, inp, hb = layer
    x = inp["x"][:m].contiguous()
    logits = inp["logits"][:m].contiguous()
    forced = ids is not None
    if not forced:
        ids, w = moe.moe_route_topk(logits, inp["bias"], cfg.top_k)
    oid, ow = _oracle_routing(oracle_mod, logits, None if forced else inp["bias"], cfg.top_k,
                              ids, w)
    y = moe.moe_ffn_forward(x, ids, w, inp["W_gate"], inp["W_up"], inp["W_down"])
    torch.cuda.synchronize()
    want = oracle_mod.ffn(bits(x), oid, ow, hb["W_gate"], hb["W_up"], hb["W_down"])
    r = rel(host(y), want)
    assert r <= OUTPUT_REL_TOL, r
    return y


@pytest.mark.parametrize("m", [1, 2, 8, 16, 17])  # 16*8 = 128 streams, 17*8 = 136 does not
def test_decode_ffn_matches_oracle(oracle_mod, layer, m):
    _check(oracle_mod, layer, m)


def test_decode_ffn_skewed_batch(oracle_mod, layer):
    """All 16 tokens on experts 0..7: 16 rows per expert, several passes."""
    cfg, inp, _ = layer
    ids = moe_inputs.skewed_ids(16, cfg.top_k, "cuda")
    w = moe.moe_route_weights(inp["logits"][:16].contiguous(), ids)
    y_s = _check(oracle_mod, layer, 16, ids, w)
    # balanced routing of the same rows: token 0 has the same ids, order and
    # weights in both, and its output bits must agree
    ids_b = moe_inputs.balanced_ids(16, cfg.n_experts, cfg.top_k, "cuda")
    w_b = moe.moe_route_weights(inp["logits"][:16].contiguous(), ids_b)
    y_b = moe.moe_ffn_forward(inp["x"][:16].contiguous(), ids_b, w_b, inp["W_gate"], inp["W_up"],
                              inp["W_down"])
    assert np.array_equal(host(y_s)[0].view(np.int32), host(y_b)[0].view(np.int32))


def test_decode_ffn_slotted_long_layer(oracle_mod):
    cfg = moe_inputs.LONG
    inp = moe_inputs.ffn_inputs(cfg, seed=4, device="cuda", m=6)
    ids, w = moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k)
    oid, ow = _oracle_routing(oracle_mod, inp["logits"], inp["bias"], cfg.top_k, ids, w)
    y = moe.moe_ffn_forward(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"],
                            layout=moe.SLOTTED)
    torch.cuda.synchronize()
    want = oracle_mod.ffn(bits(inp["x"]), oid, ow, bits(inp["W_gate"]),
                          bits(inp["W_up"]), bits(inp["W_down"]), layout=1)
    assert rel(host(y), want) <= OUTPUT_REL_TOL


def test_decode_ffn_repeat_bits():
    cfg = moe_inputs.LONG
    inp = moe_inputs.ffn_inputs(cfg, seed=5, device="cuda", m=16)
    ids, w = moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k)
    args = (inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"])
    a = host(moe.moe_ffn_forward(*args, layout=moe.SLOTTED))
    b = host(moe.moe_ffn_forward(*args, layout=moe.SLOTTED))
    assert np.array_equal(a.view(np.int32), b.view(np.int32))


def test_decode_ffn_row_independence():
    """Among decode-size batches (the streaming path) a token's bits do not
    depend on the batch it is in."""
    cfg = moe_inputs.LONG
    inp = moe_inputs.ffn_inputs(cfg, seed=6, device="cuda", m=16)
    ids, w = moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k)
    W = (inp["W_gate"], inp["W_up"], inp["W_down"])
    y = host(moe.moe_ffn_forward(inp["x"], ids, w, *W, layout=moe.SLOTTED))
    sub = slice(5, 12)
    ys = host(moe.moe_ffn_forward(inp["x"][sub].contiguous(), ids[sub].contiguous(),
                                  w[sub].contiguous(), *W, layout=moe.SLOTTED))
    assert np.array_equal(ys.view(np.int32), y[sub].view(np.int32))

"""GPU routed SwiGLU MoE FFN vs the oracle, at small sizes (every row) and at
the full prefill, skewed and long workloads (sampled rows; rows are
independent given ids and weights, so a sampled row is an exact check of that
row), plus the balanced/skewed bit-identity and determinism."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import (OUTPUT_REL_TOL, WEIGHT_REL_TOL, assert_overwritten_and_guarded, bits, host,
                     poisoned_f32, rel, sample_tokens)

pytestmark = pytest.mark.gpu


def _weights(seed, E, inter, hidden, std, device="cuda"):
    g = moe_inputs.generator(seed, device)
    Wg = moe_inputs.bf16_normal((E, inter, hidden), std, g, device)
    Wu = moe_inputs.bf16_normal((E, inter, hidden), std, g, device)
    Wd = moe_inputs.bf16_normal((E, hidden, inter), std, g, device)
    return Wg, Wu, Wd


def _oracle_y(oracle_mod, x, ids, w, Wg, Wu, Wd, layout, tokens=None):
    return oracle_mod.ffn(bits(x), host(ids), host(w), bits(Wg), bits(Wu), bits(Wd),
                          layout=layout, tokens=tokens)


@pytest.mark.parametrize("m,hidden,inter,E,top_k,layout", [
    (64, 256, 128, 8, 2, 0),
    (200, 136, 200, 5, 3, 0),     # hidden and inter off the 64/128 tile grid
    (130, 64, 72, 4, 4, 1),       # slotted layout, top_k = E
    (1, 512, 256, 16, 8, 0),      # a single token
    (300, 128, 1536, 2, 1, 0),    # top_k = 1, long inter
    (40, 128, 64, 64, 32, 0),     # top_k = 32 (the maximum): 4 combine load batches
    (4, 128, 64, 64, 32, 0),      # top_k = 32, 128 routed rows: the streaming path
    (96, 136, 72, 24, 12, 1),     # top_k = 12: a partial combine batch, slotted
])
def test_ffn_small_all_rows(oracle_mod, m, hidden, inter, E, top_k, layout):
    g = moe_inputs.generator(m + hidden + inter, "cuda")
    x = moe_inputs.bf16_normal((m * top_k if layout else m, hidden), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, hidden)
    logits = torch.randn((m, E), generator=g, device="cuda")
    bias = moe_inputs.uniform_bias(E, 0.1, g, "cuda")
    Wg, Wu, Wd = _weights(m + 1, E, inter, hidden, 0.05)
    ids, w = moe.moe_route_topk(logits, bias, top_k)
    buf, y = poisoned_f32((m, hidden))
    moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=layout, y=y)
    torch.cuda.synchronize()
    assert_overwritten_and_guarded(buf, m * hidden)
    want = _oracle_y(oracle_mod, x, ids, w, Wg, Wu, Wd, layout)
    assert rel(host(y), want) <= OUTPUT_REL_TOL


def _full_layer(cfg, oracle_mod, n_sample, seed=0):
    inp = moe_inputs.ffn_inputs(cfg, seed=seed, device="cuda")
    logits, bias = inp["logits"], inp["bias"]
    if "ids" in inp:
        ids = inp["ids"]
        w = moe.moe_route_weights(logits, ids)
        np.testing.assert_allclose(host(w), oracle_mod.route_weights(host(logits), host(ids)),
                                   rtol=WEIGHT_REL_TOL, atol=0)
    else:
        ids, w = moe.moe_route_topk(logits, bias, cfg.top_k)
        oid, ow, _ = oracle_mod.route(host(logits), host(bias), cfg.top_k)
        assert np.array_equal(host(ids), oid)
        np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)
    y = moe.moe_ffn_forward(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"],
                            layout=cfg.layout)
    torch.cuda.synchronize()
    tokens = sample_tokens(cfg.m, n_sample, seed=seed + 1)
    want = _oracle_y(oracle_mod, inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"],
                     cfg.layout, tokens=tokens)
    got = host(y)
    assert np.isfinite(got).all()
    r = rel(got[tokens], want)
    assert r <= OUTPUT_REL_TOL, r
    return inp, ids, w, y


def test_prefill_workload_sampled(oracle_mod):
    _full_layer(moe_inputs.PREFILL, oracle_mod, n_sample=24)


def test_long_workload_sampled(oracle_mod):
    _full_layer(moe_inputs.LONG, oracle_mod, n_sample=48)


def test_skewed_workload_and_bit_identity(oracle_mod):
    """Skewed (all tokens on experts 0..7) vs balanced ((t + j) mod E) routing
    of the same layer: tokens with t = 0 mod E have the same ids, slot order
    and weights in both, and their outputs must be bit-identical."""
    cfg = moe_inputs.SKEWED
    inp, ids_s, w_s, y_s = _full_layer(cfg, oracle_mod, n_sample=16)
    ids_b = moe_inputs.balanced_ids(cfg.m, cfg.n_experts, cfg.top_k, "cuda")
    w_b = moe.moe_route_weights(inp["logits"], ids_b)
    y_b = moe.moe_ffn_forward(inp["x"], ids_b, w_b, inp["W_gate"], inp["W_up"], inp["W_down"])
    same = np.arange(0, cfg.m, cfg.n_experts)
    assert np.array_equal(host(ids_s)[same], host(ids_b)[same])
    assert np.array_equal(host(w_s)[same].view(np.int32), host(w_b)[same].view(np.int32))
    assert np.array_equal(host(y_s)[same].view(np.int32), host(y_b)[same].view(np.int32))
    # the balanced run is itself correct
    tokens = sample_tokens(cfg.m, 8, seed=3)
    want = _oracle_y(oracle_mod, inp["x"], ids_b, w_b, inp["W_gate"], inp["W_up"], inp["W_down"],
                     0, tokens=tokens)
    assert rel(host(y_b)[tokens], want) <= OUTPUT_REL_TOL


def test_row_independence_and_repeat_runs():
    """A token's output bits do not depend on the batch it is in (among
    batches that take the same path: here both run the grouped GEMMs), and
    repeated calls give identical bits."""
    m, hidden, inter, E, top_k = 600, 256, 256, 16, 4
    g = moe_inputs.generator(77, "cuda")
    x = moe_inputs.bf16_normal((m, hidden), 1.0, g, "cuda")
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    w = torch.rand((m, top_k), generator=g, device="cuda")
    Wg, Wu, Wd = _weights(78, E, inter, hidden, 0.05)
    y1 = host(moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd))
    y2 = host(moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd))
    assert np.array_equal(y1.view(np.int32), y2.view(np.int32))
    sub = slice(123, 193)  # 70 tokens x 4 = 280 routed rows: still the grouped-GEMM path
    ys = host(moe.moe_ffn_forward(x[sub].contiguous(), ids[sub].contiguous(),
                                  w[sub].contiguous(), Wg, Wu, Wd))
    assert np.array_equal(ys.view(np.int32), y1[sub].view(np.int32))


def test_bad_id_reports_and_leaves_output():
    m, hidden, inter, E, top_k = 32, 64, 64, 4, 2
    g = moe_inputs.generator(1, "cuda")
    x = moe_inputs.bf16_normal((m, hidden), 1.0, g, "cuda")
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    ids[3, 0] = -1
    w = torch.full((m, top_k), 0.5, device="cuda")
    Wg, Wu, Wd = _weights(2, E, inter, hidden, 0.05)
    ws = torch.empty(moe.moe_ffn_workspace(m, hidden, inter, top_k, E), dtype=torch.uint8,
                     device="cuda")
    buf, y = poisoned_f32((m, hidden))
    moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, y=y, ws=ws)
    assert moe.moe_check_status(ws) == 6
    assert (buf.view(torch.int32).cpu().numpy() == 0x7FC000C7).all()


def test_empty_input():
    W = torch.zeros((4, 32, 64), dtype=torch.bfloat16, device="cuda")
    Wd = torch.zeros((4, 64, 32), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    w = torch.zeros((0, 2), device="cuda")
    y = moe.moe_ffn_forward(x, ids, w, W, W, Wd, ws=torch.empty(256, dtype=torch.uint8,
                                                                device="cuda"))
    assert y.shape == (0, 64)

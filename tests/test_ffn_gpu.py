"""GPU routed SwiGLU MoE FFN vs the oracle on every output row: small shapes,
the full prefill, skewed and long workloads, and repeated ids (MayRepeat),
plus the balanced/skewed bit-identity and determinism.  The oracle always
takes its own routing (ids and weights), which the GPU routing must match:
ids bit for bit, weights within 1e-6."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import (FP16_ACT_TOL, OUTPUT_REL_TOL, WEIGHT_REL_TOL, assert_overwritten_and_guarded,
                     bits, host, poisoned_f32, rel, sample_tokens)

pytestmark = pytest.mark.gpu


def _weights(seed, E, inter, hidden, std, device="cuda"):
    g = moe_inputs.generator(seed, device)
    Wg = moe_inputs.bf16_normal((E, inter, hidden), std, g, device)
    Wu = moe_inputs.bf16_normal((E, inter, hidden), std, g, device)
    Wd = moe_inputs.bf16_normal((E, hidden, inter), std, g, device)
    return Wg, Wu, Wd


def _oracle_y(oracle_mod, x, ids, w, Wg, Wu, Wd, layout, tokens=None, act_mode=0):
    return oracle_mod.ffn(bits(x), host(ids), host(w), bits(Wg), bits(Wu), bits(Wd),
                          layout=layout, tokens=tokens, act_mode=act_mode)


@pytest.mark.parametrize("m,hidden,inter,E,top_k,layout", [
    (64, 256, 128, 8, 2, 0),
    (200, 136, 200, 5, 3, 0),     # hidden and inter off the 64/128 tile grid
    (130, 64, 72, 4, 4, 1),       # slotted layout, top_k = E
    (1, 512, 256, 16, 8, 0),      # a single token
    (300, 128, 1536, 2, 1, 0),    # top_k = 1, long inter
    (40, 128, 64, 64, 32, 0),     # top_k = 32 (the maximum): 4 combine load batches
    (4, 128, 64, 64, 32, 0),      # top_k = 32, 128 routed rows: the streaming path
    (96, 136, 72, 24, 12, 1),     # top_k = 12: a partial combine batch, slotted
    (600, 136, 200, 2, 2, 0),     # 600 rows per expert (W_down converted up front), ragged widths
    (520, 72, 136, 3, 3, 1),      # 520 rows per expert, slotted, ragged widths
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
    oid, ow = _oracle_routing(oracle_mod, logits, bias, top_k, ids, w)
    buf, y = poisoned_f32((m, hidden))
    moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=layout, y=y)
    torch.cuda.synchronize()
    assert_overwritten_and_guarded(buf, m * hidden)
    want = _oracle_y(oracle_mod, x, oid, ow, Wg, Wu, Wd, layout)
    assert rel(host(y), want) <= OUTPUT_REL_TOL
    if m * top_k > 128:  # the grouped GEMMs
        want2 = _oracle_y(oracle_mod, x, oid, ow, Wg, Wu, Wd, layout, act_mode=2)
        assert rel(host(y), want2) <= FP16_ACT_TOL


def _oracle_routing(oracle_mod, logits, bias, top_k, ids, w):
    """The oracle's own routing of the logits; the GPU's must match it (ids bit
    for bit, weights to 1e-6).  Returns the oracle's (ids, weights)."""
    oid, ow, _ = oracle_mod.route(host(logits), None if bias is None else host(bias), top_k)
    assert np.array_equal(host(ids), oid)
    np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)
    return oid, ow


def _oracle_forced(oracle_mod, logits, ids, w):
    """The oracle's weights of caller-fixed ids; the GPU's must match to 1e-6."""
    ow = oracle_mod.route_weights(host(logits), host(ids))
    np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)
    return host(ids), ow


def _full_layer(cfg, oracle_mod, seed=0):
    """The whole workload on the GPU and every output row against the oracle
    fed its own routing of the same logits."""
    inp = moe_inputs.ffn_inputs(cfg, seed=seed, device="cuda")
    logits, bias = inp["logits"], inp["bias"]
    if "ids" in inp:
        ids = inp["ids"]
        w = moe.moe_route_weights(logits, ids)
        oid, ow = _oracle_forced(oracle_mod, logits, ids, w)
    else:
        ids, w = moe.moe_route_topk(logits, bias, cfg.top_k)
        oid, ow = _oracle_routing(oracle_mod, logits, bias, cfg.top_k, ids, w)
    y = moe.moe_ffn_forward(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"],
                            layout=cfg.layout)
    torch.cuda.synchronize()
    want = _oracle_y(oracle_mod, inp["x"], oid, ow, inp["W_gate"], inp["W_up"], inp["W_down"],
                     cfg.layout)
    got = host(y)
    assert np.isfinite(got).all()
    r = rel(got, want)
    assert r <= OUTPUT_REL_TOL, r
    return inp, ids, w, y


def test_prefill_workload_every_row(oracle_mod):
    inp, ids, w, y = _full_layer(moe_inputs.PREFILL, oracle_mod)
    # a token sample against the oracle's rounding of the fp16 activation
    oid, ow, _ = oracle_mod.route(host(inp["logits"]), host(inp["bias"]), 8)
    tokens = sample_tokens(moe_inputs.PREFILL.m, 256, seed=4)
    want2 = _oracle_y(oracle_mod, inp["x"], oid, ow, inp["W_gate"], inp["W_up"], inp["W_down"], 0,
                      tokens=tokens, act_mode=2)
    assert rel(host(y)[tokens], want2) <= FP16_ACT_TOL


def test_long_workload_every_row(oracle_mod):
    _full_layer(moe_inputs.LONG, oracle_mod)


def test_skewed_workload_every_row_and_bit_identity(oracle_mod):
    """Skewed (all tokens on experts 0..7) vs balanced ((t + j) mod E) routing
    of the same layer: tokens with t = 0 mod E have the same ids, slot order
    and weights in both, and their outputs must be bit-identical."""
    cfg = moe_inputs.SKEWED
    inp, ids_s, w_s, y_s = _full_layer(cfg, oracle_mod)
    ids_b = moe_inputs.balanced_ids(cfg.m, cfg.n_experts, cfg.top_k, "cuda")
    w_b = moe.moe_route_weights(inp["logits"], ids_b)
    y_b = moe.moe_ffn_forward(inp["x"], ids_b, w_b, inp["W_gate"], inp["W_up"], inp["W_down"])
    same = np.arange(0, cfg.m, cfg.n_experts)
    assert np.array_equal(host(ids_s)[same], host(ids_b)[same])
    assert np.array_equal(host(w_s)[same].view(np.int32), host(w_b)[same].view(np.int32))
    assert np.array_equal(host(y_s)[same].view(np.int32), host(y_b)[same].view(np.int32))
    # the balanced run is itself correct (a sample: its rows are the prefill
    # layer's cost again)
    oid, ow = _oracle_forced(oracle_mod, inp["logits"], ids_b, w_b)
    tokens = sample_tokens(cfg.m, 64, seed=3)
    want = _oracle_y(oracle_mod, inp["x"], oid, ow, inp["W_gate"], inp["W_up"], inp["W_down"],
                     0, tokens=tokens)
    assert rel(host(y_b)[tokens], want) <= OUTPUT_REL_TOL


@pytest.mark.parametrize("m,hidden,inter,E,top_k,layout", [
    (8, 256, 128, 16, 8, 0),       # 64 routed rows: the streaming path
    (16, 136, 72, 8, 8, 1),        # 128 routed rows, slotted, ragged widths: streaming
    (512, 256, 192, 32, 8, 0),     # 4096 routed rows: the grouped GEMMs, 128 rows per expert
    (300, 128, 136, 7, 4, 1),      # grouped, slotted, ragged widths, partial tiles
])
def test_ffn_repeated_ids_every_row(oracle_mod, m, hidden, inter, E, top_k, layout):
    """mlx-native's MayRepeat profile (every slot of token t picks expert
    t mod E): each slot is its own routed row, so a token's output is its
    expert's MLP at the summed weight; repeated rows of the shared layout have
    identical per-slot bits."""
    g = moe_inputs.generator(m + E, "cuda")
    x = moe_inputs.bf16_normal((m * top_k if layout else m, hidden), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, hidden)
    logits = torch.randn((m, E), generator=g, device="cuda")
    Wg, Wu, Wd = _weights(m + 3, E, inter, hidden, 0.05)
    ids = moe_inputs.may_repeat_ids(m, E, top_k, "cuda")
    w = moe.moe_route_weights(logits, ids)
    oid, ow = _oracle_forced(oracle_mod, logits, ids, w)
    buf, y = poisoned_f32((m, hidden))
    moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=layout, y=y)
    torch.cuda.synchronize()
    assert_overwritten_and_guarded(buf, m * hidden)
    want = _oracle_y(oracle_mod, x, oid, ow, Wg, Wu, Wd, layout)
    assert rel(host(y), want) <= OUTPUT_REL_TOL
    if layout == 0:
        d = host(moe.moe_ffn_slots(x, ids, Wg, Wu, Wd))
        assert np.array_equal(d.view(np.int32), np.repeat(d[:, :1], top_k, 1).view(np.int32))


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


@pytest.mark.parametrize("m", [64, 512])
def test_fp16_range_is_reported_and_leaves_output(oracle_mod, m):
    """The grouped path's down projection multiplies in fp16: the activation
    is stored as fp16(a * 2^-4) and W_down as fp16(w), converted in shared
    memory (m = 64: 64 rows per expert) or once before the GEMM (m = 512: 512
    rows per expert).  An activation above 65504 * 2^4, a W_down entry of
    65536 or more, or a non-finite input gives a non-finite accumulator:
    MOE_ERR_DEVICE_RANGE, the output unwritten.  The largest in-range W_down
    entry (65280) is computed correctly."""
    hidden, inter, E, top_k = 64, 64, 4, 4   # every token picks every expert
    g = moe_inputs.generator(3, "cuda")
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    w = torch.full((m, top_k), 0.25, device="cuda")
    Wg, Wu, Wd = _weights(4, E, inter, hidden, 0.05)
    ws = torch.empty(moe.moe_ffn_workspace(m, hidden, inter, top_k, E), dtype=torch.uint8,
                     device="cuda")
    x = moe_inputs.bf16_normal((m, hidden), 1.0, g, "cuda")

    def rejected(x_, Wd_):
        buf, y = poisoned_f32((m, hidden))
        moe.moe_ffn_forward(x_, ids, w, Wg, Wu, Wd_, y=y, ws=ws)
        assert moe.moe_check_status(ws) == 7
        assert (buf.view(torch.int32).cpu().numpy() == 0x7FC000C7).all()

    # activations far past 2^20: x ~ N(0, 10^4) gives |g|, |u| in the thousands
    rejected(moe_inputs.bf16_normal((m, hidden), 1.0e4, g, "cuda"), Wd)
    Wd_big = Wd.clone()
    Wd_big[1, 5, 7] = 1.0e5
    rejected(x, Wd_big)
    x_nan = x.clone()
    x_nan[3, 9] = float("nan")
    rejected(x_nan, Wd)
    # the edge of the range, then a clean call on the same workspace
    Wd_edge = Wd.clone()
    Wd_edge[1, 5, 7] = 65280.0
    Wd_edge[2, 6, 8] = -65280.0
    y = moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd_edge, ws=ws)
    assert moe.moe_check_status(ws) == 0
    tokens = sample_tokens(m, 64, seed=5)
    want = _oracle_y(oracle_mod, x, ids, w, Wg, Wu, Wd_edge, 0, tokens=tokens, act_mode=2)
    assert rel(host(y)[tokens], want) <= FP16_ACT_TOL
    y = moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, ws=ws)
    assert moe.moe_check_status(ws) == 0 and np.isfinite(host(y)).all()


def test_empty_input():
    W = torch.zeros((4, 32, 64), dtype=torch.bfloat16, device="cuda")
    Wd = torch.zeros((4, 64, 32), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    w = torch.zeros((0, 2), device="cuda")
    y = moe.moe_ffn_forward(x, ids, w, W, W, Wd, ws=torch.empty(256, dtype=torch.uint8,
                                                                device="cuda"))
    assert y.shape == (0, 64)

"""Router projection + routing on the GPU vs the oracle.

Logits come from the tensor cores in f32 (for few row tiles the projection's
K is split into ranges whose partial sums the routing kernel adds in order:
1, 2, 4 and 8 ranges are covered); they are compared with the oracle's f64
logits within the output bar.  The expert choice is an integer decision
taken on those f32 logits, so it is compared bit-exactly with the oracle's
routing applied to the same GPU logits (the decision in the kernel's
precision), and the weights within 1e-6.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, WEIGHT_REL_TOL, bits, host, rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,hidden,E,top_k,use_bias", [
    (4096, 4096, 256, 8, True),     # the prefill layer's router
    (300, 2048, 128, 8, True),      # long-layer width, ragged m
    (1, 512, 8, 2, False),          # a single token
    (130, 136, 1000, 32, True),     # K off the 64 grid, E over 3 column tiles, top-32
    (257, 64, 37, 5, False),        # N tail not a multiple of 4
    (64, 1024, 512, 8, True),       # two 256-column tiles, each split into 4 K ranges
    (20, 520, 300, 6, True),        # 2 K ranges, the last one past K; E over 2 column tiles
])
def test_router_matches_oracle(oracle_mod, m, hidden, E, top_k, use_bias):
    g = moe_inputs.generator(m + E, "cuda")
    x = moe_inputs.bf16_normal((m, hidden), 1.0, g, "cuda")
    W = moe_inputs.bf16_normal((E, hidden), 0.02, g, "cuda")
    bias = moe_inputs.uniform_bias(E, 0.1, g, "cuda") if use_bias else None
    ids, w, logits = moe.moe_router_topk(x, W, bias, top_k)
    torch.cuda.synchronize()
    want = oracle_mod.router_logits(bits(x), bits(W))
    lg = host(logits)
    assert rel(lg, want) <= OUTPUT_REL_TOL
    oid, ow, _ = oracle_mod.route(lg, None if bias is None else host(bias), top_k)
    assert np.array_equal(host(ids), oid)
    np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)


def test_router_then_ffn_end_to_end(oracle_mod):
    """Hidden state -> router -> routed SwiGLU layer, against the oracle.  The
    expert choice is an integer decision taken on the projection's f32
    logits, so the oracle routes those same logits itself (its ids must equal
    the GPU's) and then runs the layer with its own ids and weights."""
    m, hidden, inter, E, top_k = 256, 512, 256, 16, 4
    g = moe_inputs.generator(5, "cuda")
    x = moe_inputs.bf16_normal((m, hidden), 1.0, g, "cuda")
    Wr = moe_inputs.bf16_normal((E, hidden), 0.05, g, "cuda")
    bias = moe_inputs.uniform_bias(E, 0.1, g, "cuda")
    Wg = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wu = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wd = moe_inputs.bf16_normal((E, hidden, inter), 0.05, g, "cuda")
    ids, w, logits = moe.moe_router_topk(x, Wr, bias, top_k)
    y = moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd)
    torch.cuda.synchronize()
    assert rel(host(logits), oracle_mod.router_logits(bits(x), bits(Wr))) <= OUTPUT_REL_TOL
    oid, ow, _ = oracle_mod.route(host(logits), host(bias), top_k)
    assert np.array_equal(host(ids), oid)
    np.testing.assert_allclose(host(w), ow, rtol=WEIGHT_REL_TOL, atol=0)
    want = oracle_mod.ffn(bits(x), oid, ow, bits(Wg), bits(Wu), bits(Wd))
    assert rel(host(y), want) <= OUTPUT_REL_TOL

"""GPU per-slot rows of the routed FFN (moe_ffn_slots): each slot against the
oracle, moe_ffn_forward's output as their weighted slot-order f32 sum bit for
bit, and every (token, expert) pair that the balanced and the maximally
skewed routing profiles share bit-identical on the full skewed layer."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, bits, host, rel

pytestmark = pytest.mark.gpu


def _slot_sum(d, w):
    """sum_j w[t, j] * d[t, j] in f32, in slot order (numpy f32 arithmetic)."""
    acc = (w[:, 0:1] * d[:, 0]).astype(np.float32)
    for j in range(1, d.shape[1]):
        acc = (acc + (w[:, j:j + 1] * d[:, j]).astype(np.float32)).astype(np.float32)
    return acc


@pytest.mark.parametrize("m,hidden,inter,E,top_k,layout", [
    (8, 256, 128, 16, 8, 0),      # 64 routed rows: the streaming kernels
    (300, 136, 200, 5, 3, 0),     # grouped GEMMs, widths off the tile grids
    (130, 64, 72, 4, 4, 1),       # grouped, slotted layout
    (60, 128, 64, 32, 12, 0),     # top_k = 12: the combine sums 8 slots, then 4
])
def test_slots_match_oracle_and_forward(oracle_mod, m, hidden, inter, E, top_k, layout):
    g = moe_inputs.generator(m + inter, "cuda")
    x = moe_inputs.bf16_normal((m * top_k if layout else m, hidden), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, hidden)
    Wg = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wu = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wd = moe_inputs.bf16_normal((E, hidden, inter), 0.05, g, "cuda")
    logits = torch.randn((m, E), generator=g, device="cuda")
    ids, w = moe.moe_route_topk(logits, moe_inputs.uniform_bias(E, 0.1, g, "cuda"), top_k)
    d = host(moe.moe_ffn_slots(x, ids, Wg, Wu, Wd, layout=layout))
    y = host(moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=layout))
    assert np.array_equal(_slot_sum(d, host(w)).view(np.int32), y.view(np.int32))
    hids = host(ids)
    xb = bits(x)
    for j in range(top_k):
        xj = xb[:, j] if layout else xb
        want = oracle_mod.ffn(xj, hids[:, j:j + 1], np.ones((m, 1), np.float32), bits(Wg),
                              bits(Wu), bits(Wd))
        assert rel(d[:, j], want) <= OUTPUT_REL_TOL


def test_balanced_and_skewed_pairs_bit_identical():
    """The skewed layer (4096 tokens on experts 0..7) and its balanced
    counterpart ((t + j) mod 256): every (token, expert) pair present in both
    has identical per-slot bits."""
    cfg = moe_inputs.SKEWED
    inp = moe_inputs.ffn_inputs(cfg, seed=0, device="cuda")
    W = (inp["W_gate"], inp["W_up"], inp["W_down"])
    skw = inp["ids"]
    bal = moe_inputs.balanced_ids(cfg.m, cfg.n_experts, cfg.top_k, "cuda")
    ds = moe.moe_ffn_slots(inp["x"], skw, *W)
    db = moe.moe_ffn_slots(inp["x"], bal, *W)
    hs, hb = host(skw), host(bal)
    pairs = 0
    for js in range(cfg.top_k):
        for jb in range(cfg.top_k):
            t = np.nonzero(hs[:, js] == hb[:, jb])[0]
            if len(t) == 0:
                continue
            tt = torch.from_numpy(t).cuda()
            a = ds[tt, js].contiguous().view(torch.int32)
            b = db[tt, jb].contiguous().view(torch.int32)
            assert torch.equal(a, b)
            pairs += len(t)
    assert pairs == 1024  # tokens with t mod 256 in [0, 8) or [249, 256)

"""Expert parallelism on the GPU: the dispatch kernels against their plain
definition, one rank against moe_ffn_forward bit for bit, and G = 2 and 4
ranks emulated on one GPU (threads exchanging rows through the host; no
kernel waits on another) against the single-rank layer and the oracle."""
import threading

import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from ep_reference import LoopbackComm, LoopbackHub
from helpers import OUTPUT_REL_TOL, bits, host, rel
from mixture_experts_routed_sigmoid_b200.ep import SelfComm, ep_moe_forward

pytestmark = pytest.mark.gpu


def _layer(seed, E, hidden, inter, std=0.05):
    g = moe_inputs.generator(seed, "cuda")
    return (moe_inputs.bf16_normal((E, inter, hidden), std, g, "cuda"),
            moe_inputs.bf16_normal((E, inter, hidden), std, g, "cuda"),
            moe_inputs.bf16_normal((E, hidden, inter), std, g, "cuda"))


def _tokens(seed, m, E, top_k, hidden, layout=0, ids=None):
    g = moe_inputs.generator(seed, "cuda")
    x = moe_inputs.bf16_normal((m * top_k if layout else m, hidden), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, hidden)
    logits = torch.randn((m, E), generator=g, device="cuda")
    bias = moe_inputs.uniform_bias(E, 0.1, g, "cuda")
    if ids is None:
        ids, w = moe.moe_route_topk(logits, bias, top_k)
    else:
        w = moe.moe_route_weights(logits, ids)
    return x, ids, w


@pytest.mark.parametrize("layout", [0, 1])
def test_dispatch_matches_its_definition(layout):
    m, E, G, top_k, hidden = 300, 16, 4, 4, 136
    x, ids, _ = _tokens(1, m, E, top_k, hidden, layout)
    send_x, send_e, counts, ws = moe.moe_ep_dispatch(x, ids, E, G, layout)
    torch.cuda.synchronize()
    flat = host(ids).reshape(-1).astype(np.int64)
    owner = flat // (E // G)
    perm = np.argsort(owner, kind="stable")
    assert np.array_equal(host(counts), np.bincount(owner, minlength=G))
    assert np.array_equal(host(send_e), flat[perm] - owner[perm] * (E // G))
    src = perm if layout else perm // top_k
    assert np.array_equal(bits(send_x), bits(x).reshape(-1, hidden)[src])
    assert moe.moe_check_status(ws) == 0


def test_dispatch_reports_a_bad_id():
    m, E, G, top_k, hidden = 40, 8, 2, 2, 64
    x, ids, _ = _tokens(2, m, E, top_k, hidden)
    ids[7, 1] = E
    _, _, _, ws = moe.moe_ep_dispatch(x, ids, E, G)
    assert moe.moe_check_status(ws) == 6


@pytest.mark.parametrize("m,hidden,inter,E,top_k,layout", [
    (256, 256, 192, 32, 8, 0),     # 2048 routed rows: the grouped GEMMs
    (200, 136, 72, 8, 4, 1),       # grouped, slotted, ragged widths
    (8, 256, 128, 64, 8, 0),       # 64 routed rows: the streaming kernels
    (600, 256, 128, 4, 4, 0),      # 600 rows per expert: W_down converted up front
])
def test_one_rank_equals_moe_ffn_forward_bits(oracle_mod, m, hidden, inter, E, top_k, layout):
    Wg, Wu, Wd = _layer(m + E, E, hidden, inter)
    x, ids, w = _tokens(m, m, E, top_k, hidden, layout)
    y_ep = host(ep_moe_forward(x, ids, w, Wg, Wu, Wd, E, SelfComm(), layout=layout))
    y = host(moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=layout))
    assert np.array_equal(y_ep.view(np.int32), y.view(np.int32))
    want = oracle_mod.ffn(bits(x), host(ids), host(w), bits(Wg), bits(Wu), bits(Wd), layout=layout)
    assert rel(y_ep, want) <= OUTPUT_REL_TOL


def _run_ranks(G, per_rank_inputs, Wg, Wu, Wd, E, layout):
    hub = LoopbackHub(G)
    out, errors = [None] * G, []
    per = E // G

    def body(rank):
        try:
            x, ids, w = per_rank_inputs[rank]
            loc = slice(rank * per, (rank + 1) * per)
            out[rank] = ep_moe_forward(x, ids, w, Wg[loc], Wu[loc], Wd[loc], E,
                                       LoopbackComm(hub, rank), layout=layout)
            torch.cuda.synchronize()
        except Exception as e:  # surfaced below
            errors.append(e)
            hub.barrier.abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    if errors:
        raise errors[0]
    return out


@pytest.mark.parametrize("G,layout", [(2, 0), (4, 0), (4, 1)])
def test_emulated_ranks_match_single_rank_layer(oracle_mod, G, layout):
    """Each rank's tokens through G expert owners equal moe_ffn_forward on
    those tokens with all experts, bit for bit: every owner receives more
    than 128 rows, so all calls run the grouped GEMMs, whose rows do not
    depend on their neighbours."""
    E, hidden, inter, top_k = 16, 256, 128, 4
    Wg, Wu, Wd = _layer(11, E, hidden, inter)
    ms = [300, 180, 260, 220][:G]
    inputs = [_tokens(20 + r, ms[r], E, top_k, hidden, layout) for r in range(G)]
    ys = _run_ranks(G, inputs, Wg, Wu, Wd, E, layout)
    for r in range(G):
        x, ids, w = inputs[r]
        y1 = host(moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=layout))
        assert np.array_equal(host(ys[r]).view(np.int32), y1.view(np.int32)), r
        want = oracle_mod.ffn(bits(x), host(ids), host(w), bits(Wg), bits(Wu), bits(Wd),
                              layout=layout)
        assert rel(host(ys[r]), want) <= OUTPUT_REL_TOL


def test_emulated_ranks_small_batches_and_repeats(oracle_mod):
    """Decode-size batches (owners take the streaming kernels on a handful of
    rows), a rank with no tokens, and repeated ids: within the output bar of
    the oracle."""
    E, hidden, inter, top_k, G = 8, 128, 64, 4, 2
    Wg, Wu, Wd = _layer(12, E, hidden, inter)
    x0, ids0, w0 = _tokens(30, 6, E, top_k, hidden,
                           ids=moe_inputs.may_repeat_ids(6, E, top_k, "cuda"))
    x1, ids1, w1 = _tokens(31, 0, E, top_k, hidden)
    ys = _run_ranks(G, [(x0, ids0, w0), (x1, ids1, w1)], Wg, Wu, Wd, E, 0)
    assert ys[1].shape == (0, hidden)
    want = oracle_mod.ffn(bits(x0), host(ids0), host(w0), bits(Wg), bits(Wu), bits(Wd))
    assert rel(host(ys[0]), want) <= OUTPUT_REL_TOL

"""GPU matmul by expert id vs the oracle, on both paths (weight streaming for
m*top_k <= 256, tcgen05 grouped GEMM above), both input layouts, ragged
tails, routing profiles, poisoned outputs with a guard, and determinism."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import (OUTPUT_REL_TOL, assert_overwritten_and_guarded, bits, host, poisoned_f32,
                     rel, sample_tokens)

pytestmark = pytest.mark.gpu


def _inputs(seed, m, n, k, E, top_k, layout, w_std=0.05, ids=None):
    g = moe_inputs.generator(seed, "cuda")
    x_rows = m * top_k if layout else m
    x = moe_inputs.bf16_normal((x_rows, k), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, k)
    W = moe_inputs.bf16_normal((E, n, k), w_std, g, "cuda")
    if ids is None:
        ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    return x, W, ids.cuda()


def _run_and_check(oracle_mod, x, W, ids, layout, tokens=None):
    m, top_k = ids.shape
    n = W.shape[1]
    buf, y = poisoned_f32((m, top_k, n))
    moe.moe_matmul_id(x, ids, W, layout=layout, y=y)
    torch.cuda.synchronize()
    assert_overwritten_and_guarded(buf, m * top_k * n)
    got = host(y)
    if tokens is None:
        want = oracle_mod.matmul_id(bits(x), host(ids), bits(W), layout)
        assert rel(got, want) <= OUTPUT_REL_TOL
    else:
        xs = bits(x)[tokens]
        want = oracle_mod.matmul_id(xs, host(ids)[tokens], bits(W), layout)
        assert rel(got[tokens], want) <= OUTPUT_REL_TOL
    return y


# ---------------------------------------------------------------- streaming path
def test_tiny_workload(oracle_mod):
    cfg = moe_inputs.TINY
    inp = moe_inputs.matmul_id_inputs(cfg, seed=0, device="cuda")
    _run_and_check(oracle_mod, inp["x"], inp["W"], inp["ids"], 0)


def test_decode_workload(oracle_mod):
    cfg = moe_inputs.DECODE
    inp = moe_inputs.matmul_id_inputs(cfg, seed=0, device="cuda")
    _run_and_check(oracle_mod, inp["x"], inp["W"], inp["ids"], 0)


@pytest.mark.parametrize("m,n,k,top_k,E,layout", [
    (9, 11, 40, 6, 8, 0),      # tail shape of the mlx-native proof harness, k rounded to 8
    (3, 5, 8, 3, 4, 0),
    (13, 31, 48, 3, 5, 1),
    (18, 41, 56, 3, 5, 0),
    (32, 8, 4096, 8, 8, 0),    # skew-prone: every expert has many rows (several passes)
    (1, 1536, 4096, 8, 256, 1),
])
def test_stream_path_tails(oracle_mod, m, n, k, top_k, E, layout):
    x, W, ids = _inputs(m * 7 + n, m, n, k, E, top_k, layout)
    _run_and_check(oracle_mod, x, W, ids, layout)


# ---------------------------------------------------------------- grouped GEMM path
@pytest.mark.parametrize("m,n,k,top_k,E,layout", [
    (300, 256, 64, 1, 1, 0),     # one expert, full tiles in N and K
    (129, 256, 128, 2, 2, 0),    # ragged M tile
    (300, 80, 136, 2, 8, 0),     # ragged N and K tails
    (300, 37, 40, 3, 5, 0),      # N not a multiple of 4, K below one k-block
    (260, 300, 200, 4, 16, 1),   # slotted layout, two column tiles
    (1000, 512, 512, 8, 64, 0),
])
def test_grouped_path(oracle_mod, m, n, k, top_k, E, layout):
    x, W, ids = _inputs(m + n + k, m, n, k, E, top_k, layout)
    _run_and_check(oracle_mod, x, W, ids, layout)


def test_grouped_prefill_shape_sampled(oracle_mod):
    m, n, k, top_k, E = 4096, 1536, 4096, 8, 256
    x, W, ids = _inputs(11, m, n, k, E, top_k, 0, w_std=0.02)
    _run_and_check(oracle_mod, x, W, ids, 0, tokens=sample_tokens(m, 24))


def test_balanced_and_skewed_rows_bit_identical():
    """Rows shared by the balanced and the maximally skewed routing profile
    have identical bits: reordering rows by expert does not change a row."""
    for (m, n, k, E, top_k) in [(512, 256, 256, 64, 8), (16, 64, 64, 8, 4)]:
        g = moe_inputs.generator(21, "cuda")
        x = moe_inputs.bf16_normal((m, k), 1.0, g, "cuda")
        W = moe_inputs.bf16_normal((E, n, k), 0.05, g, "cuda")
        bal = moe_inputs.balanced_ids(m, E, top_k, "cuda")
        skw = moe_inputs.skewed_ids(m, top_k, "cuda")
        yb = host(moe.moe_matmul_id(x, bal, W))
        ys = host(moe.moe_matmul_id(x, skw, W))
        hb, hs = host(bal), host(skw)
        pairs = 0
        for t in range(m):
            for jb in range(top_k):
                js = np.nonzero(hs[t] == hb[t, jb])[0]
                if len(js):
                    assert np.array_equal(yb[t, jb].view(np.int32), ys[t, js[0]].view(np.int32))
                    pairs += 1
        assert pairs > 0


@pytest.mark.parametrize("m,n,k,top_k,E,layout", [
    (16, 96, 128, 8, 8, 0),      # 128 routed rows: weight streaming
    (32, 41, 56, 8, 8, 1),       # 256 routed rows (the streaming limit), slotted, N tail
    (200, 300, 136, 4, 16, 0),   # 800 routed rows: grouped GEMM, two column tiles
    (130, 80, 64, 3, 7, 1),      # grouped, slotted, partial tiles
    (1024, 256, 256, 2, 2, 0),   # grouped, 1024 rows per expert (8 full m-tiles each)
])
def test_repeated_ids(oracle_mod, m, n, k, top_k, E, layout):
    """mlx-native's MayRepeat profile: every slot of token t picks expert
    t mod E.  Each slot is its own routed row; with the shared-per-token
    layout all slots of a token read the same row through the same expert,
    so they must carry identical bits."""
    ids = moe_inputs.may_repeat_ids(m, E, top_k, "cuda")
    x, W, ids = _inputs(m + 3 * n, m, n, k, E, top_k, layout, ids=ids)
    y = host(_run_and_check(oracle_mod, x, W, ids, layout))
    if layout == 0:
        assert np.array_equal(y.view(np.int32), np.repeat(y[:, :1], top_k, 1).view(np.int32))


def test_repeat_runs_bit_identical():
    x, W, ids = _inputs(5, 700, 384, 256, 32, 4, 0)
    a = host(moe.moe_matmul_id(x, ids, W))
    b = host(moe.moe_matmul_id(x, ids, W))
    assert np.array_equal(a.view(np.int32), b.view(np.int32))


def test_empty_input():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((4, 32, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    y = moe.moe_matmul_id(x, ids, W, ws=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert y.shape == (0, 2, 32)


def test_bad_id_is_reported_and_output_untouched():
    x, W, ids = _inputs(1, 300, 64, 64, 4, 2, 0)
    ids[5, 1] = 4  # out of range
    ws = torch.empty(moe.moe_matmul_id_workspace(300, 64, 64, 2, 4), dtype=torch.uint8,
                     device="cuda")
    buf, y = poisoned_f32((300, 2, 64))
    moe.moe_matmul_id(x, ids, W, y=y, ws=ws)
    assert moe.moe_check_status(ws) == 6
    raw = buf.view(torch.int32).cpu().numpy()
    assert (raw == 0x7FC000C7).all()

"""Pins for the CPU oracle against facts other than its own formulas.

Each test checks the oracle against a closed form, a brute-force search, an
invariant, or a special case that reduces to numpy's dense matmul, chosen so
that a plausible slip (bias added to the logit, bias kept in the weights,
softmax instead of sigmoid, reversed tie order, transposed weight, wrong input
row for the slotted layout, missing up factor, gate/up swapped, combine not
weighted) fails at least one of them.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import moe_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(v):
    return float(np.float32(v))


def _parse_logit(tok):
    if tok.startswith("-ln"):
        return _f32(-math.log(float(tok[3:])))
    if tok.startswith("ln"):
        return _f32(math.log(float(tok[2:])))
    return _f32(float(tok))


def load_route_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "route_closed_form.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "case":
                cur = {"name": vals[0]}
                cases.append(cur)
            elif key == "logits":
                cur["logits"] = [_parse_logit(v) for v in vals]
            elif key == "bias":
                cur["bias"] = [_f32(float(v)) for v in vals]
            elif key == "top_k":
                cur["top_k"] = int(vals[0])
            elif key == "ids":
                cur["ids"] = [int(v) for v in vals]
            elif key == "weights":
                cur["weights"] = [float(Fraction(v)) for v in vals]
    return cases


ROUTE_CASES = load_route_cases()


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("case", ROUTE_CASES, ids=[c["name"] for c in ROUTE_CASES])
def test_route_closed_form(oracle_mod, case):
    logits = np.array([case["logits"]], np.float32)
    bias = np.array(case["bias"], np.float32)
    ids, w, s = oracle_mod.route(logits, bias, case["top_k"])
    assert ids[0].tolist() == case["ids"]
    np.testing.assert_allclose(w[0], case["weights"], rtol=1e-6, atol=1e-7)


def test_sigmoid_closed_forms_and_library(oracle_mod):
    # exact closed forms
    assert oracle_mod.sigmoid_f32(0.0) == 0.5
    assert oracle_mod.sigmoid_f32(_f32(math.log(3.0))) == 0.75
    assert oracle_mod.sigmoid_f32(_f32(-math.log(3.0))) == 0.25
    assert oracle_mod.sigmoid_f32(-200.0) == 0.0
    assert oracle_mod.sigmoid_f32(200.0) == 1.0
    # scipy's logistic function (a library routine), rounded once to f32
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.standard_normal(2000) * 4, [-30.0, -17.5, 17.5, 30.0]]).astype(np.float32)
    got = np.array([oracle_mod.sigmoid_f32(float(v)) for v in xs], np.float32)
    want = scipy.special.expit(xs.astype(np.float64)).astype(np.float32)
    assert np.array_equal(got, want)


def _brute_force_topk(keys, top_k):
    """Pick the set S with |S| = top_k such that every picked expert beats
    every unpicked one in (key desc, index asc); order S the same way."""
    E = len(keys)
    beats = lambda a, b: keys[a] > keys[b] or (keys[a] == keys[b] and a < b)
    winners = [S for S in itertools.combinations(range(E), top_k)
               if all(beats(a, b) for a in S for b in range(E) if b not in S)]
    assert len(winners) == 1
    S = list(winners[0])
    # insertion by pairwise beats (selection sort by the same relation)
    out = []
    while S:
        best = next(a for a in S if all(a == b or beats(a, b) for b in S))
        out.append(best)
        S.remove(best)
    return out


def test_route_brute_force_small(oracle_mod):
    rng = np.random.default_rng(7)
    for trial in range(200):
        E = int(rng.integers(1, 9))
        top_k = int(rng.integers(1, E + 1))
        # coarse values so that ties occur often
        logits = (rng.integers(-3, 4, size=(1, E)) * 0.5).astype(np.float32)
        bias = (rng.integers(-2, 3, size=E) * 0.05).astype(np.float32)
        ids, w, s = oracle_mod.route(logits, bias, top_k)
        keys = (s[0] + bias).astype(np.float32)  # f32 add of score and bias
        assert ids[0].tolist() == _brute_force_topk(keys.tolist(), top_k)
        # weights: picked scores over their sum (ratios and unit sum)
        sel = s[0][ids[0]].astype(np.float64)
        np.testing.assert_allclose(w[0], sel / sel.sum(), rtol=1e-6)


def test_route_weights_ignore_bias_and_sum_to_one(oracle_mod):
    g = moe_inputs.generator(3)
    logits = torch.randn((64, 32), generator=g).numpy()
    b1 = moe_inputs.uniform_bias(32, 0.1, g).numpy()
    ids1, w1, s1 = oracle_mod.route(logits, b1, 4)
    np.testing.assert_allclose(w1.astype(np.float64).sum(1), 1.0, atol=1e-6)
    # bias changes the pick but never the scores; where the picked set and
    # order agree, the weights agree bitwise
    ids0, w0, s0 = oracle_mod.route(logits, None, 4)
    assert np.array_equal(s0, s1)
    same = (ids0 == ids1).all(1)
    assert same.any() and (~same).any()
    assert np.array_equal(w0[same], w1[same])
    # sigmoid (not softmax) scores: weight ratio = score ratio, not exp(logit) ratio
    r = np.arange(64)
    ratio = w1[:, 0].astype(np.float64) / w1[:, 1]
    np.testing.assert_allclose(ratio, s1[r, ids1[:, 0]] / s1[r, ids1[:, 1]], rtol=2e-6)


def test_route_weights_for_forced_ids(oracle_mod):
    g = moe_inputs.generator(4)
    logits = torch.randn((40, 16), generator=g).numpy()
    bias = moe_inputs.uniform_bias(16, 0.1, g).numpy()
    ids, w, _ = oracle_mod.route(logits, bias, 5)
    # forced ids equal to the router's own picks give the router's weights
    assert np.array_equal(oracle_mod.route_weights(logits, ids), w)
    # skewed forced ids: weights of experts 0..4 in slot order
    sk = moe_inputs.skewed_ids(40, 5).numpy()
    ws = oracle_mod.route_weights(logits, sk)
    s = scipy.special.expit(logits.astype(np.float64)).astype(np.float32).astype(np.float64)
    np.testing.assert_allclose(ws, s[:, :5] / s[:, :5].sum(1, keepdims=True), rtol=1e-6)


def test_router_logits_are_a_dense_matmul(oracle_mod):
    g = moe_inputs.generator(19)
    x = moe_inputs.bf16_normal((7, 40), 1.0, g)
    W = moe_inputs.bf16_normal((5, 40), 0.3, g)
    got = oracle_mod.router_logits(_bits(x), _bits(W))
    np.testing.assert_allclose(got, _f64(x) @ _f64(W).T, rtol=1e-12, atol=1e-12)
    # one-hot rows pick columns of W: logits[t, e] = W[e, c_t]
    xo = torch.zeros((3, 40)); xo[0, 2] = 1.0; xo[1, 39] = 1.0; xo[2, 0] = 1.0
    lo = oracle_mod.router_logits(_bits(xo.to(torch.bfloat16)), _bits(W))
    Wf = _f64(W)
    assert np.array_equal(lo[0], Wf[:, 2]) and np.array_equal(lo[1], Wf[:, 39])


# ---------------------------------------------------------------- expert map
def test_expert_map_invariants_and_sort(oracle_mod):
    for (m, top_k, E, seed) in [(1, 1, 1, 0), (37, 3, 5, 1), (200, 8, 64, 2), (33, 2, 100, 3)]:
        g = moe_inputs.generator(seed)
        ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g).numpy()
        counts, offsets, perm, inv = oracle_mod.expert_map(ids, E)
        flat = ids.reshape(-1)
        R = m * top_k
        assert counts.sum() == R and offsets[0] == 0 and offsets[-1] == R
        assert np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(np.sort(perm), np.arange(R))
        assert np.array_equal(inv[perm], np.arange(R))
        # library sort on the key (expert, routed row) gives the same permutation
        assert perm.tolist() == sorted(range(R), key=lambda r: (flat[r], r))
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()


def test_expert_map_rejects_out_of_range(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.expert_map(np.array([[0, 4]], np.int32), 4)


# ---------------------------------------------------------------- matmul_id
def _bits(t):
    return moe_inputs.bf16_bits(t)


def _f64(t):
    return t.to(torch.float64).numpy()


def test_matmul_id_single_expert_is_dense_matmul(oracle_mod):
    g = moe_inputs.generator(5)
    x = moe_inputs.bf16_normal((13, 40), 1.0, g)
    W = moe_inputs.bf16_normal((1, 11, 40), 0.05, g)
    ids = np.zeros((13, 1), np.int32)
    y = oracle_mod.matmul_id(_bits(x), ids, _bits(W), 0)
    want = _f64(x) @ _f64(W[0]).T
    np.testing.assert_allclose(y[:, 0, :], want, rtol=1e-12, atol=1e-12)


def test_matmul_id_each_expert_group_is_dense_matmul(oracle_mod):
    for layout in (0, 1):
        g = moe_inputs.generator(6)
        m, k, n, E, top_k = 9, 48, 11, 8, 6
        x = moe_inputs.bf16_normal((m * top_k if layout else m, k), 1.0, g)
        W = moe_inputs.bf16_normal((E, n, k), 0.05, g)
        ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g).numpy()
        y = oracle_mod.matmul_id(_bits(x), ids, _bits(W), layout).reshape(m * top_k, n)
        xr = _f64(x)
        rows_x = np.arange(m * top_k) if layout else np.repeat(np.arange(m), top_k)
        flat = ids.reshape(-1)
        for e in range(E):
            rr = np.nonzero(flat == e)[0]
            np.testing.assert_allclose(y[rr], xr[rows_x[rr]] @ _f64(W[e]).T, rtol=1e-12, atol=1e-12)


def test_matmul_id_token_permutation_and_layouts(oracle_mod):
    g = moe_inputs.generator(8)
    m, k, n, E, top_k = 12, 32, 16, 6, 3
    x = moe_inputs.bf16_normal((m, k), 1.0, g)
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g)
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g).numpy()
    y = oracle_mod.matmul_id(_bits(x), ids, _bits(W), 0)
    p = np.random.default_rng(0).permutation(m)
    yp = oracle_mod.matmul_id(_bits(x)[p], ids[p], _bits(W), 0)
    assert np.array_equal(yp, y[p])
    # slotted layout with every slot row equal to the token row == shared layout
    xs = np.repeat(_bits(x)[:, None, :], top_k, axis=1)
    assert np.array_equal(oracle_mod.matmul_id(xs, ids, _bits(W), 1), y)


def test_matmul_id_balanced_vs_skewed_rows(oracle_mod):
    g = moe_inputs.generator(9)
    m, k, n, E, top_k = 16, 32, 8, 8, 3
    x = moe_inputs.bf16_normal((m, k), 1.0, g)
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g)
    bal = moe_inputs.balanced_ids(m, E, top_k).numpy()
    skw = moe_inputs.skewed_ids(m, top_k).numpy()
    yb = oracle_mod.matmul_id(_bits(x), bal, _bits(W), 0)
    ys = oracle_mod.matmul_id(_bits(x), skw, _bits(W), 0)
    hits = 0
    for t in range(m):
        for jb in range(top_k):
            for js in range(top_k):
                if bal[t, jb] == skw[t, js]:
                    assert np.array_equal(yb[t, jb], ys[t, js])
                    hits += 1
    assert hits > 0


# ---------------------------------------------------------------- FFN
def _dense_swiglu(x, Wg, Wu, Wd):
    """Dense SwiGLU MLP with numpy matmul and scipy's logistic function."""
    gate = x @ Wg.T
    up = x @ Wu.T
    return (gate * scipy.special.expit(gate) * up) @ Wd.T


def test_ffn_single_expert_is_dense_swiglu(oracle_mod):
    g = moe_inputs.generator(10)
    m, H, I = 5, 24, 16
    x = moe_inputs.bf16_normal((m, H), 1.0, g)
    Wg = moe_inputs.bf16_normal((1, I, H), 0.3, g)
    Wu = moe_inputs.bf16_normal((1, I, H), 0.3, g)
    Wd = moe_inputs.bf16_normal((1, H, I), 0.3, g)
    ids = np.zeros((m, 1), np.int32)
    w = np.ones((m, 1), np.float32)
    y = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd))
    want = _dense_swiglu(_f64(x), _f64(Wg[0]), _f64(Wu[0]), _f64(Wd[0]))
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12)


def test_ffn_one_hot_closed_form(oracle_mod):
    """x = e_0 makes gate/up the first weight column; W_down is a shifted
    permutation (expert 0) or 2*identity (expert 1), so each output is one
    silu(g)*u value in closed form."""
    H = I = 8
    g0 = [1.0, -1.0, 2.0, 0.0, 0.5, -2.0, 3.0, 1.0]
    u0 = [1.0, 0.5, 2.0, 3.0, -1.0, 1.0, 0.25, -0.5]
    Wg = torch.zeros((2, I, H)); Wu = torch.zeros((2, I, H)); Wd = torch.zeros((2, H, I))
    for i in range(I):
        Wg[0, i, 0] = g0[i]; Wu[0, i, 0] = u0[i]
        Wg[1, i, 0] = -g0[i]; Wu[1, i, 0] = u0[i]
    for h in range(H):
        Wd[0, h, (h + 1) % I] = 1.0
        Wd[1, h, h] = 2.0
    x = torch.zeros((1, H)); x[0, 0] = 1.0
    ids = np.array([[1, 0]], np.int32)
    w = np.array([[0.25, 0.75]], np.float32)
    bf = lambda t: _bits(t.to(torch.bfloat16))
    y = oracle_mod.ffn(bf(x), ids, w, bf(Wg), bf(Wu), bf(Wd))
    silu = lambda v: v / (1.0 + math.exp(-v))
    act0 = [silu(g0[i]) * u0[i] for i in range(I)]
    act1 = [silu(-g0[i]) * u0[i] for i in range(I)]
    want = [0.25 * 2.0 * act1[h] + 0.75 * act0[(h + 1) % I] for h in range(H)]
    np.testing.assert_allclose(y[0], want, rtol=1e-15, atol=1e-15)


def _ffn_case(seed, m, H, I, E, top_k, layout=0):
    g = moe_inputs.generator(seed)
    x = moe_inputs.bf16_normal((m * top_k if layout else m, H), 1.0, g)
    Wg = moe_inputs.bf16_normal((E, I, H), 0.2, g)
    Wu = moe_inputs.bf16_normal((E, I, H), 0.2, g)
    Wd = moe_inputs.bf16_normal((E, H, I), 0.2, g)
    return x, Wg, Wu, Wd


def test_ffn_combine_is_weighted_sum_of_single_experts(oracle_mod):
    m, H, I, E, top_k = 6, 16, 8, 4, 2
    x, Wg, Wu, Wd = _ffn_case(11, m, H, I, E, top_k)
    ids = np.array([[0, 3], [1, 2], [2, 0], [3, 1], [0, 1], [2, 3]], np.int32)
    w = np.array([[0.3, 0.7], [0.5, 0.5], [0.9, 0.1], [0.2, 0.8], [1.0, 0.0], [0.25, 0.75]],
                 np.float32)
    y = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd))
    want = np.zeros((m, H))
    for t in range(m):
        for j in range(top_k):
            e = ids[t, j]
            d = _dense_swiglu(_f64(x[t:t + 1]), _f64(Wg[e]), _f64(Wu[e]), _f64(Wd[e]))[0]
            want[t] += float(w[t, j]) * d
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12)


def test_ffn_row_independence_and_subsets(oracle_mod):
    m, H, I, E, top_k = 10, 16, 8, 5, 3
    x, Wg, Wu, Wd = _ffn_case(12, m, H, I, E, top_k)
    g = moe_inputs.generator(13)
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g).numpy()
    w = np.random.default_rng(0).random((m, top_k)).astype(np.float32)
    y = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd))
    sub = np.array([7, 2, 9], np.int32)
    ys = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), tokens=sub)
    assert np.array_equal(ys, y[sub])
    # one token alone gives the same bits as inside the batch
    y1 = oracle_mod.ffn(_bits(x)[4:5], ids[4:5], w[4:5], _bits(Wg), _bits(Wu), _bits(Wd))
    assert np.array_equal(y1[0], y[4])


def test_ffn_slotted_layout(oracle_mod):
    m, H, I, E, top_k = 4, 16, 8, 4, 2
    x, Wg, Wu, Wd = _ffn_case(14, m, H, I, E, top_k, layout=1)
    ids = np.array([[0, 1], [2, 3], [1, 0], [3, 2]], np.int32)
    w = np.full((m, top_k), 0.5, np.float32)
    y = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), layout=1)
    xr = _f64(x).reshape(m, top_k, H)
    for t in range(m):
        want = sum(0.5 * _dense_swiglu(xr[t, j][None], _f64(Wg[ids[t, j]]), _f64(Wu[ids[t, j]]),
                                       _f64(Wd[ids[t, j]]))[0] for j in range(top_k))
        np.testing.assert_allclose(y[t], want, rtol=1e-11, atol=1e-12)


def test_ffn_balanced_vs_skewed_same_rows(oracle_mod):
    m, H, I, E, top_k = 16, 16, 8, 8, 3
    x, Wg, Wu, Wd = _ffn_case(15, m, H, I, E, top_k)
    logits = torch.randn((m, E), generator=moe_inputs.generator(16)).numpy()
    bal = moe_inputs.balanced_ids(m, E, top_k).numpy()
    skw = moe_inputs.skewed_ids(m, top_k).numpy()
    yb = oracle_mod.ffn(_bits(x), bal, oracle_mod.route_weights(logits, bal), _bits(Wg),
                        _bits(Wu), _bits(Wd))
    ys = oracle_mod.ffn(_bits(x), skw, oracle_mod.route_weights(logits, skw), _bits(Wg),
                        _bits(Wu), _bits(Wd))
    same = [t for t in range(m) if t % E == 0]
    assert same and np.array_equal(yb[same], ys[same])
    assert not np.array_equal(yb[1], ys[1])


# ---------------------------------------------------------------- repeated ids
# mlx-native 0.13.0 dense_matmul_id_auto.rs, DenseMatmulIdMultiplicity::MayRepeat:
# a token may name one expert in several slots (its proof profile gives every
# slot of token t the expert t mod E).  Each slot stays its own routed row.
def test_expert_map_with_repeated_ids(oracle_mod):
    m, E, top_k = 11, 4, 3
    ids = moe_inputs.may_repeat_ids(m, E, top_k).numpy()
    counts, offsets, perm, inv = oracle_mod.expert_map(ids, E)
    # token t sends all top_k slots to expert t mod E
    assert counts.tolist() == [top_k * len(range(e, m, E)) for e in range(E)]
    # expert e's rows are the slots of tokens e, e+E, ..., in ascending routed row
    for e in range(E):
        want = [t * top_k + j for t in range(e, m, E) for j in range(top_k)]
        assert perm[offsets[e]:offsets[e + 1]].tolist() == want
    assert np.array_equal(inv[perm], np.arange(m * top_k))


def test_matmul_id_repeated_ids_give_equal_rows(oracle_mod):
    g = moe_inputs.generator(41)
    m, k, n, E, top_k = 7, 24, 9, 3, 4
    x = moe_inputs.bf16_normal((m, k), 1.0, g)
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g)
    ids = moe_inputs.may_repeat_ids(m, E, top_k).numpy()
    y = oracle_mod.matmul_id(_bits(x), ids, _bits(W), 0)
    for t in range(m):
        want = _f64(x[t:t + 1]) @ _f64(W[t % E]).T
        for j in range(top_k):
            np.testing.assert_allclose(y[t, j][None], want, rtol=1e-12, atol=1e-12)
            assert np.array_equal(y[t, j], y[t, 0])  # same row, same expert: same bits
    # slotted: slot j of token t reads its own row, through the repeated expert
    xs = moe_inputs.bf16_normal((m * top_k, k), 1.0, g)
    ys = oracle_mod.matmul_id(_bits(xs), ids, _bits(W), 1)
    xsf = _f64(xs).reshape(m, top_k, k)
    for t in range(m):
        np.testing.assert_allclose(ys[t], xsf[t] @ _f64(W[t % E]).T, rtol=1e-12, atol=1e-12)


def test_ffn_repeated_expert_equals_one_pick_at_the_summed_weight(oracle_mod):
    """Picking expert e in two slots at weights w1, w2 is one pick at w1 + w2
    (the layer is linear in the combine weights); dyadic weights keep w1 + w2
    exact in f32."""
    m, H, I, E = 5, 16, 8, 4
    x, Wg, Wu, Wd = _ffn_case(42, m, H, I, E, 3)
    ids3 = np.array([[1, 1, 2], [0, 3, 0], [2, 2, 2], [3, 0, 3], [1, 2, 1]], np.int32)
    w3 = np.array([[0.25, 0.125, 0.625], [0.5, 0.25, 0.25], [0.5, 0.25, 0.25],
                   [0.375, 0.25, 0.375], [0.125, 0.5, 0.375]], np.float32)
    y3 = oracle_mod.ffn(_bits(x), ids3, w3, _bits(Wg), _bits(Wu), _bits(Wd))
    want = np.zeros((m, H))
    for t in range(m):
        merged = {}
        for j in range(3):
            merged[int(ids3[t, j])] = merged.get(int(ids3[t, j]), 0.0) + float(w3[t, j])
        for e, wsum in merged.items():
            want[t] += wsum * _dense_swiglu(_f64(x[t:t + 1]), _f64(Wg[e]), _f64(Wu[e]),
                                            _f64(Wd[e]))[0]
    np.testing.assert_allclose(y3, want, rtol=1e-11, atol=1e-12)
    # the MayRepeat profile with equal weights 1/top_k is the single expert's MLP
    top_k = 4
    ids = moe_inputs.may_repeat_ids(m, E, top_k).numpy()
    w = np.full((m, top_k), 0.25, np.float32)
    y = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd))
    for t in range(m):
        e = t % E
        np.testing.assert_allclose(
            y[t], _dense_swiglu(_f64(x[t:t + 1]), _f64(Wg[e]), _f64(Wu[e]), _f64(Wd[e]))[0],
            rtol=1e-11, atol=1e-12)


def test_route_weights_with_repeated_ids_are_equal_shares(oracle_mod):
    logits = torch.randn((6, 5), generator=moe_inputs.generator(43)).numpy()
    ids = moe_inputs.may_repeat_ids(6, 5, 4).numpy()
    w = oracle_mod.route_weights(logits, ids)
    # s/(4 s) = 1/4 for every slot, whatever the score
    np.testing.assert_allclose(w, 0.25, rtol=1e-7, atol=0)


def test_ffn_bf16_activation_rounding_is_visible(oracle_mod):
    """Rounding silu(g)*u to bf16 moves the output by a relative error of order
    2^-9, the size that the 1e-3 output bar cannot absorb at real widths."""
    m, H, I, E, top_k = 8, 256, 128, 4, 2
    x, Wg, Wu, Wd = _ffn_case(17, m, H, I, E, top_k)
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, moe_inputs.generator(18)).numpy()
    w = np.full((m, top_k), 0.5, np.float32)
    y0 = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), act_mode=0)
    y1 = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), act_mode=1)
    r = oracle_mod.rel(y1, y0)
    assert 1e-4 < r < 1e-2


def test_ffn_fp16_activation_mode_bound_and_range(oracle_mod):
    """act_mode 2 (the activation as an fp16 down projection with a 2^-4 scale
    sees it): every output moves by at most the fp16 rounding bound of its
    terms, about 8x less than bf16 rounding moves it; and the scale fixes the
    range edge: a = 960 * silu(960) = 921600 survives (57600 in fp16) while
    a = 1024 * silu(1024) = 2^20 overflows (65536 > 65504) -- a scale of the
    wrong sign or none at all would move that edge."""
    m, H, I, E, top_k = 8, 256, 128, 4, 2
    x, Wg, Wu, Wd = _ffn_case(17, m, H, I, E, top_k)
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, moe_inputs.generator(18)).numpy()
    w = np.full((m, top_k), 0.5, np.float32)
    y0 = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), act_mode=0)
    y1 = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), act_mode=1)
    y2 = oracle_mod.ffn(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), act_mode=2)
    bound = np.zeros_like(y0)
    for t in range(m):
        for j in range(top_k):
            e = ids[t, j]
            g = _f64(x[t:t + 1]) @ _f64(Wg[e]).T
            u = _f64(x[t:t + 1]) @ _f64(Wu[e]).T
            a = np.abs(scipy.special.expit(g) * g * u)[0]
            bound[t] += 0.5 * np.abs(_f64(Wd[e])) @ a * (2.0 ** -11 + 2.0 ** -23)
    d2 = np.abs(y2 - y0)
    assert (d2 <= bound).all()
    assert 0 < oracle_mod.rel(y2, y0) < oracle_mod.rel(y1, y0) / 3
    # range edge: E = 1, top_k = 1, g = u = c on every intermediate row,
    # W_down the identity: y = silu(c) * c
    H2 = I2 = 8
    Wg1 = torch.zeros((1, I2, H2)); Wg1[0, :, 0] = 1.0
    Wd1 = torch.eye(H2).reshape(1, H2, I2)
    one = np.zeros((1, 1), np.int32)
    wt = np.ones((1, 1), np.float32)
    for c, finite in ((960.0, True), (1024.0, False)):
        xc = torch.zeros((1, H2)); xc[0, 0] = c
        bf = lambda t: _bits(t.to(torch.bfloat16))  # noqa: E731
        ya = oracle_mod.ffn(bf(xc), one, wt, bf(Wg1), bf(Wg1), bf(Wd1), act_mode=0)
        yb = oracle_mod.ffn(bf(xc), one, wt, bf(Wg1), bf(Wg1), bf(Wd1), act_mode=2)
        assert np.all(ya == c * c)
        if finite:
            assert np.array_equal(yb, ya)
        else:  # the infinite activation meets W_down's zeros: no finite output
            assert not np.isfinite(yb).any()


def _shared_case(seed, m, H, I, I_sh, E, top_k, w_sh_std=0.2):
    g = moe_inputs.generator(seed)
    x, Wg, Wu, Wd = _ffn_case(seed, m, H, I, E, top_k)
    w_sh = moe_inputs.bf16_normal((H,), w_sh_std, g)
    Wsg = moe_inputs.bf16_normal((I_sh, H), 0.2, g)
    Wsu = moe_inputs.bf16_normal((I_sh, H), 0.2, g)
    Wsd = moe_inputs.bf16_normal((H, I_sh), 0.2, g)
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g).numpy()
    w = torch.rand((m, top_k), generator=g).numpy()
    return x, ids, w, (Wg, Wu, Wd), (w_sh, Wsg, Wsu, Wsd)


def test_ffn_shared_is_routed_plus_gated_dense_swiglu(oracle_mod):
    """The shared expert adds expit(x . w_sh) times a dense SwiGLU MLP of its
    own width (numpy matmul, scipy's logistic function) to the routed FFN."""
    m, H, I, I_sh, E, top_k = 7, 24, 8, 12, 5, 2
    x, ids, w, R, S = _shared_case(12, m, H, I, I_sh, E, top_k)
    y = oracle_mod.ffn_shared(_bits(x), ids, w, *[_bits(t) for t in R], *[_bits(t) for t in S])
    routed = oracle_mod.ffn(_bits(x), ids, w, *[_bits(t) for t in R])
    xf = _f64(x)
    gate = scipy.special.expit(xf @ _f64(S[0]))
    dense = _dense_swiglu(xf, _f64(S[1]), _f64(S[2]), _f64(S[3]))
    np.testing.assert_allclose(y - routed, gate[:, None] * dense, rtol=1e-9, atol=1e-12)
    # a token subset gives the same rows
    tok = np.array([5, 0, 3], np.int32)
    sub = oracle_mod.ffn_shared(_bits(x), ids, w, *[_bits(t) for t in R], *[_bits(t) for t in S],
                                tokens=tok)
    assert np.array_equal(sub, y[tok])


def test_ffn_shared_gate_limits(oracle_mod):
    """w_sh = 0 halves the shared MLP exactly; a one-hot token with a logit of
    +256 adds it whole and one of -256 leaves the routed result."""
    m, H, I, I_sh, E, top_k = 3, 16, 8, 8, 4, 2
    x, ids, w, R, S = _shared_case(13, m, H, I, I_sh, E, top_k)
    Rb = [_bits(t) for t in R]
    _, Wsg, Wsu, Wsd = S
    dense = _dense_swiglu(_f64(x), _f64(Wsg), _f64(Wsu), _f64(Wsd))
    routed = oracle_mod.ffn(_bits(x), ids, w, *Rb)
    zero = torch.zeros(H, dtype=torch.bfloat16)
    y0 = oracle_mod.ffn_shared(_bits(x), ids, w, *Rb, _bits(zero), _bits(Wsg), _bits(Wsu),
                               _bits(Wsd))
    np.testing.assert_allclose(y0 - routed, 0.5 * dense, rtol=1e-9, atol=1e-12)
    x1 = torch.zeros((2, H), dtype=torch.bfloat16)
    x1[:, 3] = 2.0
    ids1, w1 = ids[:2], w[:2]
    for sign in (1.0, -1.0):
        w_sh = torch.zeros(H, dtype=torch.bfloat16)
        w_sh[3] = 128.0 * sign
        y1 = oracle_mod.ffn_shared(_bits(x1), ids1, w1, *Rb, _bits(w_sh), _bits(Wsg),
                                   _bits(Wsu), _bits(Wsd))
        r1 = oracle_mod.ffn(_bits(x1), ids1, w1, *Rb)
        d1 = _dense_swiglu(_f64(x1), _f64(Wsg), _f64(Wsu), _f64(Wsd))
        np.testing.assert_allclose(y1, r1 + (d1 if sign > 0 else 0.0), rtol=1e-12, atol=1e-12)


def test_ffn_shared_as_an_extra_routed_expert(oracle_mod):
    """With inter_sh == inter the shared expert is a routed expert appended to
    the stack, picked last by every token with weight sigmoid(x . w_sh)."""
    m, H, I, E, top_k = 6, 16, 8, 4, 2
    x, ids, w, (Wg, Wu, Wd), (w_sh, Wsg, Wsu, Wsd) = _shared_case(14, m, H, I, I, E, top_k)
    y = oracle_mod.ffn_shared(_bits(x), ids, w, _bits(Wg), _bits(Wu), _bits(Wd), _bits(w_sh),
                              _bits(Wsg), _bits(Wsu), _bits(Wsd))
    ids2 = np.concatenate([ids, np.full((m, 1), E, np.int32)], axis=1)
    gate = scipy.special.expit(_f64(x) @ _f64(w_sh))
    w2 = np.concatenate([w, gate[:, None]], axis=1)  # rounded to f32 by the routed oracle
    y2 = oracle_mod.ffn(_bits(x), ids2, w2.astype(np.float32),
                        _bits(torch.cat([Wg, Wsg[None]])), _bits(torch.cat([Wu, Wsu[None]])),
                        _bits(torch.cat([Wd, Wsd[None]])))
    np.testing.assert_allclose(y, y2, rtol=1e-6, atol=1e-9)


def test_rel_metric(oracle_mod):
    assert oracle_mod.rel([1.0, 2.0], [1.0, 2.0]) == 0.0
    assert oracle_mod.rel([1.0, 2.5], [1.0, 2.0]) == 0.25
    assert oracle_mod.rel([float("nan")], [1.0]) == float("inf")

"""The documented maximum of routed rows (m * top_k = 2^24) on both the
matmul-by-id and the FFN path, with narrow rows so the buffers stay a few GB;
sampled rows against the oracle (rows are independent given ids and
weights).  One row more is rejected on the host."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, bits, host, rel, sample_tokens

pytestmark = pytest.mark.gpu

M, TOP_K, E = 1 << 21, 8, 1024     # 2^24 routed rows over 1024 experts


def test_matmul_id_at_max_routed_rows(oracle_mod):
    k, n = 64, 32
    g = moe_inputs.generator(41, "cuda")
    x = moe_inputs.bf16_normal((M, k), 1.0, g, "cuda")
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g, "cuda")
    ids = moe_inputs.balanced_ids(M, E, TOP_K, "cuda")
    y = moe.moe_matmul_id(x, ids, W)
    torch.cuda.synchronize()
    tok = sample_tokens(M, 30, seed=2)
    want = oracle_mod.matmul_id(bits(x[torch.from_numpy(tok).cuda()]), host(ids)[tok], bits(W), 0)
    assert rel(host(y[torch.from_numpy(tok).cuda()]), want) <= OUTPUT_REL_TOL
    with pytest.raises(moe.MoeError):
        moe.moe_matmul_id(torch.zeros((M + 1, k), dtype=torch.bfloat16, device="cuda"),
                          torch.zeros((M + 1, TOP_K), dtype=torch.int32, device="cuda"), W)


def test_ffn_at_max_routed_rows(oracle_mod):
    hidden, inter = 64, 64
    g = moe_inputs.generator(42, "cuda")
    x = moe_inputs.bf16_normal((M, hidden), 1.0, g, "cuda")
    Wg = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wu = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wd = moe_inputs.bf16_normal((E, hidden, inter), 0.05, g, "cuda")
    ids = moe_inputs.balanced_ids(M, E, TOP_K, "cuda")
    w = torch.rand((M, TOP_K), generator=g, device="cuda")
    y = moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd)
    torch.cuda.synchronize()
    tok = sample_tokens(M, 30, seed=3)
    tt = torch.from_numpy(tok).cuda()
    want = oracle_mod.ffn(bits(x[tt]), host(ids)[tok], host(w)[tok], bits(Wg), bits(Wu), bits(Wd))
    got = host(y[tt])
    assert np.isfinite(got).all()
    assert rel(got, want) <= OUTPUT_REL_TOL

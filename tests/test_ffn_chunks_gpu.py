"""Experts whose routed-row counts sit at and around the 128-row tile edges
(one row over a tile, exactly two tiles, 511/512 rows, a lone small expert,
and 64/65 rows: the edge between the down projection's swapped form for
tiles of at most 64 rows and its plain form; 512 rows is also the edge at
which an expert's W_down is converted to fp16 once before the down GEMM
instead of in shared memory by every tile): every row against the oracle,
and a token's per-slot bits independent of how many other rows its expert
got (a 200-token sub-batch, every expert within one tile of at most 64 rows,
recomputes rows that the full batch put in full and partial tiles)."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import FP16_ACT_TOL, OUTPUT_REL_TOL, bits, host, rel

pytestmark = pytest.mark.gpu

COUNTS = [128, 129, 300, 511, 512, 20, 256, 257, 64, 65]   # rows per expert, top_k = 1


def _layer(hidden=256, inter=192, seed=31):
    E = len(COUNTS)
    m = sum(COUNTS)
    g = moe_inputs.generator(seed, "cuda")
    x = moe_inputs.bf16_normal((m, hidden), 1.0, g, "cuda")
    Wg = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wu = moe_inputs.bf16_normal((E, inter, hidden), 0.05, g, "cuda")
    Wd = moe_inputs.bf16_normal((E, hidden, inter), 0.05, g, "cuda")
    ids = torch.repeat_interleave(torch.arange(E, dtype=torch.int32), torch.tensor(COUNTS))
    ids = ids[torch.randperm(m, generator=torch.Generator().manual_seed(seed))]
    ids = ids.view(m, 1).contiguous().cuda()
    w = torch.rand((m, 1), generator=g, device="cuda")
    return x, ids, w, (Wg, Wu, Wd)


def test_boundary_counts_match_oracle(oracle_mod):
    x, ids, w, W = _layer()
    y = moe.moe_ffn_forward(x, ids, w, *W)
    torch.cuda.synchronize()
    want = oracle_mod.ffn(bits(x), host(ids), host(w), *[bits(t) for t in W])
    assert rel(host(y), want) <= OUTPUT_REL_TOL
    # against the oracle's rounding of the activation to fp16(a * 2^-4)
    want2 = oracle_mod.ffn(bits(x), host(ids), host(w), *[bits(t) for t in W], act_mode=2)
    assert rel(host(y), want2) <= FP16_ACT_TOL


def test_bits_independent_of_expert_row_count():
    """Tokens of every expert, recomputed in a 200-token call where no expert
    has more than 64 rows (every tile in the down projection's swapped form),
    keep the per-slot bits the full batch gave them in full 128-row tiles
    (plain form) and in partial tiles."""
    x, ids, w, W = _layer()
    d_all = host(moe.moe_ffn_slots(x, ids, *W))
    sub = torch.randperm(x.shape[0], generator=torch.Generator().manual_seed(5))[:200]
    sub = sub.sort().values.cuda()
    counts = torch.bincount(ids[sub].view(-1).long(), minlength=len(COUNTS))
    assert int(counts.max()) <= 64
    d_sub = host(moe.moe_ffn_slots(x[sub].contiguous(), ids[sub].contiguous(), *W))
    assert np.array_equal(d_sub.view(np.int32), d_all[host(sub)].view(np.int32))

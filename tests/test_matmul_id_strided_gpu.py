"""GPU matmul by expert id over a padded expert stack (experts at a stride
larger than n*k*2 bytes) vs the oracle on the dense experts, on both paths.
The padding is filled with NaN bits, so a read of it would show in y."""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, assert_overwritten_and_guarded, bits, host, poisoned_f32, rel

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC1  # quiet NaN bit pattern


def _padded_stack(W, stride_bytes):
    """Copy the dense stack W [E, n, k] into a buffer whose experts start
    stride_bytes apart, with every padding element set to NaN."""
    E, n, k = W.shape
    per = stride_bytes // 2
    buf = torch.full((E * per,), NAN_BF16, dtype=torch.int16, device=W.device)
    buf = buf.view(torch.bfloat16)
    buf.view(E, per)[:, : n * k] = W.reshape(E, n * k)
    return buf


@pytest.mark.parametrize("m,n,k,top_k,E,layout,pad", [
    (9, 11, 40, 6, 8, 0, 16),        # streaming path; 880 -> 896 bytes per expert
    (13, 31, 48, 3, 5, 1, 4096),     # streaming, slotted, a page of padding
    (300, 37, 40, 3, 5, 0, 48),      # grouped path, N below one column tile
    (260, 300, 200, 4, 16, 1, 256),  # grouped, slotted, two column tiles, ragged K
    (1000, 512, 512, 8, 64, 0, 16),
])
def test_strided_matches_oracle(oracle_mod, m, n, k, top_k, E, layout, pad):
    stride = n * k * 2 + pad
    g = moe_inputs.generator(m + n + pad, "cuda")
    x = moe_inputs.bf16_normal((m * top_k if layout else m, k), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, k)
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g, "cuda")
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    buf = _padded_stack(W, stride)
    out, y = poisoned_f32((m, top_k, n))
    moe.moe_matmul_id_strided(x, ids, buf, stride, n, k, E, layout=layout, y=y)
    torch.cuda.synchronize()
    assert_overwritten_and_guarded(out, m * top_k * n)
    got = host(y)
    assert np.isfinite(got).all()
    want = oracle_mod.matmul_id(bits(x), host(ids), bits(W), layout)
    assert rel(got, want) <= OUTPUT_REL_TOL
    # same bits as the dense entry point on the dense copy of the stack
    dense = host(moe.moe_matmul_id(x, ids, W, layout=layout))
    assert np.array_equal(got.view(np.int32), dense.view(np.int32))


def test_dense_stride_equals_moe_matmul_id():
    m, n, k, top_k, E = 400, 96, 64, 4, 16
    g = moe_inputs.generator(9, "cuda")
    x = moe_inputs.bf16_normal((m, k), 1.0, g, "cuda")
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g, "cuda")
    ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    a = host(moe.moe_matmul_id_strided(x, ids, W, n * k * 2, n, k, E))
    b = host(moe.moe_matmul_id(x, ids, W))
    assert np.array_equal(a.view(np.int32), b.view(np.int32))

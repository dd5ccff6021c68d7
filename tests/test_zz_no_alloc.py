"""moe_matmul_id_noalloc against moe_matmul_id.

moe_matmul_id_noalloc serves callers that cannot allocate device memory --
a plugin whose host runtime owns every allocation, or a decode loop that must
never enter the driver's allocator.  Instead of a caller workspace it keeps
the expert-map scratch in a static device array shared by all its calls.
These tests call it through the C ABI and compare it with the workspace entry
point.  The file sorts last so that, in a run that stops at the first
failure, every other test has already run.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, rel

FAKE = 0x10000  # aligned, non-null, never dereferenced by a rejected call


def _noalloc(x, ids, W, y, layout=0):
    lib = moe.load_library()
    m, top_k = ids.shape
    n_experts, n, k = W.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.moe_matmul_id_noalloc(x.data_ptr(), ids.data_ptr(), W.data_ptr(), y.data_ptr(),
                                     m, n, k, top_k, n_experts, layout, stream)


def test_noalloc_rejects_shapes_beyond_its_static_scratch():
    lib = moe.load_library()
    # 33 tokens x top-8 = 264 routed rows > 256
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 33, 64, 64, 8, 16, 0, None) == 2
    assert b"256" in lib.moe_last_error()
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 4, 64, 37, 2, 8, 0, None) == 2
    assert lib.moe_matmul_id_noalloc(None, FAKE, FAKE, FAKE, 4, 64, 64, 2, 8, 0, None) == 1
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 0, 64, 64, 2, 8, 0, None) == 0


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    # Two calls in a row with different shapes and inputs: the second must
    # not see anything the first left in the shared static scratch.
    cases = [
        (moe_inputs.DECODE, 0, None),                 # m=8, k=4096, n=1536, 256 experts, top-8
        (moe_inputs.TINY, 1, 32),                     # 32 tokens, 8 experts, top-2, other weights
    ]
    for cfg, seed, m in cases:
        inp = moe_inputs.matmul_id_inputs(cfg, seed=seed, device="cuda", m=m)
        want = moe.moe_matmul_id(inp["x"], inp["ids"], inp["W"])
        y = torch.full_like(want, float("nan"))
        assert _noalloc(inp["x"], inp["ids"], inp["W"], y) == 0, moe.load_library().moe_last_error()
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert np.isfinite(got).all()
        assert rel(got, want.cpu().numpy()) <= OUTPUT_REL_TOL

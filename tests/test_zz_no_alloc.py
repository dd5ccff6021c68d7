"""moe_matmul_id_noalloc against the oracle and the workspace entry point.

moe_matmul_id_noalloc serves callers that cannot allocate device memory --
a plugin whose host runtime owns every allocation, or a decode loop that must
never enter the driver's allocator.  Instead of a caller workspace it keeps
the expert-map scratch in a static device array shared by all its calls.
These tests call it through the C ABI, check every output element against
the CPU oracle and the bits against moe_matmul_id (same kernels), and read
its device status word through moe_matmul_id_noalloc_status.  The file sorts
last so that, in a run that stops at the first failure, every other test has
already run.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe
from helpers import OUTPUT_REL_TOL, bits, host, poisoned_f32, rel

FAKE = 0x10000  # aligned, non-null, never dereferenced by a rejected call


def _noalloc(x, ids, W, y, layout=0):
    lib = moe.load_library()
    m, top_k = ids.shape
    n_experts, n, k = W.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.moe_matmul_id_noalloc(x.data_ptr(), ids.data_ptr(), W.data_ptr(), y.data_ptr(),
                                     m, n, k, top_k, n_experts, layout, stream)


def _status():
    return moe.load_library().moe_matmul_id_noalloc_status(torch.cuda.current_stream().cuda_stream)


def test_noalloc_rejects_shapes_beyond_its_static_scratch():
    lib = moe.load_library()
    # 33 tokens x top-8 = 264 routed rows > 256
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 33, 64, 64, 8, 16, 0, None) == 2
    assert b"256" in lib.moe_last_error()
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 4, 64, 37, 2, 8, 0, None) == 2
    assert lib.moe_matmul_id_noalloc(None, FAKE, FAKE, FAKE, 4, 64, 64, 2, 8, 0, None) == 1
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 4, 64, 64, 2, 8, 2, None) == 1
    assert lib.moe_matmul_id_noalloc(FAKE, FAKE, FAKE, FAKE, 0, 64, 64, 2, 8, 0, None) == 0


def _case(name, seed):
    """(x, W, ids, layout) of one named case."""
    if name == "decode":       # m=8, k=4096, n=1536, 256 experts, top-8
        inp = moe_inputs.matmul_id_inputs(moe_inputs.DECODE, seed=seed, device="cuda")
        return inp["x"], inp["W"], inp["ids"], 0
    shapes = {
        "tiny64": (32, 32, 64, 8, 2, 0),       # 64 routed rows, 8 experts
        "slotted": (16, 96, 128, 16, 4, 1),    # x [m, top_k, k]
        "rows256": (32, 128, 256, 64, 8, 0),   # the routed-row limit
        "e1024": (8, 64, 128, 1024, 32, 0),    # the largest expert count and top_k: biggest carve
        "repeat": (32, 64, 128, 16, 8, 0),     # every slot of token t picks expert t % E
    }
    m, n, k, E, top_k, layout = shapes[name]
    g = moe_inputs.generator(seed, "cuda")
    x = moe_inputs.bf16_normal((m * top_k if layout else m, k), 1.0, g, "cuda")
    if layout:
        x = x.view(m, top_k, k)
    W = moe_inputs.bf16_normal((E, n, k), 0.05, g, "cuda")
    if name == "repeat":
        ids = moe_inputs.may_repeat_ids(m, E, top_k, "cuda")
    else:
        ids = moe_inputs.uniform_distinct_ids(m, E, top_k, g, "cuda")
    return x, W, ids, layout


@pytest.mark.gpu
@pytest.mark.parametrize("pair", [("decode", "tiny64"), ("slotted", "rows256"),
                                  ("e1024", "repeat"), ("rows256", "e1024")])
def test_noalloc_matches_oracle_and_workspace_entry_on_two_calls_in_a_row(oracle_mod, pair):
    # Two calls in a row with different shapes and inputs: the second must
    # not see anything the first left in the shared static scratch.
    for i, name in enumerate(pair):
        x, W, ids, layout = _case(name, seed=i + 1)
        m, top_k = ids.shape
        n = W.shape[1]
        buf, y = poisoned_f32((m, top_k, n))
        assert _noalloc(x, ids, W, y, layout) == 0, moe.load_library().moe_last_error()
        assert _status() == 0
        torch.cuda.synchronize()
        got = host(y)
        assert np.isfinite(got).all()
        assert (buf.view(torch.int32)[m * top_k * n:].cpu().numpy() == 0x7FC000C7).all()
        want = oracle_mod.matmul_id(bits(x), host(ids), bits(W), layout)
        assert rel(got, want) <= OUTPUT_REL_TOL, name
        ref = host(moe.moe_matmul_id(x, ids, W, layout=layout))
        assert np.array_equal(got.view(np.int32), ref.view(np.int32)), name


@pytest.mark.gpu
def test_noalloc_bad_id_is_reported_and_the_next_call_is_clean(oracle_mod):
    x, W, ids, layout = _case("tiny64", seed=5)
    E = W.shape[0]
    bad = ids.clone()
    bad[3, 1] = E  # outside [0, n_experts)
    m, top_k = ids.shape
    buf, y = poisoned_f32((m, top_k, W.shape[1]))
    assert _noalloc(x, bad, W, y, layout) == 0  # device-side error: found by the kernels
    assert _status() == 6                        # MOE_ERR_DEVICE_BAD_ID
    assert (buf.view(torch.int32).cpu().numpy() == 0x7FC000C7).all(), "y was written"
    # the following valid call clears the word and computes the right rows
    assert _noalloc(x, ids, W, y, layout) == 0
    assert _status() == 0
    want = oracle_mod.matmul_id(bits(x), host(ids), bits(W), layout)
    assert rel(host(y), want) <= OUTPUT_REL_TOL

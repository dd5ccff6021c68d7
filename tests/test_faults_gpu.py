"""Failure detection on the GPU without faulting it: the bounded barrier wait
gives up after its limit, records MOE_ERR_DEVICE_TIMEOUT and returns, and the
CUDA context stays usable."""
import time

import numpy as np
import pytest
import torch

import mixture_experts_routed_sigmoid_b200 as moe

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.moe_selftest_wait_timeout(status, 50_000_000)  # 50 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == 5  # MOE_ERR_DEVICE_TIMEOUT
    assert elapsed < 5.0
    # the context still runs work
    ids, w = moe.moe_route_topk(torch.zeros((4, 8), device="cuda"), None, 2)
    assert np.array_equal(ids.cpu().numpy(), [[0, 1]] * 4)


def test_invalid_arguments_raise_before_launch():
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route_topk(torch.zeros((4, 8), device="cuda"), None, 9)
    assert e.value.status == 2

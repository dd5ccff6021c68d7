"""Failure detection on the GPU without faulting it: the bounded barrier wait
gives up after its limit, records MOE_ERR_DEVICE_TIMEOUT and returns, and the
CUDA context stays usable.  Also the clock probe the benchmark uses to read
the SM clock over a timed region."""
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


def test_clock_probe_measures_the_sm_clock():
    """Two probes around a kernel that spins a known number of cycles: the
    SM clock they report over the interval is a plausible B200 clock and the
    cycle delta covers the spin."""
    n = torch.cuda.get_device_properties(0).multi_processor_count
    a = torch.zeros((n, 3), dtype=torch.int64, device="cuda")
    b = torch.zeros((n, 3), dtype=torch.int64, device="cuda")
    moe.moe_clock_probe(a)
    torch.cuda._sleep(20_000_000)  # ~10 ms of spinning at ~2 GHz
    moe.moe_clock_probe(b)
    torch.cuda.synchronize()
    mhz = moe.probe_clock_mhz(a, b)
    assert mhz is not None and 300.0 <= mhz <= 3000.0, mhz
    ha, hb = a.cpu().numpy(), b.cpu().numpy()
    assert (ha[:, 0] < n).all() and (hb[:, 2] >= ha[:, 2].min()).all()

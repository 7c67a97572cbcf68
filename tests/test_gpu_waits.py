"""The bounded device waits end with an error status, not a hang.

The histogram/scan's look-back waits for the running totals of earlier chunks of tokens,
and every such wait gives up after a limit.  moe_scan_wait_check runs the same kernels
with the first chunk withheld, so that the waits of every later chunk find a word nobody
publishes: they must run out after the given limit, record MOE_DEVERR_SCAN_TIMEOUT and let
the kernels finish, and the context must stay usable (the next ordinary call is exact).
Nothing here traps or faults a GPU.
"""
import time

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from routing_dispatch_expert_moe_b200 import moe
    moe.lib()
    return moe


def _routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    gate = torch.rand((T, k), generator=g, dtype=torch.float32)
    return idx, gate


@pytest.mark.parametrize("T,E,k,wait_ns", [(4096, 64, 4, 2_000_000), (1000, 300, 8, 200_000)])
def test_scan_lookback_wait_runs_out_and_the_context_survives(M, T, E, k, wait_ns):
    idx, gate = _routing(T, E, k, seed=T)
    di, dg = idx.cuda(), gate.cuda()
    M.moe_get_device_error()                                   # start from a clear error word
    t0 = time.perf_counter()
    M.moe_scan_wait_check(di, dg, E, wait_ns)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert M.moe_get_device_error() == 4, "the withheld chunk's waiters must report MOE_DEVERR_SCAN_TIMEOUT"
    assert elapsed < 5.0                                       # bounded: a few limits, not the 1 s default
    # the next ordinary call runs normally and exactly
    r = M.moe_histogram_scan(di, dg, E, -1)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    o = O.dispatch_plan(idx.numpy(), gate.numpy().astype(np.float64), E, -1)
    for key in ("counts", "kept", "offsets", "row_of"):
        assert np.array_equal(r[key].cpu().numpy(), o[key]), key

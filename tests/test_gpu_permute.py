"""GPU parity of the permute (dispatch copy) through the C ABI, across row widths and k:
the bulk-copy kernel (rows staged in shared memory) and, for rows too long for its
buffers, the per-vector copy.  x_perm must equal the oracle's permute bit for bit on
every kept row; rows of the buffer past the kept ones are not written.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from routing_dispatch_expert_moe_b200 import moe
    moe.lib()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _plan(T, E, k, cap, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int64)
    gate = np.ones((T, k))
    return O.dispatch_plan(idx, gate, E, cap)


# (T, d, dtype, E, k, cap): 7168- and 2048-wide bf16 rows and 64-wide fp32 rows take the
# bulk copies; 10240-wide bf16 and 5120-wide fp32 rows (20 KB) exceed the buffers and
# take the per-vector copy.  Capacities drop some assignments; T not a multiple of the
# warps per block.
CASES = [
    (1, 2048, torch.bfloat16, 8, 1, -1),
    (37, 7168, torch.bfloat16, 16, 4, 9),
    (1000, 2048, torch.bfloat16, 64, 8, 100),
    (333, 64, torch.float32, 40, 32, -1),
    (129, 10240, torch.bfloat16, 12, 3, 20),
    (70, 5120, torch.float32, 9, 2, 11),
]


@pytest.mark.parametrize("T,d,dtype,E,k,cap", CASES)
def test_permute_equals_the_oracle_bit_for_bit(T, d, dtype, E, k, cap):
    from routing_dispatch_expert_moe_b200 import moe as M
    p = _plan(T, E, k, cap, seed=T + d + k)
    n = int(p["offsets"][-1])
    rows_max = M.moe_rows_max(T, E, k, cap)
    assert n <= rows_max
    rng = np.random.default_rng(d)
    x = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(dtype).cuda()
    row_of = torch.from_numpy(p["row_of"].astype(np.int32)).cuda()
    x_perm = torch.full((max(rows_max, 1), d), 7.0, dtype=dtype, device="cuda")   # sentinel
    M.moe_permute(x, row_of, rows_max, x_perm)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    want = O.permute(x.float().cpu().numpy(), p["row_of"], n)
    got = x_perm[:n].float().cpu().numpy()
    assert np.array_equal(got, want)
    if rows_max > n:                                        # rows past the kept ones untouched
        assert torch.all(x_perm[n:rows_max] == 7.0)
    if cap >= 0:
        assert (p["row_of"] < 0).any(), "the case must drop assignments"

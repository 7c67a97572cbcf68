"""The expert-parallel forward with the library's kernels on one GPU (a one-rank NCCL group).

Every step runs in the library (router, scan with per-expert capacity from the host plan,
permute, regroup, the grouped GEMMs of the rank's experts, combine with the gates); the
all-to-all is NCCL's.  With one rank the exchange moves nothing between GPUs, but the
whole path runs, and its result must match the oracle layer: routing bit-exact, outputs
within the layer's bars.  The multi-rank exchange and plan are covered on the CPU
(tests/test_ep_cpu.py) with two and three gloo ranks.
"""
import datetime
import socket

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_moe_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    torch.cuda.synchronize()
    dist.destroy_process_group()


CASES = [
    I.small_config("ep_softmax", T=300, d=128, E=16, k=4, F=128),
    I.small_config("ep_capacity_zipf", T=1000, d=256, E=32, k=6, F=64, score="sqrt_softplus", capacity_factor=1.0,
                   logit_offset="zipf1.2"),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_expert_parallel_one_rank_matches_the_oracle(group, cfg):
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.ep import ExpertParallelMoE
    host, dev = U.make_inputs(cfg)
    cap = O.capacity(cfg.T, cfg.E, cfg.k, cfg.capacity_factor, True)
    lay = ExpertParallelMoE(dev["Wg"], dev["W_gu"], dev["W_dn"], cfg.k, cfg.score, cfg.renormalize, cfg.scale, cap,
                            dev["off"], group=group)
    y = lay.forward(dev["x"])
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    o = O.layer_routing(U.cfg_dict(cfg), host["x"], host["Wg"], host["off"], None, True)
    assert np.array_equal(lay.routing["topk_idx"].cpu().numpy(), o["topk_idx"])
    assert np.array_equal(lay.routing["row_of"].cpu().numpy(), o["row_of"])
    gu, dn = U.expert_getters(host)
    n = int(o["offsets"][-1])
    yp = O.grouped_ffn(O.permute(host["x"], o["row_of"], n), o["offsets"], gu, dn, o["gate_of_row"], True)
    U.assert_y_close(y.float().cpu().numpy().astype(np.float64), O.combine(yp, o["row_of"]), "y (expert-parallel)")


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_peer_exchange_one_rank_equals_the_nccl_exchange(group, cfg):
    """exchange='peer' (moe_ep_dispatch / moe_ep_combine into the owners' buffers) against
    exchange='nccl' on the same inputs: the same rows through the same GEMMs and the same
    fp32 sums, so y agrees bit for bit."""
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.ep import ExpertParallelMoE
    host, dev = U.make_inputs(cfg)
    cap = O.capacity(cfg.T, cfg.E, cfg.k, cfg.capacity_factor, True)
    args = (dev["Wg"], dev["W_gu"], dev["W_dn"], cfg.k, cfg.score, cfg.renormalize, cfg.scale, cap, dev["off"])
    y_n = ExpertParallelMoE(*args, group=group).forward(dev["x"])
    lay = ExpertParallelMoE(*args, group=group, exchange="peer", max_tokens=cfg.T)
    y_p = lay.forward(dev["x"])
    y_p2 = lay.forward(dev["x"])                                   # the buffers are reused
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    assert torch.equal(y_n, y_p) and torch.equal(y_p, y_p2)
    lay.close()

"""Host-side checks of MoELayer's arguments and of its launch count (no GPU).

The argument checks run before the constructor touches any device memory, so CPU
tensors stand in for the weights.
"""
import types

import pytest
import torch

from routing_dispatch_expert_moe_b200.layer import MoELayer, MoEWeights


def _weights(E=8, d=64, F=64, **kw):
    return MoEWeights(Wg=torch.zeros(d, E), W_gu=torch.zeros(E, 2 * F, d, dtype=torch.bfloat16),
                      W_dn=torch.zeros(E, d, F, dtype=torch.bfloat16), **kw)


@pytest.mark.parametrize("kw,msg", [
    (dict(routing="random"), "routing must be"),
    (dict(routing="uniform", select_bias=True), "selection bias"),
    (dict(routing="hash", select_bias=True), "selection bias"),
    (dict(routing="noisy"), "W_noise"),
    (dict(routing="noisy", W_noise=True, score="sigmoid"), "softmax"),
    (dict(dispatch="scatter"), "dispatch"),
    (dict(combine="atomic"), "combine"),
    (dict(out_dtype=torch.float16), "out_dtype"),
])
def test_layer_rejects_bad_arguments_before_allocating(kw, msg):
    wkw = {}
    if kw.pop("select_bias", False):
        wkw["select_bias"] = torch.zeros(8)
    if kw.pop("W_noise", False):
        wkw["W_noise"] = torch.zeros(64, 8)
    score = kw.pop("score", "softmax")
    with pytest.raises(ValueError, match=msg):
        MoELayer(_weights(**wkw), 2, 16, score, **kw)


class _Stub:
    """The attributes launches_per_forward reads, without building a layer."""
    launches_per_forward = MoELayer.launches_per_forward
    _route_launches = MoELayer._route_launches

    def __init__(self, routing="learned", dtype=torch.bfloat16, d=2048, E=64, combine="rows", dispatch="permute",
                 shared=False, fused_bf16=False, T_max=8192, score="softmax", bias=False):
        self.routing, self.dtype, self.d, self.E = routing, dtype, d, E
        self.combine_mode, self.dispatch_mode, self.has_shared = combine, dispatch, shared
        self.T_max, self.score = T_max, score
        self.w = types.SimpleNamespace(select_bias=torch.zeros(E) if bias else None)
        self.y = object()
        self.y32 = object() if fused_bf16 else self.y


def test_launch_count_matches_the_kernels_each_form_runs():
    # handbook default: the tensor-core router with the top-k in its epilogue, rank +
    # scatter, permute, gate/up, down, combine; statistics partials, per-expert sums and
    # scalars (10 kernels)
    assert _Stub().launches_per_forward(True) == 10
    assert _Stub().launches_per_forward(False) == 7
    assert _Stub(dtype=torch.float32).launches_per_forward(True) == 11       # SIMT router GEMM + top-k
    assert _Stub(E=37).launches_per_forward(True) == 11                      # E % 4: SIMT router
    assert _Stub(T_max=200).launches_per_forward(True) == 11                 # under 256 tokens: SIMT router
    assert _Stub(score="softmax", bias=True).launches_per_forward(True) == 11   # + a separate top-k pass
    assert _Stub(score="sigmoid", bias=True).launches_per_forward(True) == 10    # biased keys fused
    assert _Stub(routing="uniform").launches_per_forward(True) == 11         # router logits -> fixed selection
    assert _Stub(routing="noisy").launches_per_forward(True) == 13           # two router GEMMs + H + top-k
    assert _Stub(combine="fused").launches_per_forward(True) == 9
    assert _Stub(combine="fused", fused_bf16=True).launches_per_forward(True) == 10
    assert _Stub(dispatch="gather").launches_per_forward(True) == 9
    assert _Stub(shared=True).launches_per_forward(True) == 12

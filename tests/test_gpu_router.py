"""GPU parity of the tensor-core router with weights that use every term of its split.

The router keeps fp32 semantics ("Mixture of Experts Explained", section "Switch
Transformer": the router stays in full precision; handbook news post, "真正难在三个环节"
item 1: FP32 routing) by splitting W_g exactly into three bf16 terms hi + mid + lo.  The
workload generator's W_g fits in one bf16, so there mid and lo are zero; these tests feed
weights whose mid and lo terms are not:

  * the prepared weight (moe_prepare_router_weight) is compared bit for bit with the split
    written out here from its definition, in the layout include/moe.h documents;
  * a construction whose every fp32 partial sum is exact (x in {-1, 0, 1} with at most 8
    non-zeros per token, W_g = m * 2^-22 with 20-bit integers m): the logits must equal
    the exact float64 logits bit for bit, and all routing must equal the oracle's;
  * general fp32 W_g ~ N(0, 0.02) with full 24-bit significands: the logits must lie
    within the rigorous bound of an fp32 sum of 3d exact products (in any order, rounded
    to nearest or toward zero), far inside the error of the bf16 weight alone, and the
    fused selection must be the exact top-k of the GPU's own logits; against the oracle's
    float64 choice the selection must agree wherever the decision margin exceeds twice
    the bound.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_moe_b200 import inputs as I
from tests import gpu_util as U

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


def _M():
    from routing_dispatch_expert_moe_b200 import moe as M
    return M


def _no_device_error():
    torch.cuda.synchronize()
    code = _M().moe_get_device_error()
    assert code == 0, f"device error {code}"


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def host_split(W):
    """hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid), from the definition (torch's
    round-to-nearest-even cast; the subtractions are exact in fp32)."""
    W = np.ascontiguousarray(W, np.float32)
    hi = _bf16(W)
    r1 = W - hi.float().numpy()
    mid = _bf16(r1)
    lo = _bf16(r1 - mid.float().numpy())
    return hi, mid, lo


def geometry(E):
    tiles = -(-E // 256)
    per = -(-E // tiles)
    return tiles, 32 * -(-per // 32)


def expected_layout(W):
    """The prepared weight as documented: tile j = experts j*NE .. j*NE+NE-1, rows hi, mid, lo
    of a K-major bf16 matrix [3 tiles NE, d], zero past E."""
    d, E = W.shape
    tiles, NE = geometry(E)
    hi, mid, lo = host_split(W)
    out = torch.zeros((tiles * 3 * NE, d), dtype=torch.bfloat16)
    for j in range(tiles):
        e0, e1 = j * NE, min(E, (j + 1) * NE)
        for t, term in enumerate((hi, mid, lo)):
            r0 = (3 * j + t) * NE
            out[r0:r0 + e1 - e0] = term[:, e0:e1].T
    return out


def general_weights(d, E, seed):
    """fp32 N(0, 0.02) with full 24-bit significands (not on any coarse grid)."""
    rng = np.random.default_rng([seed, 91])
    return (rng.standard_normal((d, E)) * 0.02).astype(np.float32)


def exact_construction(T, d, E, seed, with_offset):
    """x in {-1, 0, 1} with at most 8 non-zeros per token; W_g = m * 2^-22 with |m| in
    [2^19, 2^20) (20 significant bits: hi 8, mid 8, lo the rest); offsets on the 2^-22
    grid below 1.  Every partial sum of any order is a multiple of 2^-22 below
    8 * 2^20 * 2^-22 + 1 = 3 < 4 = 2^24 * 2^-22, hence exact in fp32."""
    rng = np.random.default_rng([seed, 92])
    x = np.zeros((T, d), np.float32)
    for t in range(T):
        nz = rng.choice(d, size=int(rng.integers(0, 9)), replace=False)
        x[t, nz] = rng.choice([-1.0, 1.0], size=len(nz))
    m = rng.integers(2 ** 19, 2 ** 20, size=(d, E)) * rng.choice([-1, 1], size=(d, E))
    W = (m.astype(np.float64) * 2.0 ** -22).astype(np.float32)
    off = None
    if with_offset:
        off = (rng.integers(-(2 ** 21), 2 ** 21, size=E).astype(np.float64) * 2.0 ** -22).astype(np.float32)
    return x, W, off


# ------------------------------------------------------------------ the prepared weight
@pytest.mark.parametrize("d,E", [(64, 8), (2048, 64), (1024, 256), (7168, 896), (512, 1024), (128, 260),
                                 (4096, 36)])
def test_prepared_weight_is_the_exact_three_term_split(d, E):
    M = _M()
    W = general_weights(d, E, seed=d + E)
    W[0, :4] = [0.0, -0.0, 2.0 ** -10, -3.0]              # exact bf16 values: mid = lo = 0
    W3 = M.moe_prepare_router_weight(torch.from_numpy(W).cuda())
    _no_device_error()
    got = W3.cpu().view(torch.bfloat16).reshape(-1, d)
    want = expected_layout(W)
    assert got.shape == want.shape
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), "split weight differs from its definition"
    hi, mid, lo = (t.double().numpy() for t in host_split(W))
    assert np.array_equal(hi + mid + lo, W.astype(np.float64)), "the three terms must carry w exactly"
    assert (mid != 0).mean() > 0.9 and (lo != 0).mean() > 0.5, "general weights must use mid and lo"


# ------------------------------------------------------------------ bit-exact, all terms used
EXACT = [  # T, d, E, k, score, renorm, scale, offset, bias
    (512, 256, 64, 8, "softmax", True, 1.0, False, False),
    (777, 1024, 256, 8, "sigmoid", True, 2.5, True, True),
    (1024, 7168, 896, 16, "sqrt_softplus", True, 1.0, True, False),
    (256, 64, 1024, 32, "softmax", False, 1.0, False, False),
    (600, 128, 36, 4, "sqrt_softplus", False, 3.0, True, True),
    (513, 512, 520, 6, "softmax", True, 1.0, True, True),      # softmax + bias: the separate top-k pass
]


@pytest.mark.parametrize("T,d,E,k,score,renorm,scale,with_off,with_bias", EXACT)
def test_router_bit_exact_when_every_split_term_is_used(T, d, E, k, score, renorm, scale, with_off, with_bias):
    M = _M()
    x, W, off = exact_construction(T, d, E, seed=T + E, with_offset=with_off)
    bias = None
    if with_bias:
        bias = np.random.default_rng([E, 93]).uniform(-0.1, 0.1, E).astype(np.float32)
    hi, mid, lo = (t.double().numpy() for t in host_split(W))
    assert (mid != 0).any() and (lo != 0).any(), "the construction must use every split term"
    xd, Wd = _bf16(x).cuda(), torch.from_numpy(W).cuda()
    offd = None if off is None else torch.from_numpy(off).cuda()
    biasd = None if bias is None else torch.from_numpy(bias).cuda()
    W3 = M.moe_prepare_router_weight(Wd)
    l, idx, gate = M.moe_route(xd, Wd, k, score, renorm, scale, offd, biasd, Wg_split=W3)
    _no_device_error()
    o = O.route(x, W, k, score, renorm, scale, off, bias)
    assert np.array_equal(l.cpu().numpy().astype(np.float64), o["logits"]), "logits not bit-exact"
    gi = idx.cpu().numpy()
    if bias is None:
        assert np.array_equal(gi, o["topk_idx"])
        err = np.abs(gate.cpu().numpy().astype(np.float64) - o["topk_gate"])
        assert (err <= U.GATE_RTOL * np.abs(o["topk_gate"]) + 1e-30).all()
    else:
        # fp64 keys score(l) + bias: equal wherever the decision is not within rounding
        sure = O.decision_margin(o["keys"], k) > 1e-9
        assert sure.mean() > 0.99
        assert np.array_equal(gi[sure], o["topk_idx"][sure])
    # the same call splitting W_g itself (no prepared weight) gives the same bits
    l2, idx2, gate2 = M.moe_route(xd, Wd, k, score, renorm, scale, offd, biasd)
    torch.cuda.synchronize()
    assert torch.equal(l, l2) and torch.equal(idx, idx2) and torch.equal(gate, gate2)
    # and the router alone gives the same logits
    l3 = M.moe_router_logits(xd, Wd, offd, Wg_split=W3)
    torch.cuda.synchronize()
    assert torch.equal(l, l3)


# ------------------------------------------------------------------ general fp32 weights
GENERAL = [  # T, d, E, k, score, renorm, bias
    (512, 2048, 64, 8, "softmax", True, False),
    (1024, 7168, 896, 16, "sqrt_softplus", True, False),
    (256, 512, 1024, 32, "softmax", True, False),
    (700, 4096, 256, 8, "sigmoid", True, True),
]


@pytest.mark.parametrize("T,d,E,k,score,renorm,with_bias", GENERAL)
def test_router_general_fp32_weights(T, d, E, k, score, renorm, with_bias):
    M = _M()
    cfg = I.small_config("general", T=T, d=d, E=E, k=k, F=64)
    x = I.gen_x(cfg, seed=5)                                   # bf16 values
    W = general_weights(d, E, seed=7)
    bias = np.random.default_rng([E, 94]).uniform(-0.1, 0.1, E).astype(np.float32) if with_bias else None
    hi, mid, lo = (t.double().numpy() for t in host_split(W))
    assert (mid != 0).mean() > 0.9 and (lo != 0).mean() > 0.5
    xd, Wd = _bf16(x).cuda(), torch.from_numpy(W).cuda()
    biasd = None if bias is None else torch.from_numpy(bias).cuda()
    l, idx, gate = M.moe_route(xd, Wd, k, score, renorm, 1.0, None, biasd, Wg_split=M.moe_prepare_router_weight(Wd))
    _no_device_error()
    lg = l.cpu().numpy().astype(np.float64)
    exact = O.router_logits(x, W)                              # float64: every product exact, sum to 2^-53
    err = np.abs(lg - exact)
    # (i) rigorous: an fp32 sum of 3d exact products in any order, each addition rounded
    # (to nearest or toward zero), is off by at most 3d * 2^-23 * sum |products|
    mag = np.abs(x).astype(np.float64) @ (np.abs(hi) + np.abs(mid) + np.abs(lo))
    bound = 3 * d * 2.0 ** -23 * mag
    assert (err <= bound).all(), f"beyond the fp32 bound: worst ratio {float((err / bound).max()):.3g}"
    # (ii) far closer than the bf16 weight alone: dropping the mid and lo terms would be off
    # by about 2^-9 of each product (the lo term is checked exactly by the construction above)
    hi_only = float(np.abs(np.asarray(x, np.float64) @ hi - exact).max())
    assert float(err.max()) < 0.01 * hi_only, (float(err.max()), hi_only)
    print(f"\nrouter d={d} E={E}: max |err| {float(err.max()):.3g}, worst err / bound "
          f"{float((err / bound).max()):.3g}, hi-only max |err| {hi_only:.3g}")
    # (iii) the fused selection is exactly the top-k of the GPU's own logits
    keys_own = O.selection_keys(lg, score, bias)
    idx_own = O.top_k(keys_own, k)
    gi = idx.cpu().numpy()
    if bias is None:
        assert np.array_equal(gi, idx_own), "selection is not the top-k of the kernel's own logits"
    else:
        sure_own = O.decision_margin(keys_own, k) > 1e-12
        assert np.array_equal(gi[sure_own], idx_own[sure_own])
    g_own = O.gates(lg, gi, score, renorm, 1.0)
    assert (np.abs(gate.cpu().numpy() - g_own) <= U.GATE_RTOL * np.abs(g_own) + 1e-30).all()
    # (iv) against the oracle's float64 choice wherever the margin exceeds twice the bound
    o = O.route(x, W, k, score, renorm, 1.0, None, bias)
    tb = bound.max(axis=1)
    if bias is not None:
        tb = tb * 0.25 + 1e-12                                 # score slope <= 1/4 (sigmoid)
    sure = O.decision_margin(o["keys"], k) > 2 * tb
    assert np.array_equal(gi[sure], o["topk_idx"][sure])


@pytest.mark.parametrize("terms", ["side", "stacked"])
@pytest.mark.parametrize("T,d,E,k,score", [(512, 256, 64, 8, "softmax"), (300, 128, 8, 2, "sigmoid"),
                                          (700, 512, 36, 4, "sqrt_softplus")])
def test_router_both_term_layouts_bit_exact(T, d, E, k, score, terms, monkeypatch):
    """Up to 64 experts per tile the three split terms can sit side by side in one MMA;
    both layouts must give the exact logits and routing."""
    monkeypatch.setenv("MOE_B200_ROUTER_TERMS", terms)
    M = _M()
    x, W, off = exact_construction(T, d, E, seed=T + d, with_offset=True)
    xd, Wd, offd = _bf16(x).cuda(), torch.from_numpy(W).cuda(), torch.from_numpy(off).cuda()
    l, idx, gate = M.moe_route(xd, Wd, k, score, True, 1.0, offd, Wg_split=M.moe_prepare_router_weight(Wd))
    _no_device_error()
    o = O.route(x, W, k, score, True, 1.0, off, None)
    assert np.array_equal(l.cpu().numpy().astype(np.float64), o["logits"])
    assert np.array_equal(idx.cpu().numpy(), o["topk_idx"])

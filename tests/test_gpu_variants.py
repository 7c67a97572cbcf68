"""GPU parity of the routing variants through the C ABI: the router alone, forced-uniform
and hash selection, noisy top-k, and the whole layer driven by each rule.

Bars: logits, indices, counts, offsets and row maps bit-exact; gates |err| <= 1e-6 |g|;
noisy H within the fp32 evaluation bound of its formula, with the selection compared
where it is unique (the top-k of the GPU's own H must match bit for bit, and the
oracle's float64 choice wherever its decision margin exceeds twice that bound).
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


def _gates_close(g, o):
    g = np.asarray(g, np.float64)
    err = np.abs(g - o)
    assert (err <= U.GATE_RTOL * np.abs(o) + 1e-30).all(), f"gate rel err {float((err / np.abs(o)).max()):.3g}"


def _random_logits(T, E, seed, spread=2.0):
    rng = np.random.default_rng([seed, 77])
    return (rng.standard_normal((T, E)) * spread).astype(np.float32)


# ---------------------------------------------------------------- the router alone
ROUTER = [
    I.small_config("tc_bf16", T=300, d=256, E=64, k=8, F=64),
    I.small_config("tc_ragged_offset", T=1000, d=128, E=36, k=4, F=64, logit_offset="zipf1.2"),
    I.small_config("simt_E_odd", T=333, d=128, E=37, k=3, F=64),
    I.small_config("simt_fp32", T=256, d=64, E=8, k=2, F=64, act="f32"),
    I.small_config("simt_small_batch_E1024", T=130, d=64, E=1024, k=32, F=64, logit_offset="normal0.5"),
    I.small_config("tc_E1024", T=300, d=64, E=1024, k=32, F=64, logit_offset="normal0.5"),
    # few row tiles: most CTA pairs idle; a ragged last tile of 700 - 512 tokens
    I.small_config("tc_long_d", T=512, d=2048, E=64, k=8, F=64),
    I.small_config("tc_ragged_tiles_offset", T=700, d=1024, E=36, k=4, F=64, logit_offset="zipf1.2"),
    I.small_config("tc_three_expert_tiles", T=520, d=256, E=520, k=6, F=64, score="sigmoid"),
]


@pytest.mark.parametrize("cfg", ROUTER, ids=lambda c: c.name)
def test_router_logits_bit_exact_and_equal_to_the_routed_logits(cfg):
    host, dev = U.make_inputs(cfg)
    M = _M()
    l = M.moe_router_logits(dev["x"], dev["Wg"], dev["off"])
    _no_device_error()
    o = O.router_logits(host["x"], host["Wg"], host["off"])
    assert np.array_equal(l.cpu().numpy().astype(np.float64), o)
    l2, _, _ = M.moe_route(dev["x"], dev["Wg"], cfg.k, cfg.score, cfg.renormalize, cfg.scale, dev["off"])
    torch.cuda.synchronize()
    assert torch.equal(l, l2)


# ---------------------------------------------------------------- fixed selection rules
FIXED = [  # (T, E, k, score, renormalize, scale)
    (1000, 64, 8, "softmax", True, 1.0),
    (777, 37, 3, "softmax", False, 1.0),
    (513, 256, 8, "sigmoid", True, 2.5),
    (300, 896, 16, "sqrt_softplus", True, 1.0),
    (129, 1024, 32, "sigmoid", False, 1.0),
    (200, 8, 8, "softmax", True, 1.0),         # k = E
    (1, 5, 1, "sqrt_softplus", False, 3.0),    # one token, top-1
]


@pytest.mark.parametrize("T,E,k,score,renorm,scale", FIXED)
@pytest.mark.parametrize("rule", ["uniform", "hash"])
def test_fixed_selection_parity(rule, T, E, k, score, renorm, scale):
    M = _M()
    l = _random_logits(T, E, seed=T + E)
    cfg = I.small_config("ids", T=T, d=64, E=E, k=k, F=64)
    tid = I.gen_token_ids(cfg, seed=3)
    tid[: min(T, 4)] = [0, -1, 2**31 - 1, -(2**31)][: min(T, 4)]         # extreme ids
    seed = 0x9E3779B9
    idx, gate = M.moe_route_fixed(torch.from_numpy(l).cuda(), k, rule, score, renorm, scale,
                                  torch.from_numpy(tid).cuda() if rule == "hash" else None, seed)
    _no_device_error()
    o = O.route_fixed(l, k, score, renorm, scale, rule, tid, seed)
    assert np.array_equal(idx.cpu().numpy(), o["topk_idx"])
    _gates_close(gate.cpu().numpy(), o["topk_gate"])
    if rule == "uniform":
        c = np.bincount(idx.cpu().numpy().ravel(), minlength=E)
        assert set(np.unique(c)) <= {T * k // E, -(-T * k // E)}


def test_hash_selection_follows_the_token_id_not_the_position():
    M = _M()
    T, E, k = 600, 64, 8
    tid = np.repeat(np.array([5, 17, 5, 99], np.int32), T // 4)
    l = _random_logits(T, E, seed=1)
    idx, _ = M.moe_route_fixed(torch.from_numpy(l).cuda(), k, "hash", token_id=torch.from_numpy(tid).cuda(), seed=7)
    idx = idx.cpu().numpy()
    for v in np.unique(tid):
        rows = idx[tid == v]
        assert (rows == rows[0]).all()
        assert sorted(rows[0].tolist()) == sorted(O.hash_experts(int(v), 7, E, k))


# ---------------------------------------------------------------- noisy top-k
def _h_bound(l, ln, n):
    """fp32 evaluation of l + n * softplus(ln): softplus from expf and log1pf (a few ulp),
    then one rounding of the fused multiply-add."""
    sp = O.softplus(ln)
    return 2.0 ** -20 * (np.abs(l) + np.abs(n) * sp) + 1e-37


NOISY = [(777, 16, 2, 1.0), (1024, 64, 8, 1.0), (300, 256, 8, 2.5), (129, 1000, 32, 1.0)]


@pytest.mark.parametrize("T,E,k,scale", NOISY)
def test_noisy_top_k_parity(T, E, k, scale):
    M = _M()
    cfg = I.small_config("noisy", T=T, d=64, E=E, k=k, F=64)
    l = _random_logits(T, E, seed=5)
    ln = _random_logits(T, E, seed=6, spread=3.0)
    n = I.gen_noise(cfg, seed=2)
    H, idx, gate = M.moe_route_noisy(torch.from_numpy(l).cuda(), torch.from_numpy(ln).cuda(),
                                     torch.from_numpy(n).cuda(), k, scale)
    _no_device_error()
    Hg = H.cpu().numpy().astype(np.float64)
    Ho = O.noisy_logits(l, ln, n)
    bound = _h_bound(l, ln, n)
    assert (np.abs(Hg - Ho) <= bound).all(), float((np.abs(Hg - Ho) / bound).max())
    # the decision on the GPU's own H: bit-exact
    idx_g = idx.cpu().numpy()
    assert np.array_equal(idx_g, O.top_k(Hg, k))
    _gates_close(gate.cpu().numpy(), O.gates(Hg, idx_g, "softmax", True, scale))
    # the oracle's float64 decision wherever it is unique at this precision
    o = O.route_noisy(l, ln, n, k, scale)
    sure = O.decision_margin(Ho, k) > 2 * bound.max(axis=1)
    assert sure.mean() > 0.95
    assert np.array_equal(np.sort(idx_g[sure], axis=1), np.sort(o["topk_idx"][sure], axis=1))


def test_noisy_top_k_without_noise_equals_the_learned_softmax_router():
    M = _M()
    T, E, k = 500, 64, 8
    l = _random_logits(T, E, seed=8)
    zeros = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    lt = torch.from_numpy(l).cuda()
    H, idx, gate = M.moe_route_noisy(lt, torch.from_numpy(_random_logits(T, E, seed=9)).cuda(), zeros, k, 1.5)
    torch.cuda.synchronize()
    assert torch.equal(H, lt)
    o = O.route_noisy(l, np.zeros((T, E)), np.zeros((T, E)), k, 1.5)
    assert np.array_equal(idx.cpu().numpy(), o["topk_idx"])
    _gates_close(gate.cpu().numpy(), o["topk_gate"])


# ---------------------------------------------------------------- the layer under each rule
VARIANT_LAYERS = [
    ("uniform", I.small_config("uniform_layer", T=700, d=256, E=32, k=4, F=128, capacity_factor=1.0,
                               logit_offset="zipf1.2")),
    ("hash", I.small_config("hash_layer", T=900, d=128, E=16, k=2, F=64, score="sigmoid", scale=2.0,
                            capacity_factor=1.25)),
    ("noisy", I.small_config("noisy_layer", T=640, d=128, E=24, k=3, F=128)),
]


@pytest.mark.parametrize("routing,cfg", VARIANT_LAYERS, ids=[v[0] for v in VARIANT_LAYERS])
def test_layer_under_each_routing_rule(routing, cfg):
    from routing_dispatch_expert_moe_b200.layer import MoELayer, MoEWeights
    M = _M()
    host, dev = U.make_inputs(cfg)
    cap = O.capacity(cfg.T, cfg.E, cfg.k, cfg.capacity_factor)
    Wn = I.gen_noise_router(cfg) if routing == "noisy" else None
    w = MoEWeights(Wg=dev["Wg"], W_gu=dev["W_gu"], W_dn=dev["W_dn"], logit_offset=dev["off"],
                   W_noise=None if Wn is None else torch.from_numpy(Wn).cuda())
    lay = MoELayer(w, cfg.k, cfg.T, cfg.score, cfg.renormalize, cfg.scale, cap, routing=routing, hash_seed=11)
    tid = I.gen_token_ids(cfg, seed=1)
    noise = I.gen_noise(cfg, seed=1)
    y = lay.forward(dev["x"], token_id=torch.from_numpy(tid).cuda(), noise=torch.from_numpy(noise).cuda())
    _no_device_error()
    logits = O.router_logits(host["x"], host["Wg"], host["off"])
    if routing == "noisy":
        Hg = lay.H.cpu().numpy().astype(np.float64)
        ln = O.router_logits(host["x"], Wn)
        assert np.array_equal(lay.logits_noise.cpu().numpy().astype(np.float64), ln)
        assert (np.abs(Hg - O.noisy_logits(logits, ln, noise)) <= _h_bound(logits, ln, noise)).all()
        idx = O.top_k(Hg, cfg.k)
        r = {"topk_idx": idx, "topk_gate": O.gates(Hg, idx, "softmax", True, cfg.scale)}
    else:
        r = O.route_fixed(logits, cfg.k, cfg.score, cfg.renormalize, cfg.scale, routing, tid, 11)
    o = dict(r, logits=logits)
    o.update(O.dispatch_plan(r["topk_idx"], r["topk_gate"], cfg.E, cap))
    g = {"logits": lay.logits.cpu().numpy(), "topk_idx": lay.topk_idx.cpu().numpy(),
         "topk_gate": lay.topk_gate.cpu().numpy(), "counts": lay.counts.cpu().numpy(),
         "kept": lay.kept.cpu().numpy(), "offsets": lay.offsets.cpu().numpy(), "row_of": lay.row_of.cpu().numpy()}
    n = int(g["offsets"][-1])
    g.update(n_rows=n, token_of_row=lay.token_of_row[:n].cpu().numpy(), gate_of_row=lay.gate_of_row[:n].cpu().numpy())
    U.assert_routing_equal(g, o)
    gu, dn = U.expert_getters(host)
    xperm = O.permute(host["x"], o["row_of"], n)
    yp = O.grouped_ffn(xperm, o["offsets"], gu, dn, o["gate_of_row"], True)
    U.assert_y_close(y.float().cpu().numpy().astype(np.float64), O.combine(yp, o["row_of"]), "y")
    st = O.router_stats(logits, o["counts"], o["kept"], cfg.k, cfg.score)
    U.assert_stats_close({"load": lay.load.cpu().numpy(), "stats5": lay.stats5.cpu().numpy()}, st)
    if routing == "uniform":
        assert set(np.unique(o["counts"])) <= {cfg.T * cfg.k // cfg.E, -(-cfg.T * cfg.k // cfg.E)}
    assert lay.launches_per_forward() >= 9

"""Pins for the CPU oracle: closed forms, hand-derived fixtures, brute force, invariants.

Each test checks the oracle against something other than itself, chosen so that
a plausible slip (a dropped term, a wrong sign or index, a transposed operand,
a swapped role) fails at least one of them.  CPU only.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import moe_oracle as O
from routing_dispatch_expert_moe_b200 import inputs as I
from tests._closed_form import ev, evf, load


# ---------------------------------------------------------------- capacity
def test_capacity_closed_forms(golden_dir):
    g = load(golden_dir, "capacity.json")
    for c in g["cases"]:
        assert O.capacity(c["T"], c["E"], c["k"], c["cf"], True) == c["per_assignment"], c
        assert O.capacity(c["T"], c["E"], c["k"], c["cf"], False) == c["literal"], c
    assert O.capacity(100, 4, 2, None) == -1
    assert O.capacity(100, 4, 2, 0.0) == -1


def test_capacity_workloads():
    c1, c5 = I.CONFIGS["c1_tiny"], I.CONFIGS["c5_stress"]
    assert O.capacity(c1.T, c1.E, c1.k, c1.capacity_factor) == 80
    assert O.capacity(c5.T, c5.E, c5.k, c5.capacity_factor) == 586
    assert O.capacity(c5.T, c5.E, c5.k, c5.capacity_factor, per_assignment=False) == 37


# ---------------------------------------------------------------- shapes
def test_param_accounting_handbook_shape(golden_dir):
    g = load(golden_dir, "param_accounting.json")
    c = I.CONFIGS["c2_handbook"]
    assert (c.E, c.k, c.F) == (g["experts"], g["top_k"], g["expert_width"])
    stored = c.E * 3 * c.d * c.F
    dense = 3 * c.d * g["dense_width"]
    assert stored == g["stored_ratio"] * dense
    assert (c.k * c.F == g["dense_width"]) == g["active_width_equals_dense"]


# ---------------------------------------------------------------- logits
def _int_grid(cfg):
    return (256, 256) if cfg.act == "f32" else (8, 1024)


@pytest.mark.parametrize("name,T", [("c1_tiny", 256), ("c2_handbook", 64), ("c3_fine_grained", 16),
                                    ("c5_stress", 8)])
def test_logits_exact_against_int64_bruteforce(name, T):
    cfg = I.CONFIGS[name]
    x = I.gen_x(cfg, 0, T=T)
    Wg, off, _ = I.gen_router(cfg, 0)
    sx, sw = _int_grid(cfg)
    xi = np.rint(x.astype(np.float64) * sx).astype(np.int64)
    wi = np.rint(Wg.astype(np.float64) * sw).astype(np.int64)
    assert np.array_equal(xi / sx, x) and np.array_equal(wi / sw, Wg)   # on the grid
    unit = sx * sw
    acc = np.zeros((T, cfg.E), np.int64)
    for c in range(cfg.d):                                              # plain integer dot product
        acc += xi[:, c:c + 1] * wi[c:c + 1, :]
    if off is not None:
        oi = np.rint(off.astype(np.float64) * unit).astype(np.int64)
        assert np.array_equal(oi / unit, off.astype(np.float64))
        acc += oi[None, :]
    assert np.abs(acc).max() < 2 ** 24                                  # exact in fp32
    l = O.router_logits(x, Wg, off)
    assert np.array_equal(l * unit, acc.astype(np.float64))
    assert np.array_equal(l.astype(np.float32).astype(np.float64), l)


def test_logit_offset_enters():
    cfg = I.CONFIGS["c3_fine_grained"]
    x = I.gen_x(cfg, 0, T=4)
    Wg, off, _ = I.gen_router(cfg, 0)
    assert not np.array_equal(O.router_logits(x, Wg, off), O.router_logits(x, Wg, None))
    np.testing.assert_array_equal(O.router_logits(x, Wg, off) - O.router_logits(x, Wg, None),
                                  np.broadcast_to(off.astype(np.float64), (4, cfg.E)))


# ---------------------------------------------------------------- top-k
def _brute_topk_set(keys_row, k):
    """The unique k-subset whose every member beats every non-member in (key desc, index asc)."""
    E = len(keys_row)
    beats = lambda a, b: (keys_row[a] > keys_row[b]) or (keys_row[a] == keys_row[b] and a < b)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if all(beats(a, b) for a in S for b in rest):
            found.append(set(S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("E", [2, 3, 5, 8, 10])
def test_topk_bruteforce_enumeration(E):
    rng = np.random.default_rng(E)
    for trial in range(40):
        keys = rng.integers(-3, 4, size=(1, E)).astype(np.float64)   # many ties
        if trial % 3 == 0:
            keys = rng.standard_normal((1, E))
        for k in range(1, E + 1):
            idx = O.top_k(keys, k)[0]
            assert set(idx.tolist()) == _brute_topk_set(keys[0], k)
            order = sorted(idx.tolist(), key=lambda e: (-keys[0, e], e))
            assert idx.tolist() == order


def test_topk_all_equal_goes_to_lower_index():
    keys = np.zeros((3, 16))
    assert O.top_k(keys, 5).tolist() == [[0, 1, 2, 3, 4]] * 3


def test_routing_hand_cases(golden_dir):
    g = load(golden_dir, "routing_hand.json")
    for c in g["topk_cases"]:
        l = np.array([[evf(v) for v in c["logits"]]])
        bias = None if c["bias"] is None else np.array([evf(v) for v in c["bias"]])
        keys = O.selection_keys(l, c["score"], bias)
        idx = O.top_k(keys, c["k"])
        assert idx[0].tolist() == c["idx"], c["name"]
        gt = O.gates(l, idx, c["score"], c["renormalize"], evf(c["scale"]))
        want = np.array([evf(v) for v in c["gates"]])
        np.testing.assert_allclose(gt[0], want, rtol=1e-13, atol=0, err_msg=c["name"])


def test_sqrt_softplus_closed_forms(golden_dir):
    g = load(golden_dir, "routing_hand.json")
    for c in g["sqrt_softplus_values"]:
        s = O.router_scores(np.array([[evf(c["logit"])]]), "sqrt_softplus")[0, 0]
        assert math.isclose(s, evf(c["value"]), rel_tol=1e-13), c


def test_sigmoid_and_softmax_closed_forms():
    l = np.array([[0.0, math.log(3.0), -math.log(3.0)]])
    np.testing.assert_allclose(O.router_scores(l, "sigmoid")[0], [0.5, 0.75, 0.25], rtol=1e-15)
    p = O.router_scores(np.array([[0.0, math.log(2), math.log(5)]]), "softmax")[0]
    np.testing.assert_allclose(p, [1 / 8, 2 / 8, 5 / 8], rtol=1e-15)


@pytest.mark.parametrize("score", ["softmax", "sigmoid", "sqrt_softplus"])
def test_renormalised_gates_sum_to_scale(score):
    rng = np.random.default_rng(1)
    l = rng.standard_normal((200, 32)) * 2
    for k, scale in [(1, 1.0), (4, 2.5), (8, 1.0), (32, 1.0)]:
        idx = O.top_k(O.selection_keys(l, score), k)
        g = O.gates(l, idx, score, True, scale)
        np.testing.assert_allclose(g.sum(axis=1), scale, rtol=1e-13)
        assert (g > 0).all()


def test_softmax_over_kept_equals_renormalised_full_softmax():
    rng = np.random.default_rng(2)
    l = rng.standard_normal((100, 24)) * 3
    idx = O.top_k(l, 6)
    p = O.softmax(l)
    pk = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(O.gates(l, idx, "softmax", True, 1.0), pk / pk.sum(1, keepdims=True),
                               rtol=1e-13)


def test_switch_top1_is_argmax_with_full_probability():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((100, 12))
    idx = O.top_k(l, 1)
    assert np.array_equal(idx[:, 0], np.argmax(l, axis=1))
    g = O.gates(l, idx, "softmax", False, 1.0)
    np.testing.assert_allclose(g[:, 0], O.softmax(l).max(axis=1), rtol=1e-14)


def test_selection_bias_changes_selection_not_gate_formula():
    l = np.array([[2.0, 1.0, 0.0, -1.0]])
    no_bias = O.top_k(O.selection_keys(l, "sigmoid"), 2)
    with_bias = O.top_k(O.selection_keys(l, "sigmoid", np.array([0.0, 0.0, 0.0, 0.9])), 2)
    assert no_bias.tolist() == [[0, 1]] and with_bias.tolist() == [[3, 0]]
    g = O.gates(l, with_bias, "sigmoid", True, 1.0)[0]
    s = 1 / (1 + np.exp(-np.array([-1.0, 2.0])))
    np.testing.assert_allclose(g, s / s.sum(), rtol=1e-14)


def test_decision_margin():
    keys = np.array([[3.0, 1.0, 2.0, 2.0], [5.0, 4.0, 0.0, 1.0]])
    np.testing.assert_array_equal(O.decision_margin(keys, 2), [0.0, 3.0])
    assert np.isinf(O.decision_margin(keys, 4)).all()


# ---------------------------------------------------------------- dispatch plan
def _brute_plan(idx, E, cap):
    T, k = idx.shape
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[idx[t, j]] += 1
    kept = [c if cap < 0 else min(c, cap) for c in counts]
    offs = [0]
    for e in range(E):
        offs.append(offs[-1] + kept[e])
    row_of = -np.ones((T, k), np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            r = sum(1 for t2 in range(t) for j2 in range(k) if idx[t2, j2] == e)
            if cap < 0 or r < cap:
                row_of[t, j] = offs[e] + r
    return np.array(counts), np.array(kept), np.array(offs), row_of


def _random_topk(rng, T, E, k, skew=False):
    p = None
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.5
        p = p / p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k,cap,skew", [(40, 6, 2, -1, False), (40, 6, 2, 5, True), (33, 8, 3, 7, True),
                                            (17, 4, 4, 3, False), (25, 5, 1, 4, True), (30, 9, 3, 0, False)])
def test_dispatch_plan_bruteforce(T, E, k, cap, skew):
    rng = np.random.default_rng(T * 100 + E)
    idx = _random_topk(rng, T, E, k, skew)
    gate = rng.random((T, k))
    p = O.dispatch_plan(idx, gate, E, cap)
    counts, kept, offs, row_of = _brute_plan(idx, E, cap)
    assert np.array_equal(p["counts"], counts)
    assert np.array_equal(p["kept"], kept)
    assert np.array_equal(p["offsets"], offs)
    assert np.array_equal(p["row_of"], row_of)
    # invariants
    assert p["counts"].sum() == T * k
    assert p["kept"].sum() + int((p["row_of"] < 0).sum()) == T * k
    assert (np.diff(p["offsets"]) >= 0).all()
    rows = p["row_of"][p["row_of"] >= 0]
    assert sorted(rows.tolist()) == list(range(int(p["offsets"][-1])))      # bijection
    for e in range(E):
        toks = p["token_of_row"][p["offsets"][e]:p["offsets"][e + 1]]
        assert (np.diff(toks) > 0).all()                                    # token order inside
        for r in range(p["offsets"][e], p["offsets"][e + 1]):
            t = p["token_of_row"][r]
            j = int(np.nonzero(idx[t] == e)[0][0])
            assert p["row_of"][t, j] == r and p["gate_of_row"][r] == gate[t, j]


def test_drop_hand_cases(golden_dir):
    g = load(golden_dir, "routing_hand.json")
    for c in g["drop_cases"]:
        idx = np.array(c["topk_idx"], np.int32)
        p = O.dispatch_plan(idx, np.ones(idx.shape), c["E"], c["cap"])
        for key in ("counts", "kept", "offsets", "row_of", "token_of_row"):
            assert np.array_equal(p[key], np.array(c[key])), (c["name"], key)


# ---------------------------------------------------------------- permute / combine
def test_bf16_round_against_library_cast():
    import torch
    rng = np.random.default_rng(4)
    v = (rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000)).astype(np.float32)
    # halfway cases between neighbouring bf16 values
    v = np.concatenate([v, np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0])])
    want = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = O.bf16_round(v.astype(np.float64))
    assert np.array_equal(got, want)
    assert O.bf16_round(np.array([1 + 2 ** -8]))[0] == 1.0
    assert O.bf16_round(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


@pytest.mark.parametrize("k", [1, 2, 4, 8])
def test_permute_then_combine_is_identity(k):
    cfg = I.small_config(T=77, d=32, E=16, k=k)
    x = I.gen_x(cfg)
    Wg, _, _ = I.gen_router(cfg)
    r = O.layer_routing(cfg.__dict__, x, Wg)
    n = int(r["offsets"][-1])
    xp = O.permute(x, r["row_of"], n)
    # identity expert, gate 1/k on every row (k a power of two: exact)
    yp = xp * (1.0 / k)
    y = O.combine(yp, r["row_of"], None, round_out=True)
    assert np.array_equal(y, x.astype(np.float64))
    # and the permuted rows really are the tokens
    assert np.array_equal(xp, x.astype(np.float64)[r["token_of_row"]])


def test_combine_applies_topk_gate_when_not_fused():
    rng = np.random.default_rng(5)
    yp = rng.standard_normal((6, 3))
    row_of = np.array([[0, 3], [1, -1], [5, 2]])
    g = rng.random((3, 2))
    y = O.combine(yp, row_of, None, round_out=False, topk_gate=g)
    np.testing.assert_allclose(y[1], yp[1] * g[1, 0])
    np.testing.assert_allclose(y[2], yp[5] * g[2, 0] + yp[2] * g[2, 1])


# ---------------------------------------------------------------- expert FFN
def test_swiglu_hand(golden_dir):
    g = load(golden_dir, "swiglu_hand.json")
    x = np.array([[evf(v) for v in g["x"]]])
    W_gu = np.array([[evf(v) for v in r] for r in g["W_gate"] + g["W_up"]])
    W_dn = np.array([[evf(v) for v in r] for r in g["W_down"]])
    y = O.swiglu_expert(x, W_gu, W_dn, bf16=False)[0]
    np.testing.assert_allclose(y, [evf(v) for v in g["y"]], rtol=1e-14)
    assert not np.allclose(y, [evf(v) for v in g["swapped_roles_would_give"]], rtol=1e-3)


def test_zero_up_projection_leaves_only_shared_expert():
    cfg = I.small_config(T=50, d=64, E=8, k=2, F=64, F_s=64)
    x = I.gen_x(cfg)
    Wg, _, _ = I.gen_router(cfg)
    W_gu, W_dn = I.gen_experts(cfg)
    W_gu[:, cfg.F:] = 0.0
    sh = I.gen_shared(cfg)
    r = O.layer_forward(cfg.__dict__, x, Wg, W_gu, W_dn, shared=sh, bf16=True)
    assert np.array_equal(r["y"], r["shared_y"])
    assert np.abs(r["shared_y"]).max() > 0


def test_k_equals_E_layer_is_dense_mixture():
    cfg = I.small_config(T=40, d=32, E=6, k=6, F=16, act="f32")
    x = I.gen_x(cfg)
    Wg, _, _ = I.gen_router(cfg)
    W_gu, W_dn = I.gen_experts(cfg)
    r = O.layer_forward(cfg.__dict__, x, Wg, W_gu, W_dn, bf16=False)
    dense = O.dense_mixture(x, Wg, W_gu, W_dn)
    np.testing.assert_allclose(r["y"], dense, rtol=1e-12, atol=1e-15)


def test_subset_evaluation_matches_full_layer():
    cfg = I.small_config(T=64, d=64, E=8, k=3, F=64, F_s=32, capacity_factor=1.0,
                         score="sigmoid", scale=2.5)
    x = I.gen_x(cfg)
    Wg, _, _ = I.gen_router(cfg)
    bias = np.linspace(-0.1, 0.1, cfg.E)
    W_gu, W_dn = I.gen_experts(cfg)
    sh = I.gen_shared(cfg)
    for rr, ro in ((False, False), (True, True), (True, False)):
        full = O.layer_forward(cfg.__dict__, x, Wg, W_gu, W_dn, select_bias=bias, shared=sh, bf16=True,
                               round_rows=rr, round_out=ro)
        assert (full["row_of"] < 0).any()              # some drops exercised
        toks = [0, 5, 17, 63]
        sub = O.layer_outputs_for_tokens(toks, x, full, W_gu, W_dn, True, shared=sh, round_rows=rr, round_out=ro)
        np.testing.assert_allclose(sub["y"], full["y"][toks], rtol=1e-14, atol=1e-16)
        if ro:
            assert np.array_equal(O.bf16_round(sub["y"]), sub["y"])


# ---------------------------------------------------------------- router stats
def test_stats_closed_forms(golden_dir):
    g = {c["name"]: c for c in load(golden_dir, "stats_hand.json")["cases"]}
    T, E, k = 64, 8, 2
    # balanced: each expert gets T*k/E assignments, uniform probabilities (zero logits)
    s = O.router_stats(np.zeros((T, E)), np.full(E, T * k // E), np.full(E, T * k // E), k, "softmax")
    assert math.isclose(s["aux"], evf(g["balanced counts, uniform probabilities"]["aux"]), rel_tol=1e-14)
    assert math.isclose(s["z"], evf(g["all-zero logits, E = 8"]["z"]), rel_tol=1e-14)
    assert s["dropped"] == 0 and s["max_over_mean"] == 1.0 and s["cv"] == 0.0
    # k = E with arbitrary logits
    rng = np.random.default_rng(6)
    l = rng.standard_normal((T, E))
    for score in ("softmax", "sigmoid", "sqrt_softplus"):
        s = O.router_stats(l, np.full(E, T), np.full(E, T), E, score)
        assert math.isclose(s["aux"], evf(g["k = E: every expert chosen by every token"]["aux"]),
                            rel_tol=1e-13)


def test_stats_drop_and_imbalance():
    T, E, k = 10, 4, 2
    counts = np.array([10, 6, 4, 0])
    kept = np.minimum(counts, 5)
    s = O.router_stats(np.zeros((T, E)), counts, kept, k, "softmax")
    assert s["dropped"] == 20 - 14
    assert math.isclose(s["max_over_mean"], 10 / 5)
    assert math.isclose(s["cv"], float(np.std([10, 6, 4, 0])) / 5)
    np.testing.assert_allclose(s["load"], counts / 20)

"""Pins for the oracle's routing variants: forced-uniform and hash selection, noisy top-k.

Each check rests on something other than the oracle's own formula: the inverse of the
hash, the hash's published verification values, an exhaustive count over every draw
sequence of Floyd's sampling, closed forms, and special cases that reduce to the learned
router.  CPU only.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import moe_oracle as O

M32 = 1 << 32


# ---------------------------------------------------------------- the hash
def _unxorshift(h, s):
    """Inverse of h ^= h >> s on 32-bit words (s >= 1): recover the bits top-down."""
    x = h
    for _ in range(32 // s + 1):
        x = h ^ (x >> s)
    return x & (M32 - 1)


def _fmix32_inverse(h):
    h = _unxorshift(h, 16)
    h = (h * pow(0xC2B2AE35, -1, M32)) % M32
    h = _unxorshift(h, 13)
    h = (h * pow(0x85EBCA6B, -1, M32)) % M32
    return _unxorshift(h, 16)


def test_fmix32_is_inverted_by_its_inverse():
    rng = np.random.default_rng(5)
    xs = [0, 1, 2, 0x7FFFFFFF, 0x80000000, M32 - 1] + [int(v) for v in rng.integers(0, M32, 2000)]
    for x in xs:
        h = O.fmix32(x)
        assert 0 <= h < M32
        assert _fmix32_inverse(h) == x, hex(x)


def test_fmix32_matches_murmur3_empty_message_values():
    # MurmurHash3_x86_32 of an empty message with seed s is the finalizer of s (no blocks,
    # no tail, length 0); its published verification values for seeds 0, 1 and 2^32 - 1:
    assert O.fmix32(0) == 0
    assert O.fmix32(1) == 0x514E28B7
    assert O.fmix32(0xFFFFFFFF) == 0x81F16F39


# ---------------------------------------------------------------- Floyd's sampling
@pytest.mark.parametrize("E,k", [(5, 3), (6, 2), (4, 4), (7, 1), (6, 5)])
def test_floyd_sampling_is_exactly_uniform_over_all_draw_sequences(E, k):
    """Every sequence r_j in [0, n_j] (n_j = E - k + j) once: each k-subset of range(E)
    must come out the same number of times, prod(n_j + 1) / C(E, k)."""
    ranges = [range(E - k + j + 1) for j in range(k)]
    seen = {}
    total = 0
    for rs in itertools.product(*ranges):
        pick = O.floyd_sample(list(rs), E, k)
        assert len(set(pick)) == k and all(0 <= p < E for p in pick)
        key = tuple(sorted(pick))
        seen[key] = seen.get(key, 0) + 1
        total += 1
    assert len(seen) == math.comb(E, k)
    assert set(seen.values()) == {total // math.comb(E, k)}


def test_floyd_sampling_takes_the_word_modulo_the_range():
    # words far above the range reduce modulo n + 1 (here n = 3, 4)
    assert O.floyd_sample([7, 9], 5, 2) == [7 % 4, 9 % 5]
    assert O.floyd_sample([2, 2], 5, 2) == [2, 4]          # repeated draw -> the new top n


def test_hash_experts_distinct_and_deterministic():
    for E, k in [(64, 8), (256, 8), (896, 16), (1024, 32), (8, 8), (3, 1)]:
        for tid in [0, 1, 17, 31999, 2**31 - 1]:
            a = O.hash_experts(tid, 11, E, k)
            assert a == O.hash_experts(tid, 11, E, k)
            assert len(set(a)) == k and all(0 <= e < E for e in a)
    # another seed or another id gives another draw (for these values)
    assert O.hash_experts(17, 11, 64, 8) != O.hash_experts(17, 12, 64, 8)
    assert O.hash_experts(17, 11, 64, 8) != O.hash_experts(18, 11, 64, 8)


def test_hash_experts_single_draw_is_the_hash_modulo_E():
    for tid in range(50):
        w = O.fmix32(O.fmix32(tid ^ 3))                       # draw 0: fmix32(base + 0)
        assert O.hash_experts(tid, 3, 37, 1) == [w % 37]


def test_hash_experts_are_balanced_over_many_token_ids():
    E, k, n = 5, 2, 20000
    counts = {}
    marg = np.zeros(E)
    for tid in range(n):
        s = tuple(sorted(O.hash_experts(tid, 0, E, k)))
        counts[s] = counts.get(s, 0) + 1
        marg[list(s)] += 1
    exp = n / math.comb(E, k)
    chi2 = sum((c - exp) ** 2 / exp for c in counts.values())
    assert len(counts) == math.comb(E, k)
    assert chi2 < 40.0                                        # 9 degrees of freedom
    assert np.abs(marg / (n * k / E) - 1).max() < 0.03


# ---------------------------------------------------------------- forced-uniform rule
def test_uniform_rule_hand_example():
    idx = O.fixed_selection(4, 5, 3, "uniform")
    assert idx.tolist() == [[0, 1, 2], [3, 4, 0], [1, 2, 3], [4, 0, 1]]


@pytest.mark.parametrize("T,E,k", [(100, 8, 2), (333, 64, 8), (17, 7, 7), (1000, 896, 16)])
def test_uniform_rule_balances_counts_exactly(T, E, k):
    idx = O.fixed_selection(T, E, k, "uniform")
    assert all(len(set(r)) == k for r in idx.tolist())
    c = np.bincount(idx.ravel(), minlength=E)
    assert c.sum() == T * k
    assert set(np.unique(c)) <= {T * k // E, -(-T * k // E)}


def test_fixed_rules_reject_k_above_E():
    with pytest.raises(ValueError):
        O.fixed_selection(4, 3, 4, "uniform")
    with pytest.raises(ValueError):
        O.hash_experts(1, 0, 3, 4)


def test_fixed_rule_gates_are_the_learned_gates_when_the_sets_agree():
    """Logits built so that the learned top-k of token t is exactly the uniform rule's
    set: the gates of both paths then agree expert by expert (the learned path's gate
    rule applied to the chosen experts)."""
    T, E, k = 12, 10, 3
    rng = np.random.default_rng(2)
    l = rng.normal(0, 1, (T, E)) - 5.0
    uni = O.fixed_selection(T, E, k, "uniform")
    for t in range(T):
        l[t, uni[t]] = rng.normal(3, 1, k)
    for score, renorm, scale in [("softmax", True, 1.0), ("softmax", False, 2.0), ("sigmoid", True, 2.5),
                                 ("sqrt_softplus", False, 1.0)]:
        learned_idx = O.top_k(l, k)
        learned_g = O.gates(l, learned_idx, score, renorm, scale)
        f = O.route_fixed(l, k, score, renorm, scale, "uniform")
        for t in range(T):
            assert set(learned_idx[t]) == set(f["topk_idx"][t])
            a = dict(zip(learned_idx[t].tolist(), learned_g[t]))
            for e, g in zip(f["topk_idx"][t].tolist(), f["topk_gate"][t]):
                assert g == pytest.approx(a[e], rel=1e-14)
        if renorm:
            np.testing.assert_allclose(f["topk_gate"].sum(axis=1), scale, rtol=1e-13)


# ---------------------------------------------------------------- noisy top-k
def test_softplus_closed_forms():
    z = np.array([-40.0, -3.0, -0.5, 0.0, 0.5, 3.0, 40.0])
    sp = O.softplus(z)
    assert sp[3] == pytest.approx(math.log(2.0), rel=1e-15)
    np.testing.assert_allclose(sp - O.softplus(-z), z, rtol=0, atol=1e-14)   # softplus(z) - softplus(-z) = z
    np.testing.assert_allclose(sp, [math.log1p(math.exp(v)) for v in z], rtol=1e-14)
    assert sp[0] == pytest.approx(math.exp(-40.0), rel=1e-12)
    assert (sp > 0).all()


def test_noisy_logits_special_cases():
    rng = np.random.default_rng(4)
    l = rng.normal(0, 2, (6, 9))
    ln = rng.normal(0, 2, (6, 9))
    n = rng.normal(0, 1, (6, 9))
    np.testing.assert_array_equal(O.noisy_logits(l, ln, np.zeros_like(n)), l)       # no draw: H = l
    np.testing.assert_allclose(O.noisy_logits(l, np.zeros_like(ln), n), l + n * math.log(2.0), rtol=1e-15)
    # a large noise logit passes the draw through at that scale (softplus(z) ~ z)
    np.testing.assert_allclose(O.noisy_logits(l, np.full_like(ln, 50.0), n), l + 50.0 * n, rtol=1e-13)


def test_noisy_top_k_without_noise_is_the_learned_softmax_router():
    rng = np.random.default_rng(6)
    l = rng.normal(0, 1, (40, 16))
    r = O.route_noisy(l, rng.normal(0, 1, (40, 16)), np.zeros((40, 16)), 4, scale=1.5)
    idx = O.top_k(l, 4)
    np.testing.assert_array_equal(r["topk_idx"], idx)
    np.testing.assert_allclose(r["topk_gate"], O.gates(l, idx, "softmax", True, 1.5), rtol=1e-15)


def test_noisy_top_k_follows_the_noise():
    """A draw large enough overturns the logit order: the noisy choice is the top-k of H,
    and its gates are the softmax over the kept H, summing to scale."""
    l = np.array([[3.0, 2.0, 1.0, 0.0]])
    ln = np.zeros((1, 4))
    n = np.array([[0.0, 0.0, 0.0, 10.0]])                       # H = [3, 2, 1, 10 ln 2]
    r = O.route_noisy(l, ln, n, 2, scale=2.0)
    assert r["topk_idx"].tolist() == [[3, 0]]
    h3 = 10.0 * math.log(2.0)
    e = np.exp(np.array([h3, 3.0]) - h3)
    np.testing.assert_allclose(r["topk_gate"][0], 2.0 * e / e.sum(), rtol=1e-15)
    # a negative draw pushes an expert out
    r = O.route_noisy(l, ln, np.array([[-5.0, 0.0, 0.0, 0.0]]), 2)
    assert r["topk_idx"].tolist() == [[1, 2]]


def test_noisy_top_k_ties_go_to_the_lower_index():
    l = np.zeros((1, 6))
    r = O.route_noisy(l, np.zeros((1, 6)), np.zeros((1, 6)), 3)
    assert r["topk_idx"].tolist() == [[0, 1, 2]]
    np.testing.assert_allclose(r["topk_gate"], 1.0 / 3, rtol=1e-15)

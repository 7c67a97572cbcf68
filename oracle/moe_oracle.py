"""CPU oracle for the token-choice top-k MoE-layer forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline / reference arm may import this module.  The library's
CUDA path never calls it, and it imports nothing from the library (the seeded
input generators live in a module of their own that holds no layer arithmetic).

Plain, slow and meant to be read against the pages by eye: numpy in float64,
one step per function, library primitives only for a matmul or a stable sort.

Sources (web pages on Mixture-of-Experts; cited by title and section):
  [MoE-Explained]  "Hugging Face 图解 Mixture of Experts（MoE）原理、训练与推理权衡"
                   (Chinese rendering of Hugging Face's "Mixture of Experts Explained"):
                   section "什么是稀疏性？" equations y = sum_i G(x)_i E_i(x),
                   G_sigma(x) = Softmax(x.W_g), KeepTopK(v,k), G(x) = Softmax(KeepTopK(H(x),k));
                   section "MoE 与 Transformer" (GShard expert capacity, overflow);
                   section "Switch Transformer" (Expert Capacity equation, capacity
                   factor, selective precision: the router in full precision);
                   section "使用路由器 Z-loss 稳定训练" (router z-loss).
  [Handbook-News]  "Hugging Face 团队投入 ~80 万 GPU 小时…「终极 MoE 训练手册」"
                   (hub.geekagi.cn): "真正难在三个环节" item 1 (FP32 routing),
                   item 2 (aux loss vs loss-free bias), and the quoted tweet
                   ("softmax, sigmoid or sqrt(softplus) router").
  [Handbook-Digest] "Hugging Face 发布 3 万词免费 MoE 训练手册" (agihunt.info),
                   "已确认": sqrt(softplus) scoring, routing scale factor near sqrt(k),
                   shared experts.
  [Handbook-Article] "Hugging Face开源MoE训练手册：基于80万GH200卡时沉淀Megatron-LM实战"
                   (zicq.com), "Router 与负载均衡为何决定训练成败" (capacity limit,
                   overflow tokens dropped; monitoring max load and drop rate).

Readings taken where the pages are silent (each listed again in the design notes):
  R1 capacity for k > 1 counts assignments: ceil(cf * T * k / E); the literal
     Switch form ceil(cf * T / E) is kept as an option (equal at k = 1).
  R2 capacity is rounded up (ceil).
  R3 drop priority is token order; a token's k experts are distinct.
  R4 a dropped assignment contributes 0; surviving gates are not re-normalised.
  R5 ties in the top-k go to the lower expert index.
  R6 selection key: the logit when no selection bias is given (KeepTopK acts on
     H = logits); with a selection bias, score(logit) + bias evaluated in fp64.
  R7 softmax gates are the softmax over the kept logits (eq. G).
  R8 the routing scale factor multiplies the gates after renormalisation.
  R9 expert FFN = SwiGLU: silu(x W_gate^T) * (x W_up^T), then W_down, no biases.
  R10 the shared expert is ungated (weight 1) and added after the routed sum.
  R11 bf16 workloads round H to bf16 (round to nearest even): it is the operand of the
     down projection, and the pages keep expert matmuls in bf16.  Gated expert rows,
     the shared output and y stay unrounded unless a bf16 output is asked for
     (round_rows / round_out); sums accumulate in float64 here.
  R12 router input: bf16 x upcast exactly; W_g and the logits in fp32 (exact on
     the generator's grids, so float64 here gives the same numbers).
  R13 an additive per-expert logit offset o[e] enters both selection and gates;
     the selection bias enters selection only.
  R15 aux loss = E * sum_e f_e P_e with f_e the pre-drop fraction of assignments
     and P_e the mean routing probability (softmax, or scores / their sum).
  R16 z-loss = mean_t (logsumexp_e l[t,e])^2.
  R20 forced-uniform routing: slot j of token t takes expert (t k + j) mod E.
  R21 hash routing: Floyd's sampling of k distinct experts driven by the MurmurHash3
     finalizer of the token id (hash_experts).
  R22 the fixed rules keep the learned path's gates over the chosen experts.
  R23 noisy top-k: the standard normal draws are an input; KeepTopK on H with ties to
     the lower index; gates = Softmax over the kept H.

Parity status: every function here is pinned by the CPU tests (brute force,
closed forms, invariants, hand-derived golden fixtures); none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

SCORE_KINDS = ("softmax", "sigmoid", "sqrt_softplus")


# ---------------------------------------------------------------------------
# Capacity  ([MoE-Explained] "Switch Transformer": Expert Capacity =
#            (tokens per batch / number of experts) x capacity factor; R1, R2)
# ---------------------------------------------------------------------------
def capacity(T: int, E: int, k: int, capacity_factor: Optional[float],
             per_assignment: bool = True) -> int:
    """Slots per expert; -1 means no dropping (capacity_factor None or <= 0)."""
    if capacity_factor is None or capacity_factor <= 0:
        return -1
    tokens = T * k if per_assignment else T
    return int(math.ceil(float(capacity_factor) * tokens / E))


# ---------------------------------------------------------------------------
# Router  ([MoE-Explained] eq. G_sigma(x) = Softmax(x . W_g); R12, R13)
# ---------------------------------------------------------------------------
def router_logits(x, Wg, logit_offset=None) -> np.ndarray:
    """l[t, e] = sum_c x[t, c] * Wg[c, e] + o[e]   (float64 result)."""
    l = np.asarray(x, np.float64) @ np.asarray(Wg, np.float64)
    if logit_offset is not None:
        l = l + np.asarray(logit_offset, np.float64)[None, :]
    return l


def softmax(v: np.ndarray) -> np.ndarray:
    """Row softmax, max-shifted."""
    m = v.max(axis=-1, keepdims=True)
    e = np.exp(v - m)
    return e / e.sum(axis=-1, keepdims=True)


def router_scores(logits: np.ndarray, score: str) -> np.ndarray:
    """Per-expert scores: softmax over experts, sigmoid, or sqrt(softplus).

    [Handbook-News] tweet: "softmax, sigmoid or sqrt(softplus) router";
    [Handbook-Digest]: DeepSeek-V4 moved its scoring from sigmoid to sqrt(softplus).
    softplus(l) = log(1 + e^l) is written max(l,0) + log1p(e^-|l|) (same value, no overflow).
    """
    l = np.asarray(logits, np.float64)
    if score == "softmax":
        return softmax(l)
    if score == "sigmoid":
        return 1.0 / (1.0 + np.exp(-l))
    if score == "sqrt_softplus":
        return np.sqrt(np.maximum(l, 0.0) + np.log1p(np.exp(-np.abs(l))))
    raise ValueError(score)


def selection_keys(logits: np.ndarray, score: str, select_bias=None) -> np.ndarray:
    """Key the top-k ranks by (R6): logits, or score + bias in float64.

    [MoE-Explained] eq. KeepTopK acts on H(x) = the logits; [Handbook-News] item 2
    (loss-free balancing bias) shifts which experts are chosen, not the gates.
    """
    l = np.asarray(logits, np.float64)
    if select_bias is None:
        return l.copy()
    return router_scores(l, score) + np.asarray(select_bias, np.float64)[None, :]


def top_k(keys: np.ndarray, k: int) -> np.ndarray:
    """The k largest keys per row; order key descending, then expert index ascending (R5).

    [MoE-Explained] eq. KeepTopK(v, k).  A stable sort on -key keeps equal keys in
    index order, so ties go to the lower index.
    """
    order = np.argsort(-np.asarray(keys, np.float64), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gates(logits: np.ndarray, idx: np.ndarray, score: str, renormalize: bool,
          scale: float) -> np.ndarray:
    """Gate weight of each kept expert (float64), in the order of idx.

    softmax + renormalize: softmax over the kept logits ([MoE-Explained] eq.
      G(x) = Softmax(KeepTopK(H(x), k)), R7);
    softmax, no renormalize: the full softmax probability (eq. G_sigma);
    sigmoid / sqrt(softplus): kept scores divided by their sum, or the raw scores
      without renormalize.  Scores exclude the selection bias (R13).
    Then x scale ([Handbook-Digest] routing scale factor, R8).
    """
    l = np.asarray(logits, np.float64)
    T = l.shape[0]
    kept_l = l[np.arange(T)[:, None], idx]
    if score == "softmax":
        if renormalize:
            g = softmax(kept_l)
        else:
            g = softmax(l)[np.arange(T)[:, None], idx]
    else:
        s = router_scores(kept_l, score)
        g = s / s.sum(axis=1, keepdims=True) if renormalize else s
    return g * float(scale)


def route(x, Wg, k: int, score: str = "softmax", renormalize: bool = True,
          scale: float = 1.0, logit_offset=None, select_bias=None) -> dict:
    """Router + KeepTopK + gates for every token."""
    l = router_logits(x, Wg, logit_offset)
    keys = selection_keys(l, score, select_bias)
    idx = top_k(keys, k)
    g = gates(l, idx, score, renormalize, scale)
    return {"logits": l, "keys": keys, "topk_idx": idx, "topk_gate": g}


def decision_margin(keys: np.ndarray, k: int) -> np.ndarray:
    """Per token: k-th largest key minus (k+1)-th largest key (inf when k = E).

    A token whose margin is below the key precision can legitimately be routed
    either way by two correct implementations; tests compare only what is unique.
    """
    E = keys.shape[1]
    if k >= E:
        return np.full(keys.shape[0], np.inf)
    s = -np.sort(-np.asarray(keys, np.float64), axis=1)
    return s[:, k - 1] - s[:, k]


# ---------------------------------------------------------------------------
# Routing variants
#   forced-uniform selection: [Handbook-News] "真正难在三个环节" item 2 (a control run
#     that forced routing to be uniform was about 1.5x faster; it shows the speed
#     headroom only, not a training recipe);
#   hash selection by token id: [Handbook-Digest] "已确认", routing bullet (the first
#     three MoE layers of DeepSeek-V4 choose experts by a fixed hash of the token id);
#   noisy top-k: [MoE-Explained] "什么是稀疏性？", eq. H(x)_i = (x.W_g)_i +
#     StandardNormal() * Softplus((x.W_noise)_i), then KeepTopK and Softmax.
# The pages give neither the hash nor the gates of the fixed rules (R20-R23).
# ---------------------------------------------------------------------------
MASK32 = 0xFFFFFFFF


def fmix32(h: int) -> int:
    """The MurmurHash3 32-bit finalizer (Appleby): two xor-shift-multiply rounds and a
    final xor-shift, all modulo 2^32.  A bijection on 32-bit words."""
    h &= MASK32
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & MASK32
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & MASK32
    h ^= h >> 16
    return h


def floyd_sample(words, E: int, k: int) -> list:
    """k distinct values out of range(E) from k 32-bit words, by Floyd's sampling
    (Bentley and Floyd, "A sample of brilliance"): for j = 0 .. k-1 with n = E - k + j,
    r = words[j] mod (n + 1); take r unless it is already taken, else take n (never
    taken yet: earlier picks are all below it).  With uniform words every k-subset is
    equally likely (up to the modulo bias of a 32-bit word).  Keeps the draw order."""
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    chosen = []
    for j in range(k):
        n = E - k + j
        r = int(words[j]) % (n + 1)
        chosen.append(n if r in chosen else r)
    return chosen


def hash_experts(token_id: int, seed: int, E: int, k: int) -> list:
    """The k experts of a token id (R21): floyd_sample of the words
    h_j = fmix32(fmix32(id xor seed) + j), j = 0 .. k-1."""
    base = fmix32((token_id & MASK32) ^ (seed & MASK32))
    return floyd_sample([fmix32((base + j) & MASK32) for j in range(k)], E, k)


def fixed_selection(T: int, E: int, k: int, rule: str, token_id=None, seed: int = 0) -> np.ndarray:
    """topk_idx [T, k] of a fixed rule.

    "uniform" (R20): slot j of token t takes expert (t k + j) mod E, so every expert
      receives floor(T k / E) or ceil(T k / E) assignments;
    "hash" (R21): hash_experts(token_id[t], seed, E, k).
    """
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        if rule == "uniform":
            idx[t] = [(t * k + j) % E for j in range(k)]
        elif rule == "hash":
            idx[t] = hash_experts(int(token_id[t]), seed, E, k)
        else:
            raise ValueError(rule)
    return idx


def route_fixed(logits, k: int, score: str, renormalize: bool, scale: float, rule: str,
                token_id=None, seed: int = 0) -> dict:
    """A fixed selection rule with the learned path's gates over the chosen experts (R22)."""
    l = np.asarray(logits, np.float64)
    idx = fixed_selection(l.shape[0], l.shape[1], k, rule, token_id, seed)
    return {"topk_idx": idx, "topk_gate": gates(l, idx, score, renormalize, scale)}


def softplus(z):
    """log(1 + e^z), written max(z, 0) + log1p(e^-|z|) (same value, no overflow)."""
    z = np.asarray(z, np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def noisy_logits(logits, logits_noise, noise) -> np.ndarray:
    """H = l + n * softplus(l_noise) ([MoE-Explained] eq. H(x)_i; the StandardNormal()
    draws n are an input, R23)."""
    return np.asarray(logits, np.float64) + np.asarray(noise, np.float64) * softplus(logits_noise)


def route_noisy(logits, logits_noise, noise, k: int, scale: float = 1.0) -> dict:
    """Noisy top-k gating: KeepTopK on H (ties to the lower index), then the softmax over
    the kept H ([MoE-Explained] eq. G(x) = Softmax(KeepTopK(H(x), k))), times scale."""
    H = noisy_logits(logits, logits_noise, noise)
    idx = top_k(H, k)
    return {"H": H, "topk_idx": idx, "topk_gate": gates(H, idx, "softmax", True, scale)}


# ---------------------------------------------------------------------------
# Capacity dropping + permutation plan
#   [MoE-Explained] "MoE 与 Transformer": an expert takes at most `capacity`
#   tokens, the overflow goes through the residual (or is dropped);
#   [Handbook-Article] capacity limit: tokens beyond it are dropped.  R3, R4.
# ---------------------------------------------------------------------------
def dispatch_plan(topk_idx: np.ndarray, topk_gate: np.ndarray, E: int, cap: int) -> dict:
    """Counts, kept counts, expert-contiguous row offsets and the row maps.

    rank(t, j) = number of tokens t' < t that chose expert idx[t, j]
    (stable sort of the assignments by expert keeps token order inside an expert);
    an assignment is kept when rank < cap (cap < 0: always);
    offsets = exclusive scan of kept counts; row_of[t, j] = offsets[e] + rank or -1.
    """
    idx = np.asarray(topk_idx, np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)                       # assignment a = t*k + j, token order
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    order = np.argsort(flat, kind="stable")      # grouped by expert, token order inside
    start = np.concatenate([[0], np.cumsum(counts)])
    rank = np.empty(T * k, np.int64)
    rank[order] = np.arange(T * k) - start[flat[order]]
    kept = counts.copy() if cap < 0 else np.minimum(counts, cap)
    offsets = np.concatenate([[0], np.cumsum(kept)]).astype(np.int64)
    keep = rank < (cap if cap >= 0 else T * k + 1)
    row_of = np.where(keep, offsets[flat] + rank, -1).reshape(T, k)
    n_rows = int(offsets[-1])
    token_of_row = np.full(n_rows, -1, np.int64)
    gate_of_row = np.zeros(n_rows, np.float64)
    a = np.nonzero(keep)[0]
    token_of_row[row_of.reshape(-1)[a]] = a // k
    gate_of_row[row_of.reshape(-1)[a]] = np.asarray(topk_gate, np.float64).reshape(-1)[a]
    return {"counts": counts, "kept": kept, "offsets": offsets, "row_of": row_of,
            "token_of_row": token_of_row, "gate_of_row": gate_of_row, "rank": rank.reshape(T, k)}


def permute(x, row_of: np.ndarray, n_rows: int) -> np.ndarray:
    """x_perm[row_of[t, j]] = x[t] for every kept assignment."""
    x = np.asarray(x, np.float64)
    T, k = row_of.shape
    out = np.zeros((n_rows, x.shape[1]), np.float64)
    for j in range(k):
        m = row_of[:, j] >= 0
        out[row_of[m, j]] = x[m]
    return out


# ---------------------------------------------------------------------------
# Expert FFN (R9, R11)
# ---------------------------------------------------------------------------
def bf16_round(a) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even), as float64.

    bf16 keeps 8 significant bits: v = m * 2^e with m in [0.5, 1) is rounded to
    rint(m * 2^8) * 2^(e - 8); rint rounds half to even.  (Exponent range is
    never reached by the values this layer produces; inf/nan pass through.)
    """
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    return np.where(np.isfinite(a), r, a)


def silu(z):
    return z / (1.0 + np.exp(-z))


def expert_hidden(x_rows, W_gu, bf16: bool) -> np.ndarray:
    """H = silu(x W_gate^T) * (x W_up^T) for one expert, float64 accumulate.

    W_gu [2F, d]: rows 0..F-1 are W_gate, rows F..2F-1 are W_up.
    bf16: H is rounded to bf16, as it is before the down projection (R11).
    """
    x = np.asarray(x_rows, np.float64)
    W_gu = np.asarray(W_gu, np.float64)
    F = W_gu.shape[0] // 2
    g = x @ W_gu[:F].T
    u = x @ W_gu[F:].T
    h = silu(g) * u
    return bf16_round(h) if bf16 else h


def swiglu_expert(x_rows, W_gu, W_dn, bf16: bool) -> np.ndarray:
    """One expert on a block of rows: H W_dn^T with H from expert_hidden; W_dn [d, F]."""
    return expert_hidden(x_rows, W_gu, bf16) @ np.asarray(W_dn, np.float64).T


def grouped_ffn(x_perm, offsets, W_gu_of, W_dn_of, gate_of_row, bf16: bool,
                round_rows: bool = False) -> np.ndarray:
    """y_perm[r] = gate_of_row[r] * expert_e(x_perm[r]) for r in [offsets[e], offsets[e+1]).

    W_gu_of(e) / W_dn_of(e) return expert e's weights (arrays or callables).
    bf16: H is rounded to bf16; round_rows: each gated row is rounded to bf16 too (R11).
    """
    x_perm = np.asarray(x_perm, np.float64)
    E = len(offsets) - 1
    d_out = np.asarray(_get(W_dn_of, 0)).shape[0]
    y = np.zeros((x_perm.shape[0], d_out), np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b <= a:
            continue
        o = swiglu_expert(x_perm[a:b], _get(W_gu_of, e), _get(W_dn_of, e), bf16)
        o = o * (1.0 if gate_of_row is None else np.asarray(gate_of_row, np.float64)[a:b, None])
        y[a:b] = bf16_round(o) if round_rows else o
    return y


def _get(W, e):
    return W(e) if callable(W) else W[e]


def shared_expert(x, W_gu_s, W_dn_s, bf16: bool, round_out: bool = False) -> np.ndarray:
    """Always-on expert with weight 1 (R10; [Handbook-Digest] shared experts)."""
    y = swiglu_expert(x, W_gu_s, W_dn_s, bf16)
    return bf16_round(y) if round_out else y


# ---------------------------------------------------------------------------
# Combine  ([MoE-Explained] eq. y = sum_i G(x)_i E_i(x); R4, R10, R11)
# ---------------------------------------------------------------------------
def combine(y_perm, row_of: np.ndarray, shared_y=None, round_out: bool = False,
            topk_gate=None) -> np.ndarray:
    """y[t] = sum_j y_perm[row_of[t, j]] (dropped slots skipped) + shared_y[t].

    topk_gate given: rows are multiplied by their gate here (rows not gated yet).
    round_out: y is rounded to bf16 (R11).
    """
    y_perm = np.asarray(y_perm, np.float64)
    T, k = row_of.shape
    y = np.zeros((T, y_perm.shape[1]), np.float64)
    for j in range(k):
        m = row_of[:, j] >= 0
        rows = y_perm[row_of[m, j]]
        if topk_gate is not None:
            rows = rows * np.asarray(topk_gate, np.float64)[m, j][:, None]
        y[m] += rows
    if shared_y is not None:
        y += np.asarray(shared_y, np.float64)
    return bf16_round(y) if round_out else y


# ---------------------------------------------------------------------------
# The layer, end to end, for all tokens or for a subset of tokens
# ---------------------------------------------------------------------------
def layer_routing(cfg_like: dict, x, Wg, logit_offset=None, select_bias=None,
                  per_assignment_capacity: bool = True) -> dict:
    """Router, top-k, gates and the dispatch plan for every token.

    cfg_like: mapping with T, E, k, score, renormalize, scale, capacity_factor.
    """
    c = cfg_like
    r = route(x, Wg, c["k"], c["score"], c["renormalize"], c["scale"], logit_offset, select_bias)
    cap = capacity(c["T"], c["E"], c["k"], c.get("capacity_factor"), per_assignment_capacity)
    plan = dispatch_plan(r["topk_idx"], r["topk_gate"], c["E"], cap)
    r.update(plan)
    r["capacity"] = cap
    return r


def layer_outputs_for_tokens(tokens, x, routing: dict, W_gu_of, W_dn_of, bf16: bool,
                             shared=None, round_rows: bool = False, round_out: bool = False) -> dict:
    """y[t] (and each kept slot's gated expert row) for the listed tokens only.

    A token's output depends only on its own row, its routing and the weights,
    so evaluating a subset gives exactly the rows the full layer would.
    shared: (W_gu_s, W_dn_s) or None.  Rounding flags as in grouped_ffn / combine.
    """
    tokens = np.asarray(tokens, np.int64)
    xs = np.asarray(np.asarray(x)[tokens], np.float64)          # the listed tokens only
    idx = routing["topk_idx"][tokens]
    row_of = routing["row_of"][tokens]
    g = np.asarray(routing["topk_gate"], np.float64)[tokens]
    n, k = idx.shape
    d = xs.shape[1]
    slot_rows = np.zeros((n, k, d), np.float64)
    kept = row_of >= 0
    for e in np.unique(idx[kept]):                  # every kept (token, slot) of expert e at once
        ii, jj = np.nonzero((idx == e) & kept)
        o = swiglu_expert(xs[ii], _get(W_gu_of, int(e)), _get(W_dn_of, int(e)), bf16)
        o = o * g[ii, jj][:, None]
        slot_rows[ii, jj] = bf16_round(o) if round_rows else o
    acc = np.zeros((n, d), np.float64)
    for j in range(k):                              # slot order; dropped slots are zero rows
        acc += slot_rows[:, j]
    if shared is not None:
        acc += shared_expert(xs, shared[0], shared[1], bf16, round_rows)
    y = bf16_round(acc) if round_out else acc
    return {"y": y, "slot_rows": slot_rows}


def layer_forward(cfg_like: dict, x, Wg, W_gu, W_dn, logit_offset=None, select_bias=None,
                  shared=None, bf16: bool = True, per_assignment_capacity: bool = True,
                  round_rows: bool = False, round_out: bool = False) -> dict:
    """The whole layer for all tokens (small sizes): routing, permute, grouped FFN, combine."""
    r = layer_routing(cfg_like, x, Wg, logit_offset, select_bias, per_assignment_capacity)
    n_rows = int(r["offsets"][-1])
    x_perm = permute(x, r["row_of"], n_rows)
    y_perm = grouped_ffn(x_perm, r["offsets"], W_gu, W_dn, r["gate_of_row"], bf16, round_rows)
    ys = shared_expert(x, shared[0], shared[1], bf16, round_rows) if shared is not None else None
    y = combine(y_perm, r["row_of"], ys, round_out)
    r.update({"x_perm": x_perm, "y_perm": y_perm, "shared_y": ys, "y": y})
    return r


def dense_mixture(x, Wg, W_gu, W_dn, logit_offset=None) -> np.ndarray:
    """y = sum_i G_sigma(x)_i E_i(x) over ALL experts, no rounding
    ([MoE-Explained] eqs. y and G_sigma): the k = E, no-drop limit of the layer."""
    l = router_logits(x, Wg, logit_offset)
    p = softmax(l)
    x = np.asarray(x, np.float64)
    y = np.zeros_like(x)
    for e in range(p.shape[1]):
        y += p[:, e:e + 1] * swiglu_expert(x, _get(W_gu, e), _get(W_dn, e), bf16=False)
    return y


# ---------------------------------------------------------------------------
# Router statistics  ([MoE-Explained] aux loss in "为 MoE 平衡 token 负载" and
#   "Switch Transformer"; z-loss in "使用路由器 Z-loss 稳定训练";
#   [Handbook-Article] monitoring: max/mean load, drop rate.  R15, R16)
# ---------------------------------------------------------------------------
def router_stats(logits, counts, kept, k: int, score: str) -> dict:
    """load f_e, aux, z, dropped, max/mean load, coefficient of variation."""
    l = np.asarray(logits, np.float64)
    T, E = l.shape
    counts = np.asarray(counts, np.float64)
    kept = np.asarray(kept, np.float64)
    f = counts / (T * k)
    if score == "softmax":
        p = softmax(l)
    else:
        s = router_scores(l, score)
        p = s / s.sum(axis=1, keepdims=True)
    P = p.mean(axis=0)
    aux = E * float(np.sum(f * P))
    m = l.max(axis=1)
    lse = m + np.log(np.exp(l - m[:, None]).sum(axis=1))
    z = float(np.mean(lse ** 2))
    dropped = float(T * k - kept.sum())
    mean = T * k / E
    max_over_mean = float(counts.max() / mean)
    cv = float(counts.std() / mean)
    return {"load": f, "aux": aux, "z": z, "dropped": dropped,
            "max_over_mean": max_over_mean, "cv": cv}

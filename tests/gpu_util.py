"""Helpers for the GPU parity tests: run the layer through the C ABI, run the oracle on
the same seeded inputs, and compare them element by element.

Bars (from the layer's acceptance criteria):
  routing indices, counts, kept, offsets, row maps, permuted rows: bit-exact;
  logits: bit-exact (the generator's grids make fp32 sums exact);
  gates: |err| <= 1e-6 * |gate|;
  layer output y (fp32 rows and output, the default): max|err| <= 2e-2 * rms(y) and
  mean|err| <= 2e-3 * rms(y).
Derived bars (where a result passes through extra bf16 roundings; see each helper):
  gated expert rows: componentwise bound from H's bf16 rounding;
  bf16 rows + bf16 output: componentwise bound from every rounding point.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_moe_b200 import inputs as I

GATE_RTOL = 1e-6
Y_MAX_REL = 2e-2
Y_MEAN_REL = 2e-3


def cfg_dict(cfg):
    return dict(T=cfg.T, E=cfg.E, k=cfg.k, score=cfg.score, renormalize=cfg.renormalize, scale=cfg.scale,
                capacity_factor=cfg.capacity_factor)


def act_dtype(cfg):
    return torch.float32 if cfg.act == "f32" else torch.bfloat16


def make_inputs(cfg, seed=0, device="cuda"):
    """Seeded inputs on the host (numpy / torch CPU) and their device copies."""
    x = I.gen_x(cfg, seed)
    Wg, off, bias = I.gen_router(cfg, seed)
    W_gu, W_dn = I.gen_experts_torch(cfg, seed)
    sh = I.gen_shared(cfg, seed)
    dt = act_dtype(cfg)
    dev = {
        "x": torch.from_numpy(x).to(dt).to(device),
        "Wg": torch.from_numpy(Wg).to(device),
        "off": None if off is None else torch.from_numpy(off).to(device),
        "bias": None if bias is None else torch.from_numpy(bias).to(device),
        "W_gu": W_gu.to(device),
        "W_dn": W_dn.to(device),
        "W_gu_s": None if sh is None else torch.from_numpy(sh[0]).to(dt).unsqueeze(0).to(device),
        "W_dn_s": None if sh is None else torch.from_numpy(sh[1]).to(dt).unsqueeze(0).to(device),
    }
    host = {"x": x, "Wg": Wg, "off": off, "bias": bias, "W_gu": W_gu, "W_dn": W_dn, "shared": sh}
    return host, dev


def expert_getters(host):
    """Per-expert float64 weights for the oracle (converted on demand, cached)."""
    cache_gu, cache_dn = {}, {}

    def gu(e):
        if e not in cache_gu:
            cache_gu[e] = host["W_gu"][e].double().numpy()
        return cache_gu[e]

    def dn(e):
        if e not in cache_dn:
            cache_dn[e] = host["W_dn"][e].double().numpy()
        return cache_dn[e]

    return gu, dn


def build_layer(cfg, dev, capacity, rows_dtype=torch.float32, out_dtype=torch.float32, combine="rows",
                dispatch="permute"):
    from routing_dispatch_expert_moe_b200.layer import MoELayer, MoEWeights
    w = MoEWeights(Wg=dev["Wg"], W_gu=dev["W_gu"], W_dn=dev["W_dn"], logit_offset=dev["off"],
                   select_bias=dev["bias"], W_gu_s=dev["W_gu_s"], W_dn_s=dev["W_dn_s"])
    return MoELayer(w, cfg.k, cfg.T, cfg.score, cfg.renormalize, cfg.scale, capacity, rows_dtype, out_dtype,
                    combine, dispatch)


def gpu_forward(cfg, dev, capacity, rows_dtype=torch.float32, out_dtype=torch.float32, combine="rows",
                dispatch="permute"):
    """Runs the layer through the C ABI; returns the layer object and host copies of every output."""
    from routing_dispatch_expert_moe_b200 import moe as M
    layer = build_layer(cfg, dev, capacity, rows_dtype, out_dtype, combine, dispatch)
    y = layer.forward(dev["x"])
    torch.cuda.synchronize()
    code = M.moe_get_device_error()
    assert code == 0, f"device error {code} ({M.DEVERR.get(code)})"
    n = int(layer.offsets[-1].item())
    out = {
        "logits": layer.logits.cpu().numpy(),
        "topk_idx": layer.topk_idx.cpu().numpy(),
        "topk_gate": layer.topk_gate.cpu().numpy(),
        "counts": layer.counts.cpu().numpy(),
        "kept": layer.kept.cpu().numpy(),
        "offsets": layer.offsets.cpu().numpy(),
        "row_of": layer.row_of.cpu().numpy(),
        "token_of_row": layer.token_of_row[:n].cpu().numpy(),
        "gate_of_row": layer.gate_of_row[:n].cpu().numpy(),
        "n_rows": n,
        "y": y.float().cpu().numpy().astype(np.float64),
        "load": layer.load.cpu().numpy(),
        "stats5": layer.stats5.cpu().numpy(),
    }
    return layer, out


def assert_routing_equal(g, o, exact_logits=True):
    if exact_logits:
        assert np.array_equal(g["logits"].astype(np.float64), o["logits"]), "logits not bit-exact"
    else:
        np.testing.assert_allclose(g["logits"], o["logits"], rtol=1e-5, atol=1e-5)
    assert np.array_equal(g["topk_idx"], o["topk_idx"]), \
        f"topk_idx differs on {int((g['topk_idx'] != o['topk_idx']).any(1).sum())} tokens"
    go = o["topk_gate"]
    err = np.abs(g["topk_gate"].astype(np.float64) - go)
    assert (err <= GATE_RTOL * np.abs(go) + 1e-30).all(), f"gate rel err {float((err / np.abs(go)).max()):.3g}"
    for key in ("counts", "kept", "offsets", "row_of"):
        assert np.array_equal(g[key], o[key]), f"{key} differs"
    n = int(o["offsets"][-1])
    assert g["n_rows"] == n
    assert np.array_equal(g["token_of_row"], o["token_of_row"][:n]), "token_of_row differs"
    ge = np.abs(g["gate_of_row"].astype(np.float64) - o["gate_of_row"][:n])
    assert (ge <= GATE_RTOL * np.abs(o["gate_of_row"][:n]) + 1e-30).all()


def bf16_step(v):
    """Spacing of bf16 values at |v| (8 significant bits): 2^(floor(log2|v|) - 7)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def row_bounds(x, tokens, experts, gates, gu, dn, bf16=True):
    """Componentwise bound on how far a correct gated row may sit from the oracle's.

    Both sides round H to bf16 from values that differ only by accumulation order, so any
    H element may land one bf16 step (<= 2^-8 |h|) away; that moves output n by at most
    2^-8 * gate * sum_f |h_f| |W_dn[n, f]|.  Returns that bound per row (float64).
    """
    x = np.asarray(x)
    out = np.zeros((len(tokens), dn(int(experts[0])).shape[0] if len(tokens) else 0), np.float64)
    if not bf16:                      # fp32 activations: H is not rounded on either side
        return out
    for e in np.unique(experts):
        i = np.nonzero(experts == e)[0]
        h = O.expert_hidden(np.asarray(x[tokens[i]], np.float64), gu(int(e)), bf16)
        out[i] = 2.0 ** -8 * np.abs(np.asarray(gates, np.float64)[i])[:, None] * (np.abs(h) @ np.abs(dn(int(e))).T)
    return out


def assert_rows_close(gy, oy, hbound, what="y_perm", rows_bf16=False):
    """Gated expert rows: each element within the H-rounding bound plus fp32 accumulation
    slack (1e-5 relative, 1e-6 of the rms), and one bf16 step of its magnitude when the
    rows themselves are stored in bf16; mean error within 2e-3 * rms."""
    gy = np.asarray(gy, np.float64)
    oy = np.asarray(oy, np.float64)
    rms = float(np.sqrt(np.mean(oy ** 2)))
    err = np.abs(gy - oy)
    bound = hbound + 1e-5 * np.abs(oy) + 1e-6 * rms
    if rows_bf16:
        bound = bound + bf16_step(np.maximum(np.abs(gy), np.abs(oy)))
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond the bound; worst err "
                           f"{float(err[bad].max()):.4g} at |ref| {float(np.abs(oy[bad]).max()):.4g}, rms {rms:.4g}")
    assert float(err.mean()) <= Y_MEAN_REL * rms, f"{what}: mean|err| {float(err.mean()):.4g} > {Y_MEAN_REL} * rms"
    return float(err.max()) / rms, float(err.mean()) / rms


def y_errors(gy, oy):
    rms = float(np.sqrt(np.mean(oy ** 2)))
    err = np.abs(gy - oy)
    return float(err.max()), float(err.mean()), rms


def assert_y_close(gy, oy, what="y"):
    mx, mean, rms = y_errors(gy, oy)
    assert rms > 0, f"{what}: reference is all zeros"
    assert mx <= Y_MAX_REL * rms, f"{what}: max|err| {mx:.4g} > {Y_MAX_REL} * rms {rms:.4g}"
    assert mean <= Y_MEAN_REL * rms, f"{what}: mean|err| {mean:.4g} > {Y_MEAN_REL} * rms {rms:.4g}"
    return mx / rms, mean / rms


def assert_y_close_bf16(gy, oy, slot_rows, slot_hbound, shared_y=None):
    """bf16 rows and bf16 output: componentwise bound derived from the rounding points.

    y[t] = bf16(sum_j row_j + shared); each row_j may differ by its own bound (one bf16
    step of the row element plus the H-rounding bound), the shared row by one step, and
    the final rounding by one bf16 step of y.  Mean error obeys the 2e-3 * rms bar.
    slot_rows / slot_hbound: [T, k, d] oracle rows and their H bounds (zeros where dropped).
    """
    gy = np.asarray(gy, np.float64)
    oy = np.asarray(oy, np.float64)
    b = bf16_step(np.maximum(np.abs(gy), np.abs(oy)))
    rows = np.asarray(slot_rows, np.float64)
    b = b + (np.where(rows != 0, bf16_step(rows), 0.0) + slot_hbound).sum(axis=1)
    if shared_y is not None:
        b = b + bf16_step(shared_y)
    rms = float(np.sqrt(np.mean(oy ** 2)))
    err = np.abs(gy - oy)
    bad = err > b + 1e-6 * rms
    assert not bad.any(), f"y (bf16): {int(bad.sum())} elements beyond the bound, worst {float(err.max()):.4g}"
    assert float(err.mean()) <= Y_MEAN_REL * rms
    return float(err.max()) / rms, float(err.mean()) / rms


def bar_report(gy, oy):
    """The layer's stated bar (max|err| <= 2e-2 rms, mean|err| <= 2e-3 rms) on a bf16 output:
    observed max and mean error over rms, and the elements past the max bar with their
    error counted in bf16 steps of the reference value (a correct sum in a different order
    may land one step away, and one step at |y| > 4 rms is more than 2e-2 rms)."""
    gy = np.asarray(gy, np.float64)
    oy = np.asarray(oy, np.float64)
    rms = float(np.sqrt(np.mean(oy ** 2)))
    err = np.abs(gy - oy)
    over = err > Y_MAX_REL * rms
    steps = err[over] / bf16_step(oy[over]) if over.any() else np.zeros(0)
    return {"max_rel": float(err.max()) / rms, "mean_rel": float(err.mean()) / rms, "n": int(err.size),
            "n_over_max_bar": int(over.sum()), "max_steps_over": float(steps.max()) if steps.size else 0.0,
            "min_abs_over_rms": float(np.abs(oy[over]).min() / rms) if over.any() else None}


def assert_stats_close(g, o_stats, dropped_exact=True):
    np.testing.assert_allclose(g["load"], o_stats["load"], rtol=1e-6, atol=0)
    s = g["stats5"].astype(np.float64)
    assert abs(s[0] - o_stats["aux"]) <= 1e-5 * abs(o_stats["aux"]) + 1e-7, (s[0], o_stats["aux"])
    assert abs(s[1] - o_stats["z"]) <= 1e-5 * abs(o_stats["z"]) + 1e-7, (s[1], o_stats["z"])
    assert s[2] == o_stats["dropped"]
    assert abs(s[3] - o_stats["max_over_mean"]) <= 1e-6 * o_stats["max_over_mean"]
    assert abs(s[4] - o_stats["cv"]) <= 1e-5 * o_stats["cv"] + 1e-7


def stratified_tokens(o, cap, n_random=1100, seed=0):
    """Hottest / coldest non-empty expert's tokens, capacity-boundary and fully dropped
    tokens, plus random ones (each token's output depends only on its own row)."""
    idx, row_of, rank = o["topk_idx"], o["row_of"], o["rank"]
    T = idx.shape[0]
    counts = o["counts"]
    picks = []
    hot = int(np.argmax(counts))
    nz = np.nonzero(counts)[0]
    cold = int(nz[np.argmin(counts[nz])])
    for e in (hot, cold):
        toks = np.nonzero((idx == e).any(1))[0]
        picks += list(toks[:64]) + list(toks[-32:])
    if cap >= 0:
        b = np.nonzero(((rank == cap - 1) | (rank == cap)).any(1))[0]
        picks += list(b[:128])
        fully = np.nonzero((row_of < 0).all(1))[0]
        picks += list(fully[:64])
        part = np.nonzero((row_of < 0).any(1) & (row_of >= 0).any(1))[0]
        picks += list(part[:64])
    rng = np.random.default_rng(seed)
    picks += list(rng.choice(T, size=min(n_random, T), replace=False))
    picks += [0, T - 1]
    out = np.unique(np.array(picks, np.int64))
    return out

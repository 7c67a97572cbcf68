"""GPU parity of the grouped expert GEMMs with 4-bit expert weights (MXFP4, NVFP4).

Handbook digest (agihunt.info), "已确认", bullet "量化与推理": routed experts in MXFP4,
NVFP4 with key layers kept in BF16.  The experts run on the dequantized weights (code value
x block scale x tensor scale); activations, H and the gated rows keep the bf16 path's
rounding points, so the bars are those of the bf16 layer with the dequantized weights in
place of the bf16 ones:

  * exact: every dequantized MXFP4 weight (and every NVFP4 weight before the tensor scale)
    is a bf16 value, so the 4-bit GEMMs must equal, bit for bit, the bf16 weight-major GEMMs
    run on those bf16 values -- the converter's output is checked exactly;
  * the whole layer with 4-bit experts against the oracle (codes from the oracle's own
    quantizer, weights decoded by the oracle) on small shapes, every output compared;
  * the stress workload at full size with synthetic codes and scales, sampled tokens.
"""
import numpy as np
import pytest
import torch

from oracle import fp4 as Q
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
    assert _M().moe_get_device_error() == 0


def synthetic_fp4(rows, K, fmt, seed, E=1):
    """Random codes and scale bytes in the packed layout (weights of magnitude ~0.02), and a
    per-expert tensor scale for NVFP4."""
    rng = np.random.default_rng([seed, 95])
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    if fmt == "mxfp4":
        scales = rng.integers(119, 123, size=(rows, K // 32), dtype=np.uint8)      # 2^-8 .. 2^-5
        ts = None
    else:
        scales = rng.integers(0x30, 0x50, size=(rows, K // 16), dtype=np.uint8)    # E4M3 0.25 .. 4
        ts = (2.0 ** -rng.integers(6, 9, size=E)).astype(np.float32)
    return codes, scales, ts


def to_device(fmt, codes, scales, ts):
    M = _M()
    return M.Fp4Weights(fmt, torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                        None if ts is None else torch.from_numpy(ts).cuda())


def _groups(E, rows_each, seed):
    rng = np.random.default_rng(seed)
    counts = np.array(rows_each if len(rows_each) == E else rng.integers(0, 300, E))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return counts, offsets


# ------------------------------------------------------------------ the prepared scale layout
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_prepared_scales_are_the_documented_rearrangement(fmt):
    rows, K = 384, 320
    _, scales, _ = synthetic_fp4(rows, K, fmt, seed=9)
    w = to_device(fmt, np.zeros((rows, K // 2), np.uint8), scales, np.ones(1, np.float32) if fmt == "nvfp4" else None)
    torch.cuda.synchronize()
    spr = 64 // (32 if fmt == "mxfp4" else 16)
    want = np.zeros((K // 64, rows + 256, spr), np.uint8)
    for kb in range(K // 64):
        want[kb, :rows] = scales[:, kb * spr:(kb + 1) * spr]
    got = w.scales_prepared.cpu().numpy()
    assert got.size == want.size and np.array_equal(got.reshape(want.shape), want)


# ------------------------------------------------------------------ exact against the bf16 GEMMs
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("E,d,F,rows_each", [(5, 128, 192, [0, 1, 45, 300, 129]), (3, 256, 64, [256, 97, 33]),
                                              (2, 512, 320, [513, 0])])
def test_fp4_gemms_equal_the_bf16_gemms_on_the_decoded_weights(fmt, E, d, F, rows_each, monkeypatch):
    M = _M()
    monkeypatch.setenv("MOE_B200_EXPERT_TILES", "weights")      # the same tiles and k order
    counts, offsets = _groups(E, rows_each, seed=E + d)
    R = int(offsets[-1])
    rng = np.random.default_rng(3)
    x = torch.from_numpy(np.rint(rng.standard_normal((max(R, 1), d)) * 8) / 8).to(torch.bfloat16).cuda()
    gu_c, gu_s, _ = synthetic_fp4(E * 2 * F, d, fmt, seed=1, E=E)
    dn_c, dn_s, _ = synthetic_fp4(E * d, F, fmt, seed=2, E=E)
    ones = np.ones(E, np.float32) if fmt == "nvfp4" else None    # unit tensor scale: bf16-exact weights
    W_gu = torch.from_numpy(Q.decode_packed(gu_c, gu_s, fmt)).to(torch.bfloat16).reshape(E, 2 * F, d).cuda()
    W_dn = torch.from_numpy(Q.decode_packed(dn_c, dn_s, fmt)).to(torch.bfloat16).reshape(E, d, F).cuda()
    assert torch.equal(W_gu.double().cpu().reshape(-1, d),
                       torch.from_numpy(Q.decode_packed(gu_c, gu_s, fmt))), "decoded weights must be bf16 values"
    offs = torch.from_numpy(offsets).cuda()
    gate = torch.rand(max(R, 1), dtype=torch.float32, device="cuda")
    h4 = M.moe_expert_gate_up_fp4(x, offs, to_device(fmt, gu_c, gu_s, ones), E, F, R)
    h16 = M.moe_expert_gate_up(x, offs, W_gu, R)
    _no_device_error()
    assert torch.equal(h4[:R], h16[:R]), "gate/up: the 4-bit GEMM differs from the bf16 GEMM on the same values"
    for yd in (torch.float32, torch.bfloat16):
        y4 = M.moe_expert_down_fp4(h16, offs, to_device(fmt, dn_c, dn_s, ones), E, d, R, gate, y_dtype=yd)
        y16 = M.moe_expert_down(h16, offs, W_dn, R, gate, y_dtype=yd)
        _no_device_error()
        assert torch.equal(y4[:R], y16[:R]), f"down ({yd}): the 4-bit GEMM differs from the bf16 GEMM"


# ------------------------------------------------------------------ the layer against the oracle
SMALL = [
    I.small_config("fp4_softmax", T=300, d=128, E=16, k=4, F=128),
    I.small_config("fp4_sqrt_softplus_capacity", T=700, d=192, E=24, k=6, F=64, score="sqrt_softplus",
                   capacity_factor=1.0, logit_offset="zipf1.2"),
]


def _oracle_quantize(W, fmt):
    """Oracle quantization of one expert matrix [rows, K] -> packed codes, scale bytes, tensor scale."""
    if fmt == "mxfp4":
        E_, codes = Q.mxfp4_quantize(W)
        return Q.pack_codes(codes), (E_ + 127).astype(np.uint8), None
    s_t, s_b, codes = Q.nvfp4_quantize(W)
    sb = torch.from_numpy(s_b.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return Q.pack_codes(codes), sb, s_t


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_fp4_layer_against_the_oracle(cfg, fmt):
    from routing_dispatch_expert_moe_b200.layer import MoELayer, MoEWeights
    M = _M()
    host, dev = U.make_inputs(cfg)
    packs = {"gu": [], "dn": []}
    for e in range(cfg.E):
        packs["gu"].append(_oracle_quantize(host["W_gu"][e].double().numpy(), fmt))
        packs["dn"].append(_oracle_quantize(host["W_dn"][e].double().numpy(), fmt))

    def stack(name):
        c = np.concatenate([p[0] for p in packs[name]])
        s = np.concatenate([p[1] for p in packs[name]])
        t = np.array([p[2] for p in packs[name]], np.float32) if fmt == "nvfp4" else None
        return c, s, t

    gu, dn = stack("gu"), stack("dn")
    # the weights the experts run on, decoded by the oracle
    Wgu = [Q.decode_packed(p[0], p[1], fmt, p[2] if p[2] is not None else 1.0) for p in packs["gu"]]
    Wdn = [Q.decode_packed(p[0], p[1], fmt, p[2] if p[2] is not None else 1.0) for p in packs["dn"]]
    cap = O.capacity(cfg.T, cfg.E, cfg.k, cfg.capacity_factor, True)
    w = MoEWeights(Wg=dev["Wg"], W_gu=dev["W_gu"], W_dn=dev["W_dn"], logit_offset=dev["off"],
                   W_gu_fp4=to_device(fmt, *gu), W_dn_fp4=to_device(fmt, *dn))
    layer = MoELayer(w, cfg.k, cfg.T, cfg.score, cfg.renormalize, cfg.scale, cap)
    y = layer.forward(dev["x"]).float().cpu().numpy().astype(np.float64)
    _no_device_error()
    o = O.layer_routing(U.cfg_dict(cfg), host["x"], host["Wg"], host["off"], None, True)
    assert np.array_equal(layer.topk_idx.cpu().numpy(), o["topk_idx"])
    assert np.array_equal(layer.row_of.cpu().numpy(), o["row_of"])
    n = int(o["offsets"][-1])
    yp_o = O.grouped_ffn(O.permute(host["x"], o["row_of"], n), o["offsets"], lambda e: Wgu[e], lambda e: Wdn[e],
                         o["gate_of_row"], True)
    yp_g = layer.y_perm[:n].float().cpu().numpy().astype(np.float64)
    experts = np.repeat(np.arange(cfg.E), o["kept"])
    hb = U.row_bounds(host["x"], o["token_of_row"][:n], experts, o["gate_of_row"][:n], lambda e: Wgu[e],
                      lambda e: Wdn[e])
    U.assert_rows_close(yp_g, yp_o, hb, f"y_perm ({fmt})")
    U.assert_y_close(y, O.combine(yp_o, o["row_of"]), f"y ({fmt})")


# ------------------------------------------------------------------ full size, stress workload
@pytest.mark.slow
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_c5_stress_full_size_fp4_experts(fmt):
    """The whole layer at full size with synthetic 4-bit experts; routing in full, and the
    gated rows of a spread of experts (the hottest, the coldest non-empty, capped and mid
    ones) against the oracle on those experts' decoded weights."""
    from routing_dispatch_expert_moe_b200.layer import MoELayer, MoEWeights
    cfg = I.CONFIGS["c5_stress"]
    x = I.gen_x(cfg)
    Wg, off, _ = I.gen_router(cfg)
    E, d, F = cfg.E, cfg.d, cfg.F
    gu = synthetic_fp4(E * 2 * F, d, fmt, seed=5, E=E)
    dn = synthetic_fp4(E * d, F, fmt, seed=6, E=E)
    # W_gu / W_dn stand in for the bf16 weights only through their dtype and F
    w = MoEWeights(Wg=torch.from_numpy(Wg).cuda(), W_gu=torch.empty((1, 2 * F, d), dtype=torch.bfloat16).cuda(),
                   W_dn=torch.empty((1, d, F), dtype=torch.bfloat16).cuda(), logit_offset=torch.from_numpy(off).cuda(),
                   W_gu_fp4=to_device(fmt, *gu), W_dn_fp4=to_device(fmt, *dn))
    cap = O.capacity(cfg.T, E, cfg.k, cfg.capacity_factor, True)
    layer = MoELayer(w, cfg.k, cfg.T, cfg.score, cfg.renormalize, cfg.scale, cap, torch.bfloat16, torch.bfloat16)
    layer.forward(torch.from_numpy(x).to(torch.bfloat16).cuda())
    _no_device_error()
    o = O.layer_routing(U.cfg_dict(cfg), x, Wg, off, None, True)
    assert np.array_equal(layer.topk_idx.cpu().numpy(), o["topk_idx"])
    assert np.array_equal(layer.offsets.cpu().numpy(), o["offsets"])
    kept = o["kept"]
    nz = np.nonzero(kept)[0]
    order = nz[np.argsort(kept[nz], kind="stable")]
    pick = np.unique(np.concatenate([order[:4], order[-4:], order[len(order) // 2 - 4:len(order) // 2 + 4],
                                     np.nonzero(kept == cap)[0][:4]]))

    def weights(c, s, t, R):
        return lambda e: Q.decode_packed(c[e * R:(e + 1) * R], s[e * R:(e + 1) * R], fmt,
                                         1.0 if t is None else float(t[e]))

    gu_of, dn_of = weights(*gu, 2 * F), weights(*dn, d)
    yp_all = layer.y_perm
    for e in pick:
        a, b = int(o["offsets"][e]), int(o["offsets"][e + 1])
        xr = np.asarray(x, np.float64)[o["token_of_row"][a:b]]
        g = o["gate_of_row"][a:b]
        Wgu_e, Wdn_e = gu_of(int(e)), dn_of(int(e))
        want = O.bf16_round(O.swiglu_expert(xr, Wgu_e, Wdn_e, True) * g[:, None])
        got = yp_all[a:b].float().cpu().numpy()
        hb = U.row_bounds(x, o["token_of_row"][a:b], np.full(b - a, e), g, lambda _: Wgu_e, lambda _: Wdn_e)
        U.assert_rows_close(got, want, hb, f"y_perm {fmt} expert {int(e)} ({b - a} rows)", rows_bf16=True)

"""The expert-parallel exchange fused into the dispatch and the combine (moe_ep_dispatch,
moe_ep_combine), with G ranks emulated on one GPU.

Each emulated rank has its own token batch and routing (the library's router and scan
with the per-expert capacity from the host plan), and every owner's expert-major row
buffer is a buffer of this GPU, so the "peer" pointer arrays are ordinary addresses: the
kernels' arithmetic is the multi-GPU one, only no byte crosses NVLink.  No kernel waits on
another (the ranks' barriers are the host's stream order here).

The reference is the one-GPU layer on the concatenated batch (rank 0's tokens first) run
with the same library kernels: the ranks' routing concatenated, scan with the global
capacity, permute, gate/up, down without gates, combine with the gates.  Every owner's buffer must equal the
reference's permuted rows of its experts, and every rank's y the reference's rows of its
tokens, bit for bit (the same rows in the same order through the same kernels, the same
fp32 sums).  The result is also held to the oracle's bars.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_moe_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

CASES = [
    (2, I.small_config("epp_softmax", T=300, d=128, E=16, k=4, F=128)),
    (4, I.small_config("epp_capacity_zipf", T=600, d=256, E=32, k=6, F=64, score="sqrt_softplus",
                       capacity_factor=1.0, logit_offset="zipf1.2")),
    (2, I.small_config("epp_sigmoid_bf16out", T=520, d=128, E=8, k=2, F=128, score="sigmoid", scale=2.0,
                       capacity_factor=1.25)),
]


def _route(M, x, Wg, Wsp, cfg, off):
    return M.moe_route(x, Wg, cfg.k, cfg.score, cfg.renormalize, cfg.scale, off, None, Wg_split=Wsp)


def _counts(M, topk_idx, E):
    return M.moe_histogram_scan(topk_idx, torch.zeros(topk_idx.shape, dtype=torch.float32, device=topk_idx.device), E,
                                -1)["counts"]


@pytest.mark.parametrize("G,cfg", CASES, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_fused_exchange_equals_the_one_gpu_layer_on_the_concatenated_batch(G, cfg):
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.ep import LibraryKernels, ep_plan
    host, dev = U.make_inputs(cfg)
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    assert T % G == 0 and E % G == 0
    Tr, El = T // G, E // G
    cap = O.capacity(T, E, k, cfg.capacity_factor, True)
    out_dt = torch.bfloat16 if cfg.name.endswith("bf16out") else torch.float32
    Wsp = M.moe_prepare_router_weight(dev["Wg"])
    xs = [dev["x"][s * Tr:(s + 1) * Tr].contiguous() for s in range(G)]

    # routing and counts per rank, then every rank's plan
    routes = [_route(M, xs[s], dev["Wg"], Wsp, cfg, dev["off"]) for s in range(G)]
    allc = np.stack([_counts(M, routes[s][1], E).cpu().numpy() for s in range(G)])
    plans = [ep_plan(allc, s, cap) for s in range(G)]

    # owners' buffers and the pointer arrays every rank uses
    cap_rows = max(int(plans[h]["local_offsets"][-1]) for h in range(G)) + 7
    x_loc = [torch.full((cap_rows, d), float("nan"), dtype=dev["x"].dtype, device="cuda") for _ in range(G)]
    y_loc = [torch.full((cap_rows, d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(G)]
    peer_x = torch.tensor([t.data_ptr() for t in x_loc], dtype=torch.int64, device="cuda")
    peer_y = torch.tensor([t.data_ptr() for t in y_loc], dtype=torch.int64, device="cuda")
    peer_cap = torch.full((G,), cap_rows, dtype=torch.int64, device="cuda")

    class _L:                                          # the attributes LibraryKernels reads
        pass
    lay = _L()
    lay.E, lay.k, lay.W_gu, lay.W_dn, lay.rows_dtype, lay.out_dtype = E, k, None, None, torch.float32, out_dt
    kn = LibraryKernels(lay)
    scans, bases = [], []
    for s in range(G):
        sc = kn.scan(routes[s][1], routes[s][2], plans[s]["caps"])
        sc["topk_idx"] = routes[s][1]
        base = torch.from_numpy(M.ep_dst_base(allc, s, cap)).to("cuda")
        M.moe_ep_dispatch(xs[s], sc["topk_idx"], sc["row_of"], sc["offsets"], base, E, G, Tr * k, peer_x, peer_cap)
        scans.append(sc)
        bases.append(base)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    for h in range(G):                                 # each owner's GEMMs over its rows (no gate)
        n = int(plans[h]["local_offsets"][-1])
        if n == 0:
            continue
        offs = torch.from_numpy(plans[h]["local_offsets"]).to("cuda")
        hh = M.moe_expert_gate_up(x_loc[h][:n], offs, dev["W_gu"][h * El:(h + 1) * El].contiguous(), n)
        M.moe_expert_down(hh, offs, dev["W_dn"][h * El:(h + 1) * El].contiguous(), n, None, y_rows=y_loc[h][:n])
    ys = [M.moe_ep_combine(peer_y, torch.float32, peer_cap, scans[s]["topk_idx"], scans[s]["row_of"], routes[s][2],
                           scans[s]["offsets"], bases[s], E, G, d, Tr * k, y_dtype=out_dt) for s in range(G)]
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0

    # reference: the one-GPU library path on the concatenated batch (the ranks' routing
    # concatenated: the router's result for a token does not depend on its batch)
    ti = torch.cat([routes[s][1] for s in range(G)]).contiguous()
    tg = torch.cat([routes[s][2] for s in range(G)]).contiguous()
    ref = M.moe_histogram_scan(ti, tg, E, cap)
    n_all = int(ref["offsets"][-1].item())
    x_perm = M.moe_permute(dev["x"], ref["row_of"], max(n_all, 1))
    h_all = M.moe_expert_gate_up(x_perm, ref["offsets"], dev["W_gu"], max(n_all, 1))
    y_rows = M.moe_expert_down(h_all, ref["offsets"], dev["W_dn"], max(n_all, 1), None, y_dtype=torch.float32)
    y_ref = M.moe_combine(y_rows, ref["row_of"], T, max(n_all, 1), topk_gate=tg, y_dtype=out_dt)
    torch.cuda.synchronize()

    offs_all = ref["offsets"].cpu().numpy()
    for h in range(G):
        a, b = int(offs_all[h * El]), int(offs_all[(h + 1) * El])
        assert b - a == int(plans[h]["local_offsets"][-1])
        assert torch.equal(x_loc[h][:b - a], x_perm[a:b]), f"owner {h}: rows differ from the permuted rows"
        assert torch.equal(y_loc[h][:b - a], y_rows[a:b]), f"owner {h}: result rows differ"
    for s in range(G):
        assert torch.equal(ys[s], y_ref[s * Tr:(s + 1) * Tr]), f"rank {s}: y differs from the one-GPU layer"
    # and the oracle's bars on the whole batch
    o = O.layer_routing(U.cfg_dict(cfg), host["x"], host["Wg"], host["off"], None, True)
    gu, dn = U.expert_getters(host)
    n = int(o["offsets"][-1])
    yp = O.grouped_ffn(O.permute(host["x"], o["row_of"], n), o["offsets"], gu, dn, o["gate_of_row"], True)
    y_all = torch.cat(ys).float().cpu().numpy().astype(np.float64)
    if out_dt == torch.float32:
        U.assert_y_close(y_all, O.combine(yp, o["row_of"]), "y (fused exchange)")


def test_fused_exchange_reports_a_row_past_the_owner_buffer():
    """A plan that points past an owner's capacity is recorded (MOE_DEVERR_ROW), not stored."""
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.ep import ep_plan
    cfg = I.small_config("epp_small", T=64, d=64, E=4, k=2, F=64)
    host, dev = U.make_inputs(cfg)
    Wsp = M.moe_prepare_router_weight(dev["Wg"])
    _, ti, tg = _route(M, dev["x"], dev["Wg"], Wsp, cfg, dev["off"])
    sc = M.moe_histogram_scan(ti, tg, cfg.E, -1)
    allc = sc["counts"].cpu().numpy()[None, :]
    base = torch.from_numpy(M.ep_dst_base(allc, 0, -1)).to("cuda")
    buf = torch.zeros((4, cfg.d), dtype=dev["x"].dtype, device="cuda")      # far too small on purpose
    peer = torch.tensor([buf.data_ptr()], dtype=torch.int64, device="cuda")
    pcap = torch.tensor([buf.shape[0]], dtype=torch.int64, device="cuda")
    M.moe_get_device_error()                                                 # clear
    M.moe_ep_dispatch(dev["x"], ti, sc["row_of"], sc["offsets"], base, cfg.E, 1, cfg.T * cfg.k, peer, pcap)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 3
    assert ep_plan(allc, 0, -1)["local_offsets"][-1] > buf.shape[0]

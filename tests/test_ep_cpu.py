"""The expert-parallel forward on two (and three) gloo ranks on the CPU.

ExpertParallelMoE's orchestration, the library's host plan (moe_ep_plan_host) and the
torch.distributed exchange run as they do between GPUs; the compute steps (router,
scan with per-expert capacity, permute, regroup, expert FFN, combine) are stood in for
by the oracle, so the test needs no GPU.  Each rank holds its own token batch and E/G
experts; the result on every rank must equal the single-process oracle layer run on the
concatenated batch (rank 0's tokens first), capacity drops included.

The plan itself is also checked against a brute-force recount of the global token order.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleKernels:
    """The forward's compute steps from the oracle (float64 numpy on torch CPU tensors)."""

    def __init__(self, L, W_gu_local, W_dn_local):
        self.L, self.gu, self.dn = L, W_gu_local, W_dn_local

    def route(self, x):
        import torch
        L = self.L
        r = O.route(x.numpy(), L.Wg.numpy(), L.k, L.score, L.renormalize, L.scale,
                    None if L.logit_offset is None else L.logit_offset.numpy(), None)
        return (torch.from_numpy(r["logits"]), torch.from_numpy(r["topk_idx"].astype(np.int32)),
                torch.from_numpy(r["topk_gate"]))

    def counts(self, topk_idx):
        import torch
        return torch.from_numpy(np.bincount(topk_idx.numpy().ravel(), minlength=self.L.E).astype(np.int32))

    def scan(self, topk_idx, topk_gate, caps):
        import torch
        idx = topk_idx.numpy().astype(np.int64)
        p = O.dispatch_plan(idx, topk_gate.numpy(), self.L.E, -1)
        kept = np.minimum(p["counts"], caps)
        offsets = np.concatenate([[0], np.cumsum(kept)])
        keep = p["rank"] < caps[idx]
        row_of = np.where(keep, offsets[idx] + p["rank"], -1)
        return {"row_of": torch.from_numpy(row_of.astype(np.int32)), "offsets": torch.from_numpy(offsets)}

    def permute(self, x, row_of, rows):
        import torch
        r = row_of.numpy()
        n = int(r.max()) + 1 if (r >= 0).any() else 0
        return torch.from_numpy(O.permute(x.numpy(), r, n))

    def regroup(self, src, table, inverse, rows_out):
        import torch
        s = src.numpy()
        out = np.zeros((rows_out, s.shape[1]), np.float64)
        for a, b, n in table:
            if inverse:
                out[a:a + n] = s[b:b + n]
            else:
                out[b:b + n] = s[a:a + n]
        return torch.from_numpy(out)

    def ffn(self, x_local, offsets_local, rows):
        import torch
        y = O.grouped_ffn(x_local.numpy(), offsets_local, lambda e: self.gu[e], lambda e: self.dn[e], None, False)
        return torch.from_numpy(y)

    def combine(self, y_rows, row_of, topk_gate, T):
        import torch
        return torch.from_numpy(O.combine(y_rows.numpy(), row_of.numpy(), topk_gate=topk_gate.numpy()))


def _case(G):
    from routing_dispatch_expert_moe_b200 import inputs as I
    cfg = I.small_config("ep", T=96, d=64, E=12 if G == 3 else 8, k=2, F=32, score="softmax", act="f32",
                         capacity_factor=1.0, logit_offset="zipf1.2")
    xs = [I.gen_x(cfg, seed=10 + r) for r in range(G)]
    Wg, off, _ = I.gen_router(cfg)
    W_gu, W_dn = I.gen_experts(cfg)
    cap = O.capacity(cfg.T * G, cfg.E, cfg.k, cfg.capacity_factor, True)
    return cfg, xs, Wg, off, W_gu, W_dn, cap


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from routing_dispatch_expert_moe_b200.ep import ExpertParallelMoE
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg, xs, Wg, off, W_gu, W_dn, cap = _case(world)
        El = cfg.E // world
        sl = slice(rank * El, (rank + 1) * El)
        lay = ExpertParallelMoE(torch.from_numpy(Wg), torch.from_numpy(W_gu[sl]), torch.from_numpy(W_dn[sl]), cfg.k,
                                cfg.score, cfg.renormalize, cfg.scale, cap, torch.from_numpy(off))
        lay.kernels = OracleKernels(lay, W_gu[sl].astype(np.float64), W_dn[sl].astype(np.float64))
        y = lay.forward(torch.from_numpy(xs[rank].astype(np.float64)))
        q.put((rank, y.numpy(), {k_: v.tolist() for k_, v in lay.last_plan.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_forward_equals_the_single_rank_layer(world):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (y, plan)) for r, y, plan in (q.get(timeout=240) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, xs, Wg, off, W_gu, W_dn, cap = _case(world)
    x_all = np.concatenate(xs)
    c = dict(T=x_all.shape[0], E=cfg.E, k=cfg.k, score=cfg.score, renormalize=cfg.renormalize, scale=cfg.scale,
             capacity_factor=cfg.capacity_factor)
    o = O.layer_forward(c, x_all, Wg, lambda e: W_gu[e].astype(np.float64), lambda e: W_dn[e].astype(np.float64),
                        logit_offset=off, bf16=False)
    assert o["capacity"] == cap and (o["row_of"] < 0).any(), "the case must drop assignments across ranks"
    for r in range(world):
        y, plan = res[r]
        np.testing.assert_allclose(y, o["y"][r * cfg.T:(r + 1) * cfg.T], rtol=1e-12, atol=1e-12)
    # what each rank sent is what the others received
    for r in range(world):
        for h in range(world):
            assert res[r][1]["send_rows"][h] == res[h][1]["recv_rows"][r]


def test_plan_matches_a_brute_force_recount():
    sys.path.insert(0, ROOT)
    from routing_dispatch_expert_moe_b200.ep import ep_plan
    rng = np.random.default_rng(4)
    for G, E, cap in ((2, 8, 5), (4, 16, 3), (3, 9, -1), (1, 4, 2), (4, 8, 0)):
        counts = rng.integers(0, 9, size=(G, E)).astype(np.int32)
        El = E // G
        # brute force: walk the global token order assignment by assignment
        kept = np.zeros((G, E), np.int64)
        taken = np.zeros(E, np.int64)
        for s in range(G):
            for e in range(E):
                for _ in range(counts[s, e]):
                    if cap < 0 or taken[e] < cap:
                        kept[s, e] += 1
                    taken[e] += 1
        for g in range(G):
            p = ep_plan(counts, g, cap)
            assert np.array_equal(p["caps"], kept[g])
            assert [int(v) for v in p["send_rows"]] == [int(kept[g, h * El:(h + 1) * El].sum()) for h in range(G)]
            assert [int(v) for v in p["recv_rows"]] == [int(kept[s, g * El:(g + 1) * El].sum()) for s in range(G)]
            mine = kept[:, g * El:(g + 1) * El]
            assert list(p["local_offsets"]) == [0] + list(np.cumsum(mine.sum(axis=0)))
            # the regroup table is a bijection from the receive buffer onto the expert-major rows
            tgt = np.full(int(mine.sum()), -1)
            for a, b, n in p["regroup"]:
                assert (tgt[b:b + n] == -1).all()
                tgt[b:b + n] = np.arange(a, a + n)
            assert sorted(tgt.tolist()) == list(range(int(mine.sum())))


def test_plan_host_validation():
    sys.path.insert(0, ROOT)
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.ep import ep_plan
    with pytest.raises(M.MoEError):
        ep_plan(np.zeros((2, 7), np.int32), 0, -1)                  # E % G != 0
    with pytest.raises(M.MoEError):
        ep_plan(-np.ones((2, 8), np.int32), 0, -1)                  # negative counts
    with pytest.raises(M.MoEError):
        ep_plan(np.zeros((2, 8), np.int32), 2, -1)                  # rank out of range


def test_dst_base_puts_each_rank_where_the_owner_expects_it():
    """moe_ep_dst_base_host: rank g's q-th kept row of expert e lands at dst_base[e] + q in
    the owner's expert-major rows, the row the owner's regroup table gives it."""
    sys.path.insert(0, ROOT)
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.ep import ep_plan
    rng = np.random.default_rng(9)
    for G, E, cap in ((2, 8, 5), (4, 16, 3), (3, 9, -1), (1, 4, 2), (4, 8, 0)):
        counts = rng.integers(0, 9, size=(G, E)).astype(np.int32)
        El = E // G
        plans = [ep_plan(counts, h, cap) for h in range(G)]
        for g in range(G):
            base = M.ep_dst_base(counts, g, cap)
            kept_g = plans[g]["caps"]
            for e in range(E):
                h, j = e // El, e % El
                a, b, n = (int(v) for v in plans[h]["regroup"][g * El + j])
                assert n == kept_g[e]
                assert base[e] == b, (G, E, cap, g, e)
                assert 0 <= base[e] and base[e] + n <= plans[h]["local_offsets"][-1]


def test_dst_base_host_validation():
    sys.path.insert(0, ROOT)
    from routing_dispatch_expert_moe_b200 import moe as M
    with pytest.raises(M.MoEError):
        M.ep_dst_base(np.zeros((2, 7), np.int32), 0, -1)             # E % G != 0
    with pytest.raises(M.MoEError):
        M.ep_dst_base(-np.ones((2, 8), np.int32), 0, -1)             # negative counts
    with pytest.raises(M.MoEError):
        M.ep_dst_base(np.zeros((2, 8), np.int32), 2, -1)             # rank out of range

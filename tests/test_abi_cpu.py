"""C-ABI checks that need no GPU: the library builds and loads, exports every entry point
include/moe.h declares, and its host-side logic (capacity, sizes, validation) behaves.

Every validation case below is rejected on the host before any launch, so none of
them touches device memory even on a machine that has a GPU.
"""
import ctypes
import os
import re

import pytest

from tests._closed_form import load

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from routing_dispatch_expert_moe_b200 import build
    build.build()
    from routing_dispatch_expert_moe_b200 import moe
    return moe.lib()


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^MOE_API [^(]*?\b(moe_\w+)\(", txt, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) >= 17
    for n in names:
        assert hasattr(L, n), n
    from routing_dispatch_expert_moe_b200 import moe
    assert sorted(moe.exported_symbols()) == names      # binding covers the whole header


def test_status_strings(L):
    assert L.moe_status_str(0) == b"MOE_OK"
    assert L.moe_status_str(3) == b"MOE_ERR_WORKSPACE"
    assert L.moe_version() >= 10000


def test_capacity_matches_closed_forms(L, golden_dir):
    g = load(golden_dir, "capacity.json")
    for c in g["cases"]:
        assert L.moe_capacity(c["T"], c["E"], c["k"], c["cf"], 1) == c["per_assignment"], c
        assert L.moe_capacity(c["T"], c["E"], c["k"], c["cf"], 0) == c["literal"], c
    assert L.moe_capacity(10, 4, 2, 0.0, 1) == -1
    assert L.moe_capacity(10, 0, 2, 1.0, 1) == -2


def test_rows_max(L):
    assert L.moe_rows_max(100, 8, 2, -1) == 200
    assert L.moe_rows_max(100, 8, 2, 10) == 80
    assert L.moe_rows_max(100, 8, 2, 1000) == 200
    assert L.moe_rows_max(0, 8, 2, -1) == 0


def test_gate_up_orientation_query(L, monkeypatch):
    """Weight-major tiles below 1024 rows per expert on average; the override variable wins."""
    monkeypatch.delenv("MOE_B200_EXPERT_TILES", raising=False)
    assert L.moe_gate_up_weight_major(32768 * 16, 896) == 1          # stress layer: 585 rows per expert
    assert L.moe_gate_up_weight_major(8192 * 8, 64) == 0             # handbook layer: 1024 rows per expert
    assert L.moe_gate_up_weight_major(1023, 1) == 1
    assert L.moe_gate_up_weight_major(1024, 1) == 0
    assert L.moe_gate_up_weight_major(-1, 8) == -1 and L.moe_gate_up_weight_major(10, 0) == -1
    monkeypatch.setenv("MOE_B200_EXPERT_TILES", "tokens")
    assert L.moe_gate_up_weight_major(32768 * 16, 896) == 0
    monkeypatch.setenv("MOE_B200_EXPERT_TILES", "weights")
    assert L.moe_gate_up_weight_major(8192 * 8, 64) == 1


def test_workspace_queries(L):
    assert L.moe_histogram_scan_workspace_bytes(8192, 8, 64) >= 8192 * 8 * 4
    assert L.moe_router_stats_workspace_bytes(8192, 64) > 0
    w = L.moe_workspace_bytes(8192, 2048, 64, 8)
    assert w >= L.moe_histogram_scan_workspace_bytes(8192, 8, 64)
    assert L.moe_histogram_scan_workspace_bytes(0, 8, 64) == 0


FAKE = ctypes.c_void_p(4096)   # non-null, aligned; never dereferenced (host checks fail first)
NUL = None


def _route(L, **kw):
    a = dict(x=FAKE, dt=0, Wg=FAKE, W3=NUL, off=NUL, bias=NUL, T=64, d=128, E=16, k=4, score=0, renorm=1, scale=1.0,
             logits=FAKE, idx=FAKE, gate=FAKE, ws=FAKE, wsb=1 << 30, s=NUL)
    a.update(kw)
    return L.moe_route(a["x"], a["dt"], a["Wg"], a["W3"], a["off"], a["bias"], a["T"], a["d"], a["E"], a["k"],
                       a["score"], a["renorm"], a["scale"], a["logits"], a["idx"], a["gate"], a["ws"], a["wsb"],
                       a["s"])


@pytest.mark.parametrize("d,E", [(2048, 64), (4096, 63), (7168, 896), (1024, 36), (64, 8), (512, 1024)])
def test_workspace_queries_cover_every_smaller_batch(L, d, E):
    """A smaller batch may split the SIMT router's GEMM more ways, so a query for T must
    cover every T' <= T: one layer workspace serves them all."""
    ts = sorted(set(list(range(1, 1200, 37)) + list(range(1024, 20000, 389)) + [256, 2368, 4608, 4864, 5000, 8192]))
    prev_r = prev_w = 0
    for T in ts:
        r = L.moe_route_workspace_bytes(T, d, E)
        w = L.moe_workspace_bytes(T, d, E, 8)
        assert r >= prev_r and w >= prev_w, (T, r, prev_r)
        assert w >= r
        prev_r, prev_w = r, w


@pytest.mark.parametrize("kw,status", [
    (dict(x=NUL), 1), (dict(Wg=NUL), 1), (dict(logits=NUL), 1), (dict(k=17), 1), (dict(k=0), 1),
    (dict(E=0), 1), (dict(T=-1), 1), (dict(score=3), 1), (dict(dt=7), 1), (dict(renorm=2), 1),
    (dict(scale=float("nan")), 1), (dict(E=1025, k=4), 2), (dict(k=33, E=64), 2), (dict(d=100), 2),
    (dict(x=ctypes.c_void_p(4104)), 2), (dict(W3=ctypes.c_void_p(4104)), 2),
])
def test_route_host_validation(L, kw, status):
    assert _route(L, **kw) == status


def test_route_workspace_check(L):
    need = L.moe_route_workspace_bytes(64, 4096, 16)
    if need:
        assert _route(L, d=4096, wsb=need - 1) == 3
        assert _route(L, d=4096, ws=NUL) == 3
    # the tensor-core path (T >= 256) splits W_g into the workspace unless given the split
    need = L.moe_route_workspace_bytes(512, 2048, 64)
    assert need >= L.moe_router_weight_bytes(2048, 64) > 0
    assert _route(L, T=512, d=2048, E=64, wsb=need - 1) == 3


def test_router_weight_size_and_prepare_validation(L):
    # experts in ceil(E / 256) tiles of NE = 32 * ceil(ceil(E / tiles) / 32), three bf16 terms each
    for d, E, NE, tiles in ((2048, 64, 64, 1), (4096, 256, 256, 1), (7168, 896, 224, 4), (512, 1024, 256, 4),
                            (64, 8, 32, 1), (128, 260, 160, 2), (4096, 520, 192, 3)):
        assert L.moe_router_weight_bytes(d, E) == tiles * 3 * NE * d * 2, (d, E)
    assert L.moe_router_weight_bytes(56, 64) == 0          # d < 64: SIMT router, no split
    assert L.moe_router_weight_bytes(2048, 66) == 0        # E % 4
    assert L.moe_router_weight_bytes(2048, 2048) == 0      # E > 1024
    f = L.moe_prepare_router_weight                        # (Wg, d, E, out, bytes, stream)
    nb = L.moe_router_weight_bytes(2048, 64)
    assert f(NUL, 2048, 64, FAKE, nb, NUL) == 1
    assert f(FAKE, 2048, 64, NUL, nb, NUL) == 1
    assert f(FAKE, 0, 64, FAKE, nb, NUL) == 1
    assert f(FAKE, 2048, 64, FAKE, nb - 1, NUL) == 3
    assert f(FAKE, 2048, 66, FAKE, nb, NUL) == 2
    assert f(FAKE, 2048, 64, ctypes.c_void_p(4104), nb, NUL) == 2


def test_route_empty_batch_is_ok_without_launch(L):
    assert _route(L, T=0, x=NUL, logits=NUL, idx=NUL, gate=NUL) == 0


def test_router_logits_host_validation(L):
    def f(*a):                         # (x, dt, Wg, off, T, d, E, logits, ws, wsb, s), Wg_split NULL
        return L.moe_router_logits(a[0], a[1], a[2], NUL, *a[3:])
    assert f(NUL, 0, FAKE, NUL, 64, 128, 16, FAKE, FAKE, 1 << 30, NUL) == 1          # x
    assert f(FAKE, 0, FAKE, NUL, 64, 128, 16, NUL, FAKE, 1 << 30, NUL) == 1          # logits
    assert f(FAKE, 5, FAKE, NUL, 64, 128, 16, FAKE, FAKE, 1 << 30, NUL) == 1         # dtype
    assert f(FAKE, 0, FAKE, NUL, -1, 128, 16, FAKE, FAKE, 1 << 30, NUL) == 1         # T < 0
    assert f(FAKE, 0, FAKE, NUL, 64, 128, 2048, FAKE, FAKE, 1 << 30, NUL) == 2       # E > 1024
    assert f(FAKE, 0, FAKE, NUL, 64, 100, 16, FAKE, FAKE, 1 << 30, NUL) == 2         # d % 8
    assert f(ctypes.c_void_p(4104), 0, FAKE, NUL, 64, 128, 16, FAKE, FAKE, 1 << 30, NUL) == 2
    assert L.moe_router_logits_workspace_bytes(64, 128, 16) == 0                    # under 256 tokens: SIMT
    need = L.moe_router_logits_workspace_bytes(512, 128, 16)
    assert need == L.moe_router_weight_bytes(128, 16) > 0                           # the split, made by the call
    assert f(FAKE, 0, FAKE, NUL, 512, 128, 16, FAKE, FAKE, need - 1, NUL) == 3
    assert L.moe_router_logits_workspace_bytes(512, 128, 18) == 0                   # E % 4: SIMT, no workspace
    assert f(NUL, 0, NUL, NUL, 0, 128, 16, NUL, NUL, 0, NUL) == 0                    # T = 0: nothing to do


def test_route_fixed_host_validation(L):
    f = L.moe_route_fixed              # (logits, T, E, k, score, renorm, scale, rule, token_id, seed, idx, gate, s)
    ok = dict(l=FAKE, T=64, E=16, k=4, sc=0, rn=1, scale=1.0, rule=0, tid=NUL, seed=0, idx=FAKE, g=FAKE)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["l"], a["T"], a["E"], a["k"], a["sc"], a["rn"], a["scale"], a["rule"], a["tid"], a["seed"],
                 a["idx"], a["g"], NUL)

    assert call(rule=2) == 1
    assert call(rule=1) == 1                   # hash without token ids
    assert call(k=17) == 1                     # k > E
    assert call(sc=3) == 1
    assert call(rn=2) == 1
    assert call(scale=float("inf")) == 1
    assert call(l=NUL) == 1
    assert call(E=2000, k=4) == 2
    assert call(k=33, E=64) == 2
    assert call(T=0, l=NUL, idx=NUL, g=NUL) == 0


def test_route_noisy_host_validation(L):
    f = L.moe_route_noisy              # (logits, logits_noise, noise, T, E, k, scale, H, idx, gate, s)
    assert f(FAKE, FAKE, NUL, 64, 16, 4, 1.0, FAKE, FAKE, FAKE, NUL) == 1             # noise
    assert f(FAKE, FAKE, FAKE, 64, 16, 4, 1.0, NUL, FAKE, FAKE, NUL) == 1             # H
    assert f(FAKE, FAKE, FAKE, 64, 16, 17, 1.0, FAKE, FAKE, FAKE, NUL) == 1           # k > E
    assert f(FAKE, FAKE, FAKE, 64, 16, 4, float("nan"), FAKE, FAKE, FAKE, NUL) == 1
    assert f(FAKE, FAKE, FAKE, 64, 2048, 4, 1.0, FAKE, FAKE, FAKE, NUL) == 2
    assert f(NUL, NUL, NUL, 0, 16, 4, 1.0, NUL, NUL, NUL, NUL) == 0


def test_histogram_scan_host_validation(L):
    f = L.moe_histogram_scan
    ok = dict(idx=FAKE, g=FAKE, T=64, k=4, E=16, cap=-1, c=FAKE, kp=FAKE, o=FAKE, r=FAKE, t=FAKE, gr=FAKE,
              ws=FAKE, wsb=1 << 30)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["idx"], a["g"], a["T"], a["k"], a["E"], a["cap"], a["c"], a["kp"], a["o"], a["r"], a["t"],
                 a["gr"], a["ws"], a["wsb"], NUL)

    assert call(cap=-2) == 1
    assert call(c=NUL) == 1
    assert call(idx=NUL) == 1
    assert call(wsb=16) == 3
    assert call(ws=NUL) == 3
    assert call(k=20) == 1
    assert call(E=2000, k=4) == 2


def test_ffn_host_validation(L):
    f = L.moe_expert_gate_up
    assert f(FAKE, 0, FAKE, 4, 100, 64, 128, FAKE, FAKE, NUL) == 2        # d % 8
    assert f(FAKE, 0, FAKE, 4, 128, 60, 128, FAKE, FAKE, NUL) == 2        # F % 8
    assert f(FAKE, 0, NUL, 4, 128, 64, 128, FAKE, FAKE, NUL) == 1         # offsets
    assert f(FAKE, 0, FAKE, 0, 128, 64, 128, FAKE, FAKE, NUL) == 1        # E
    assert f(FAKE, 9, FAKE, 4, 128, 64, 128, FAKE, FAKE, NUL) == 1        # dtype
    assert f(ctypes.c_void_p(4100), 0, FAKE, 4, 128, 64, 128, FAKE, FAKE, NUL) == 2   # alignment
    assert f(FAKE, 0, FAKE, 4, 128, 64, 0, FAKE, FAKE, NUL) == 0          # no rows: nothing to do
    g = L.moe_expert_down
    assert g(FAKE, 0, FAKE, 4, 128, 64, -1, FAKE, NUL, 1, FAKE, NUL) == 1
    assert g(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, 7, FAKE, NUL) == 1        # y dtype
    q = L.moe_expert_gate_up_gather    # (x, dt, T, tok, offs, E, d, F, rows_max, W_gu, h, s)
    assert q(FAKE, 0, -1, FAKE, FAKE, 4, 128, 64, 128, FAKE, FAKE, NUL) == 1       # T < 0
    assert q(FAKE, 0, 64, NUL, FAKE, 4, 128, 64, 128, FAKE, FAKE, NUL) == 1        # token_of_row
    assert q(FAKE, 0, 64, FAKE, FAKE, 4, 100, 64, 128, FAKE, FAKE, NUL) == 2       # d % 8
    assert q(ctypes.c_void_p(4098), 0, 64, FAKE, FAKE, 4, 128, 64, 128, FAKE, FAKE, NUL) == 2   # alignment
    assert q(FAKE, 0, 0, FAKE, FAKE, 4, 128, 64, 128, FAKE, FAKE, NUL) == 0        # no tokens
    h = L.moe_expert_down_combine      # (h, dt, offs, E, d, F, rows_max, W_dn, gate, tok, T, accumulate, y, s)
    assert h(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, FAKE, 64, 2, FAKE, NUL) == 1      # accumulate flag
    assert h(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, FAKE, -1, 0, FAKE, NUL) == 1      # T < 0
    assert h(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, NUL, 64, 0, FAKE, NUL) == 1       # token_of_row
    assert h(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, FAKE, 64, 0, NUL, NUL) == 1       # y
    assert h(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, FAKE, 64, 0, ctypes.c_void_p(4104), NUL) == 2
    assert h(FAKE, 0, FAKE, 4, 100, 64, 128, FAKE, NUL, FAKE, 64, 0, FAKE, NUL) == 2      # d % 8
    assert h(FAKE, 0, FAKE, 4, 128, 64, 128, FAKE, NUL, FAKE, 0, 0, FAKE, NUL) == 0       # no tokens


def test_permute_combine_host_validation(L):
    assert L.moe_permute(FAKE, 0, 64, 100, 4, FAKE, 256, FAKE, NUL) == 2
    assert L.moe_permute(NUL, 0, 64, 128, 4, FAKE, 256, FAKE, NUL) == 1
    assert L.moe_permute(FAKE, 0, 64, 128, 40, FAKE, 256, FAKE, NUL) == 2
    assert L.moe_permute(FAKE, 0, 0, 128, 4, FAKE, 0, FAKE, NUL) == 0
    assert L.moe_combine(FAKE, 0, NUL, NUL, NUL, 64, 128, 4, 256, 1, FAKE, NUL) == 1
    assert L.moe_combine(FAKE, 0, FAKE, NUL, ctypes.c_void_p(4097), 64, 128, 4, 256, 1, FAKE, NUL) == 2
    assert L.moe_combine(FAKE, 0, FAKE, NUL, NUL, 64, 128, 4, 256, 5, FAKE, NUL) == 1     # y dtype


def test_round_output_host_validation(L):
    assert L.moe_round_output(NUL, 64, FAKE, 0, NUL) == 1
    assert L.moe_round_output(FAKE, -1, FAKE, 0, NUL) == 1
    assert L.moe_round_output(FAKE, 64, FAKE, 2, NUL) == 1
    assert L.moe_round_output(FAKE, 64, ctypes.c_void_p(4098), 0, NUL) == 2
    assert L.moe_round_output(NUL, 0, NUL, 1, NUL) == 0


def test_zero_host_validation(L):
    assert L.moe_zero(NUL, 64, NUL) == 1
    assert L.moe_zero(ctypes.c_void_p(4100), 64, NUL) == 2
    assert L.moe_zero(NUL, 0, NUL) == 0


def test_router_stats_host_validation(L):
    f = L.moe_router_stats
    assert f(FAKE, FAKE, FAKE, 64, 16, 4, 5, FAKE, FAKE, FAKE, 1 << 30, NUL) == 1
    assert f(FAKE, FAKE, FAKE, 64, 16, 4, 0, FAKE, FAKE, FAKE, 8, NUL) == 3
    assert f(FAKE, NUL, FAKE, 64, 16, 4, 0, FAKE, FAKE, FAKE, 1 << 30, NUL) == 1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    import routing_dispatch_expert_moe_b200.moe as m
    monkeypatch.setattr(m, "_lib", None)
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        m.lib()
    importlib.reload(m)


def test_capacity_and_rows_max_agree_with_the_oracle_on_random_sizes(L):
    """The library's host arithmetic against the oracle: the capacity formula in both
    readings, and the rows bound holding every plan the oracle builds."""
    import numpy as np
    from oracle import moe_oracle as O
    rng = np.random.default_rng(11)
    for _ in range(400):
        T = int(rng.integers(0, 40000))
        E = int(rng.integers(1, 1025))
        k = int(rng.integers(1, min(E, 32) + 1))
        cf = float(rng.choice([0.0, -1.0, rng.uniform(0.01, 4.0), 1.0, 1.25]))
        for per in (True, False):
            want = O.capacity(T, E, k, cf if cf > 0 else None, per)
            assert L.moe_capacity(T, E, k, cf, 1 if per else 0) == want, (T, E, k, cf, per)
    for _ in range(60):
        T, E = int(rng.integers(1, 300)), int(rng.integers(1, 40))
        k = int(rng.integers(1, min(E, 8) + 1))
        cap = int(rng.choice([-1, 0, 1, int(rng.integers(1, 60))]))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        plan = O.dispatch_plan(idx, np.ones((T, k)), E, cap)
        assert int(plan["offsets"][-1]) <= L.moe_rows_max(T, E, k, cap)
        assert L.moe_rows_max(T, E, k, cap) == (T * k if cap < 0 else min(T * k, E * cap))


def test_scan_wait_check_host_validation(L):
    f = L.moe_scan_wait_check          # (idx, gate, T, k, E, cap, counts, kept, offs, row_of, tor, gor, ns, ws, wsb, s)

    def call(T=1000, ns=10 ** 6, ws=FAKE, wsb=1 << 30, ptr=FAKE):
        return f(ptr, FAKE, T, 4, 64, -1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ns, ws, wsb, NUL)
    assert call(T=256) == 1                      # no chunk after the withheld first one
    assert call(ns=999) == 1 and call(ns=2 * 10 ** 9) == 1
    assert call(ptr=NUL) == 1
    assert call(ws=NUL) == 3 and call(wsb=16) == 3


def test_fp4_gemm_host_validation(L):
    gu = L.moe_expert_gate_up_fp4      # (x, offs, E, d, F, rows, codes, scales, fmt, ts, h, s)
    dn = L.moe_expert_down_fp4         # (h, offs, E, d, F, rows, codes, scales, fmt, ts, gate, ydt, y, s)

    def g(**kw):
        a = dict(x=FAKE, offs=FAKE, E=8, d=128, F=64, rows=100, codes=FAKE, scales=FAKE, fmt=0, ts=NUL, out=FAKE)
        a.update(kw)
        return gu(a["x"], a["offs"], a["E"], a["d"], a["F"], a["rows"], a["codes"], a["scales"], a["fmt"], a["ts"],
                  a["out"], NUL)
    assert g(fmt=2) == 1 and g(codes=NUL) == 1 and g(offs=NUL) == 1 and g(x=NUL) == 1
    assert g(fmt=1) == 1                                   # NVFP4 needs the tensor scales
    assert g(d=96) == 2 and g(F=32) == 2 and g(E=2000) == 2
    assert g(codes=ctypes.c_void_p(4104)) == 2 and g(scales=ctypes.c_void_p(4100)) == 2
    assert g(rows=0, x=NUL, out=NUL) == 0                  # nothing to do
    assert dn(FAKE, FAKE, 8, 128, 64, 100, FAKE, FAKE, 0, NUL, NUL, 7, FAKE, NUL) == 1   # output dtype
    assert dn(FAKE, FAKE, 8, 128, 64, 100, FAKE, FAKE, 1, NUL, NUL, 0, FAKE, NUL) == 1   # NVFP4 without scales


def test_fp4_scale_preparation_size_and_validation(L):
    # k-block-major with 256 zero rows per k-block: (K/64) * (rows + 256) * (64 / block) bytes
    assert L.moe_fp4_scales_bytes(512, 7168, 0) == (7168 // 64) * (512 + 256) * 2
    assert L.moe_fp4_scales_bytes(512, 256, 1) == (256 // 64) * (512 + 256) * 4
    assert L.moe_fp4_scales_bytes(512, 96, 0) == 0 and L.moe_fp4_scales_bytes(512, 128, 5) == 0
    f = L.moe_prepare_fp4_scales       # (scales, rows, K, fmt, out, bytes, stream)
    nb = L.moe_fp4_scales_bytes(512, 128, 0)
    assert f(FAKE, 512, 128, 0, NUL, nb, NUL) == 1
    assert f(NUL, 512, 128, 0, FAKE, nb, NUL) == 1
    assert f(FAKE, 512, 128, 7, FAKE, nb, NUL) == 1
    assert f(FAKE, 512, 96, 0, FAKE, nb, NUL) == 2
    assert f(FAKE, 512, 128, 0, FAKE, nb - 1, NUL) == 3
    assert f(FAKE, 512, 128, 0, ctypes.c_void_p(4100), nb, NUL) == 2


def test_fused_exchange_host_validation(L):
    """moe_ep_dispatch / moe_ep_combine / moe_ipc_*: every check before any launch or CUDA call."""
    import ctypes
    v = ctypes.c_void_p(16)                                           # never dereferenced: rejected first
    d = L.moe_ep_dispatch
    assert d(v, 0, 0, 64, 2, v, v, v, v, 8, 2, 0, v, v, None) == 0                 # T = 0: nothing to do
    assert d(None, 0, 4, 64, 2, v, v, v, v, 8, 2, 8, v, v, None) == 1              # null x
    assert d(v, 0, 4, 64, 2, v, v, v, v, 8, 3, 8, v, v, None) == 1                 # E % G != 0
    assert d(v, 2, 4, 64, 2, v, v, v, v, 8, 2, 8, v, v, None) == 1                 # bad dtype
    assert d(v, 0, 4, 12, 2, v, v, v, v, 8, 2, 8, v, v, None) == 2                 # 24-byte rows
    assert d(v, 0, 4, 64, 2, v, v, v, v, 8, 2, 8, None, v, None) == 1              # no owner pointers
    c = L.moe_ep_combine
    assert c(v, 1, v, 2, v, v, v, v, v, 8, 0, 64, 2, 0, 1, v, None) == 0          # T = 0
    assert c(None, 1, v, 2, v, v, v, v, v, 8, 4, 64, 2, 8, 1, v, None) == 1       # null owner pointers
    assert c(v, 1, v, 2, v, v, None, v, v, 8, 4, 64, 2, 8, 1, v, None) == 1       # no gates
    assert c(v, 1, v, 2, v, v, v, v, v, 8, 4, 60, 2, 8, 1, v, None) == 2          # d % 8
    assert L.moe_ipc_handle_bytes() == 64
    off = ctypes.c_int64(0)
    assert L.moe_ipc_get_handle(None, ctypes.create_string_buffer(64), ctypes.byref(off)) == 1
    p, b = ctypes.c_void_p(), ctypes.c_void_p()
    assert L.moe_ipc_open_handle(None, 0, ctypes.byref(p), ctypes.byref(b)) == 1
    assert L.moe_ipc_close(None) == 1

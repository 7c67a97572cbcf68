"""Benchmark of the MoE-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole layer (router, top-k, histogram/scan, permute, grouped
gate/up GEMM + SwiGLU, grouped down GEMM x gate, combine, router statistics) over one
batch of synthetic tokens.  The default workload is the largest one, the very-many-
experts stress layer (T=32768, d=7168, E=896, k=16, F=256, sqrt(softplus) scores, Zipf
skew, capacity factor 1.0 with token-order dropping; bf16 with an fp32 router);
--workload picks another.  Inputs are resident in HBM; L2 is flushed (256 MB write)
before every step and each step is timed with CUDA events on the launching stream.
With N > 1 (torchrun) every rank runs an independent replica on its own token batch
(the layer has no data-path collective); the timing is the max over ranks.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead, on a
bounded token sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s on 1 B200; grouped-GEMM TFLOP/s; route/permute GB/s"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (read + write bytes) of the dominant kernel, the gate/up GEMM, per launch, keyed
# by (workload, dispatch, kept rows), from ncu captures of the same kernel build
# (profiles/gate_up_traffic.md); absent when the kernel changed since the capture.  The
# stress workload's entry is the reduced shape's measured traffic / algorithmic ratio
# (1.019) times the full launch's algorithmic bytes (the capture holds a quarter of the
# tokens and experts; both the weight and the row bytes grow with the units).
GATE_UP_TRAFFIC = {
    ("c2_handbook", "permute", 65536): 932886016,
    ("c5_stress", "permute", 131356): 8784605026,
}


def peaks(path=None):
    """The roofline denominators: MEASURED_PEAKS.json's figures where it has them (a number,
    or an object with a numeric "value"), the fallback figures for any it lacks.  Returns
    the figures and, per figure, "measured" or "fallback"."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    d = None
    if os.path.exists(p):
        try:
            with open(p) as f:
                d = json.load(f)
        except (OSError, ValueError):
            d = None
    out, src = {}, {}
    for key, fb in FALLBACK_PEAKS.items():
        v = d.get(key) if isinstance(d, dict) else None
        if isinstance(v, dict):
            v = v.get("value")
        ok = isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0
        out[key] = float(v) if ok else fb
        src[key] = "measured" if ok else "fallback"
    return out, src


def max_over_ranks(v: float, device=None) -> float:
    """Max of v over every rank of the process group (v itself without one).  All ranks
    must call it at the same point: it is a collective."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time (weak scaling:
    each replica processes its own batch of tokens_per_rank per step)."""
    return tokens_per_rank * world * steps / (total_ms / 1e3)


def workload_config(name: str, cfg, cap: int) -> dict:
    """The workload identity both arms report (the same keys and values in each line)."""
    return {"workload": name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "F": cfg.F, "F_shared": cfg.F_s,
            "score": cfg.score, "capacity": cap}


def replica_seed(rank: int) -> int:
    """Seed of a replica's token batch: every rank gets its own batch, same weights."""
    return rank


def env_rank():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.idx), "-lms", "100"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def layer_roofline_ms(cfg, A, pk, rb=4, ob=4, fused=False, gather=False, E_act=None):
    """Sum over steps of max(compute, memory) time at the measured peaks (algorithmic bytes / flops).
    A: kept assignment rows; E_act: experts with at least one kept row (only their weights are
    read).  rb / ob: bytes per element of the gated rows / of the layer output.  fused: the
    combine runs inside the down GEMM, whose algorithmic bytes are then H, W_dn and y (zero
    fill + result).  gather: the permute runs inside the gate/up GEMM, whose algorithmic bytes
    are then x, W_gu, H.  The router is priced at its algorithmic 2 T d E flops on the bf16
    tensor cores (however many terms an implementation issues) or its bytes, whichever is
    slower, so the sum is a lower bound for any implementation."""
    T, d, E, k, F = cfg.T, cfg.d, cfg.E, cfg.k, cfg.F
    Ea = E if E_act is None else E_act
    hbm = pk["hbm_gbs"] * 1e9
    tc = pk["bf16_tflops"] * 1e12
    b = 2
    steps = {
        "route": max(2 * T * d * E / tc, (T * d * b + d * E * 4 + T * E * 4 + T * k * 8) / hbm),
        "histogram_scan": (T * k * 4 * 3 + A * 8) / hbm,
        "stats": (T * E * 4) / hbm,
    }
    if gather:
        steps["gate_up_gather"] = max(4 * A * d * F / tc, (T * d * b + Ea * 2 * F * d * b + A * F * b) / hbm)
    else:
        steps["permute"] = (T * d * b + A * d * b) / hbm
        steps["gate_up"] = max(4 * A * d * F / tc, (A * d * b + Ea * 2 * F * d * b + A * F * b) / hbm)
    if fused:
        steps["down_combine"] = max(2 * A * F * d / tc, (A * F * b + Ea * d * F * b + 2 * T * d * 4) / hbm)
        if ob == 2:
            steps["round_output"] = (T * d * 4 + T * d * 2) / hbm
    else:
        steps["down"] = max(2 * A * F * d / tc, (A * F * b + Ea * d * F * b + A * d * rb) / hbm)
        steps["combine"] = (A * d * rb + T * d * ob) / hbm
    if cfg.F_s:
        Fs = cfg.F_s
        steps["shared"] = max(6 * T * d * Fs / tc, (T * d * b + 3 * d * Fs * b + T * Fs * b + T * d * rb) / hbm)
    return sum(steps.values()) * 1e3, {k_: v * 1e3 for k_, v in steps.items()}


def gate_up_work(cfg, A, E_act, gather=False):
    """Algorithmic work of one gate/up GEMM launch: 4 d F flops per kept assignment row, and the
    bytes it must move: its A rows (the permuted copy, or x itself when gathered), the weights of
    every expert that has a row (2 F x d each), and H (F per row); all bf16."""
    flops = 4.0 * A * cfg.d * cfg.F
    rows_in = (cfg.T if gather else A) * cfg.d * 2
    nbytes = rows_in + E_act * 2 * cfg.F * cfg.d * 2 + A * cfg.F * 2
    return flops, nbytes


def run_ours(args):
    import torch
    import torch.distributed as dist

    from routing_dispatch_expert_moe_b200 import inputs as I
    from routing_dispatch_expert_moe_b200 import moe as M
    from routing_dispatch_expert_moe_b200.layer import MoELayer, MoEWeights

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    cfg = I.CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.with_(T=args.tokens)
    if args.experts:
        cfg = cfg.with_(E=args.experts)
    dt = torch.float32 if cfg.act == "f32" else torch.bfloat16
    x_np = I.gen_x(cfg, seed=replica_seed(rank))        # each replica has its own token batch
    Wg, off, bias = I.gen_router(cfg, 0)
    W_gu, W_dn = I.gen_experts_torch(cfg, 0)
    sh = I.gen_shared(cfg, 0)
    routing = args.routing
    if routing != "learned" and bias is not None:
        bias = None                                     # a fixed rule has no selection to bias
    w = MoEWeights(Wg=torch.from_numpy(Wg).to(dev), W_gu=W_gu.to(dev), W_dn=W_dn.to(dev),
                   logit_offset=None if off is None else torch.from_numpy(off).to(dev),
                   select_bias=None if bias is None else torch.from_numpy(bias).to(dev),
                   W_gu_s=None if sh is None else torch.from_numpy(sh[0]).to(dt).unsqueeze(0).to(dev),
                   W_dn_s=None if sh is None else torch.from_numpy(sh[1]).to(dt).unsqueeze(0).to(dev),
                   W_noise=(torch.from_numpy(I.gen_noise_router(cfg, 0)).to(dev) if routing == "noisy" else None))
    del W_gu, W_dn
    # the routing rule's own per-batch inputs (token ids for hash routing, normal draws for
    # noisy top-k), resident like x
    rin_np = {}
    if routing == "hash":
        rin_np["token_id"] = I.gen_token_ids(cfg, seed=replica_seed(rank))
    elif routing == "noisy":
        rin_np["noise"] = I.gen_noise(cfg, seed=replica_seed(rank))
    rin = {k_: torch.from_numpy(v).to(dev) for k_, v in rin_np.items()}
    cap = M.moe_capacity(cfg.T, cfg.E, cfg.k, cfg.capacity_factor, True)
    x = torch.from_numpy(x_np).to(dt).to(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    out_dt = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    rows_dt = torch.bfloat16 if args.rows_dtype == "bf16" else torch.float32

    def make_layer(combine, dispatch, weights=None):
        return MoELayer(weights or w, cfg.k, cfg.T, cfg.score, cfg.renormalize, cfg.scale, cap, combine=combine,
                        dispatch=dispatch, out_dtype=out_dt, rows_dtype=rows_dt, routing=routing,
                        overlap=not args.no_overlap)

    def capture(fn):
        """One CUDA graph of fn(stream), captured on a side stream."""
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                fn(cs)
        stream.wait_stream(cs)
        return g

    def time_layer(layer, steps, clocks=None, breakdown_steps=0):
        """Warm-up, then `steps` replays of one forward (the layer's own schedule, including
        its second branch) captured as a CUDA graph with timing events as graph nodes on
        the launching stream.  L2 is flushed (256 MB write) before every step, outside the
        timed span.  breakdown_steps > 0: the same kernels replayed one stage after the
        other with an event between stages, for the per-stage split.  Returns per-step ms,
        mean ms per stage, the rows processed and the clock record."""
        for _ in range(args.warmup):
            flush.zero_()
            layer.forward(x, stream, **rin)
        torch.cuda.synchronize()
        assert M.moe_get_device_error() == 0
        rows = int(layer.offsets[-1].item())
        e_act = int((layer.kept > 0).sum().item())
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
        gu_name = "gate_up_gather" if layer.dispatch_mode == "gather" else "gate_up"

        def fwd(s):
            ev[0].record(s)
            layer.forward(x, s, marks={gu_name: (ev[2], ev[3])}, **rin)
            ev[1].record(s)

        graph = capture(fwd)
        for _ in range(3):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize()
        assert M.moe_get_device_error() == 0
        if clocks is not None:
            clocks.start()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        per_step = np.zeros(steps)
        gu_ms = 0.0
        for i in range(steps):
            flush.zero_()                      # L2 flush outside the step
            graph.replay()
            torch.cuda.synchronize()           # read this step's in-graph events
            per_step[i] = ev[0].elapsed_time(ev[1])
            gu_ms += ev[2].elapsed_time(ev[3])
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        clk = clocks.stop() if clocks is not None else None
        assert M.moe_get_device_error() == 0
        del graph

        stage_ms = {"timed_" + gu_name: gu_ms / steps}
        if breakdown_steps > 0:
            stages = layer.stages(x, True, rin.get("token_id"), rin.get("noise"))
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(stages) + 1)]

            def seq(s):
                for i, (_, fn) in enumerate(stages):
                    evs[i].record(s)
                    fn(s)
                evs[len(stages)].record(s)

            g2 = capture(seq)
            acc = np.zeros(len(stages))
            for i in range(breakdown_steps + 2):
                flush.zero_()
                g2.replay()
                torch.cuda.synchronize()
                if i >= 2:
                    acc += [evs[j].elapsed_time(evs[j + 1]) for j in range(len(stages))]
            stage_ms.update({n: float(acc[j] / breakdown_steps) for j, (n, _) in enumerate(stages)})
            del g2
        return per_step, stage_ms, (rows, e_act), clk

    layer = make_layer(args.combine, args.dispatch)
    per_step, stage_ms, (A, E_act), clk = time_layer(layer, args.steps, ClockSampler(local_rank),
                                                     breakdown_steps=args.breakdown_steps)
    total_ms = max_over_ranks(float(per_step.sum()), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(cfg.T, world, args.steps, total_ms)

    other = None
    if args.alt_steps > 0:
        # the other combine form on the same inputs: fused into the down GEMM (fp32 atomics),
        # or gated rows + ordered combine (bitwise reproducible)
        alt = "fused" if args.combine == "rows" else "rows"
        rl = make_layer(alt, layer.dispatch_mode)
        ps, sm, _, _ = time_layer(rl, args.alt_steps, breakdown_steps=min(args.breakdown_steps, 50))
        t = max_over_ranks(float(ps.sum()), dev)
        other = {"dispatch": rl.dispatch_mode,
                 "combine": ("fused into the down GEMM (fp32 atomics)" if alt == "fused"
                             else "gated rows + ordered combine (bitwise reproducible)"),
                 "ms_per_step": round(t / args.alt_steps, 4),
                 "value": round(job_throughput(cfg.T, world, args.alt_steps, t), 1), "steps": args.alt_steps,
                 "stages_ms": {k_: round(v, 4) for k_, v in sm.items()}}
        del rl
        torch.cuda.empty_cache()

    # The routed experts in 4-bit formats (weight-only): the same layer and inputs, the expert
    # GEMMs reading packed codes.  The codes are drawn at random on the device: the kernels do
    # the same work whatever the code values (parity of these GEMMs is tested separately).
    fp4_forms = {}
    for fmt in ([] if args.fp4_steps <= 0 or dt != torch.bfloat16 else ["mxfp4", "nvfp4"]):
        gen = torch.Generator(device=dev).manual_seed(7)
        blk = 32 if fmt == "mxfp4" else 16

        def packed(rows, K):
            codes = torch.randint(0, 256, (rows, K // 2), dtype=torch.uint8, device=dev, generator=gen)
            sc = torch.randint(119, 123, (rows, K // blk), dtype=torch.uint8, device=dev, generator=gen) \
                if fmt == "mxfp4" else torch.randint(0x30, 0x50, (rows, K // blk), dtype=torch.uint8, device=dev,
                                                     generator=gen)
            ts = torch.full((cfg.E,), 2.0 ** -7, dtype=torch.float32, device=dev) if fmt == "nvfp4" else None
            return M.Fp4Weights(fmt, codes, sc, ts)

        w4 = MoEWeights(Wg=w.Wg, W_gu=w.W_gu, W_dn=w.W_dn, logit_offset=w.logit_offset, select_bias=w.select_bias,
                        W_gu_s=w.W_gu_s, W_dn_s=w.W_dn_s,
                        W_gu_fp4=packed(cfg.E * 2 * cfg.F, cfg.d), W_dn_fp4=packed(cfg.E * cfg.d, cfg.F))
        l4 = make_layer("rows", "permute", w4)
        ps, sm, (A4, E4), _ = time_layer(l4, args.fp4_steps, breakdown_steps=min(args.breakdown_steps, 50))
        t = max_over_ranks(float(ps.sum()), dev)
        gu_bytes4 = A4 * cfg.d * 2 + E4 * 2 * cfg.F * cfg.d // 2 + E4 * 2 * cfg.F * (cfg.d // blk) + A4 * cfg.F * 2
        dn_bytes4 = A4 * cfg.F * 2 + E4 * cfg.d * cfg.F // 2 + E4 * cfg.d * (cfg.F // blk) + A4 * cfg.d * rows_dt.itemsize
        fp4_forms[fmt] = {"ms_per_step": round(t / args.fp4_steps, 4),
                          "value": round(job_throughput(cfg.T, world, args.fp4_steps, t), 1), "steps": args.fp4_steps,
                          "stages_ms": {k_: round(v, 4) for k_, v in sm.items()},
                          "gate_up_gbs": round(gu_bytes4 / (sm["gate_up"] * 1e-3) / 1e9, 1) if sm.get("gate_up") else None,
                          "down_gbs": round(dn_bytes4 / (sm["down"] * 1e-3) / 1e9, 1) if sm.get("down") else None,
                          "weights": "synthetic 4-bit codes and scales (random, on the device)"}
        del l4, w4
        torch.cuda.empty_cache()

    # End to end through the public API with host buffers (pinned), copies inside the timing.
    # Two layer instances (shared weights, their own buffers and CUDA graphs) let the copy
    # of batch i+1 in, the forward of batch i and the copy of batch i-1 out run at once on
    # three streams, as a serving loop would; every step still copies its input in and its
    # result out inside the timed region.
    x_host = torch.from_numpy(x_np).to(dt).pin_memory()
    y_host = [torch.empty((cfg.T, cfg.d), dtype=layer.out_dtype).pin_memory() for _ in range(2)]
    e2e_steps = max(3, args.e2e_steps)
    lays = [layer, make_layer(args.combine, args.dispatch)]
    xs = [x, torch.empty_like(x)]
    rin_host = {k_: torch.from_numpy(v).pin_memory() for k_, v in rin_np.items()}
    rins = [rin, {k_: torch.empty_like(v) for k_, v in rin.items()}]
    for l_, x_, r_ in zip(lays, xs, rins):
        x_.copy_(x_host)
        for k_, v in rin_host.items():
            r_[k_].copy_(v)
        l_.capture(x_, token_id=r_.get("token_id"), noise=r_.get("noise"))   # capture once, replay per batch
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_run(n):
        for i in range(n):
            b = i & 1
            s_in.wait_event(ev_comp[b])    # the forward that last read xs[b] has finished
            with torch.cuda.stream(s_in):
                xs[b].copy_(x_host, non_blocking=True)
                for k_, v in rin_host.items():
                    rins[b][k_].copy_(v, non_blocking=True)
            ev_in[b].record(s_in)
            s_comp.wait_event(ev_in[b])
            s_comp.wait_event(ev_out[b])   # the copy-out that last read lays[b].y has finished
            with torch.cuda.stream(s_comp):
                lays[b].replay()
            ev_comp[b].record(s_comp)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                y_host[b].copy_(lays[b].y[:cfg.T], non_blocking=True)
            ev_out[b].record(s_out)

    for b in range(2):                     # events start out recorded (nothing pending)
        ev_comp[b].record(s_comp)
        ev_out[b].record(s_out)
    e2e_run(4)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    e2e_run(e2e_steps)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = job_throughput(cfg.T, world, e2e_steps, e2e_ms)
    h2d_bytes = x_host.numel() * x_host.element_size() + sum(v.numel() * v.element_size()
                                                             for v in rin_host.values())
    d2h_bytes = y_host[0].numel() * y_host[0].element_size()
    del lays

    pk, pk_src = peaks()
    gather = layer.dispatch_mode == "gather"
    gate_up_ms = stage_ms["timed_gate_up_gather" if gather else "timed_gate_up"]   # inside the timed region
    flops, gu_bytes = gate_up_work(cfg, A, E_act, gather)
    # the burst GEMM figure for a timed region well under a second, the sustained one (the
    # power cap settles within about a second of dense work) for longer ones
    tkey = "bf16_tflops_sustained" if total_ms > 1000.0 else "bf16_tflops"
    t_tensor, t_hbm = flops / (pk[tkey] * 1e12), gu_bytes / (pk["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": round(flops / (gate_up_ms * 1e-3) / 1e12, 1),
                "peak": pk[tkey], "unit": "TFLOP/s",
                "peak_source": f"{pk_src[tkey]} {tkey}" + (" (burst)" if tkey == "bf16_tflops" else "")}
    else:
        roof = {"bound": "hbm", "achieved": round(gu_bytes / (gate_up_ms * 1e-3) / 1e9, 1),
                "peak": pk["hbm_gbs"], "unit": "GB/s", "peak_source": f"{pk_src['hbm_gbs']} hbm_gbs"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["algorithmic"] = {"flops": flops, "bytes": gu_bytes, "rows": A, "experts_with_rows": E_act,
                           "tensor_ms": round(t_tensor * 1e3, 4), "hbm_ms": round(t_hbm * 1e3, 4),
                           "kernel_ms": round(gate_up_ms, 4)}
    roof["traffic"] = GATE_UP_TRAFFIC.get((args.workload, layer.dispatch_mode, A))
    fused = args.combine == "fused"
    rb = 4 if fused else layer.y_perm.element_size()
    ob = layer.y.element_size()
    roof_ms, roof_steps = layer_roofline_ms(cfg, A, pk, rb, ob, fused, gather, E_act)
    thr = {}                                # from the per-stage split, when it ran
    if stage_ms.get("route"):
        down_ms = stage_ms["down_combine" if fused else "down"]
        thr["down_tflops"] = round(2.0 * A * cfg.F * cfg.d / (down_ms * 1e-3) / 1e12, 1)
        thr["down_gbs"] = round((A * cfg.F * 2 + E_act * cfg.d * cfg.F * 2 + (0 if fused else A * cfg.d * rb)) /
                                (down_ms * 1e-3) / 1e9, 1)
        thr["gate_up_gbs"] = round(gu_bytes / (stage_ms["gate_up_gather" if gather else "gate_up"] * 1e-3) / 1e9, 1)
        thr["route_tflops"] = round(2.0 * cfg.T * cfg.d * cfg.E / (stage_ms["route"] * 1e-3) / 1e12, 1)
        thr["route_gbs"] = round((cfg.T * cfg.d * 2 + cfg.T * cfg.E * 8 + cfg.T * cfg.k * 8) /
                                 (stage_ms["route"] * 1e-3) / 1e9, 1)
        if not gather:
            thr["permute_gbs"] = round((cfg.T * cfg.d * 2 + A * cfg.d * 2) / (stage_ms["permute"] * 1e-3) / 1e9, 1)
        if not fused:
            thr["combine_gbs"] = round((A * cfg.d * rb + cfg.T * cfg.d * ob) / (stage_ms["combine"] * 1e-3) / 1e9,
                                       1)

    out = None
    if rank == 0:
        cpu = (cpu_baseline(cfg, args.ref_tokens, budget_s=args.cpu_budget)
               if (world == 1 and not args.no_cpu_baseline and routing == "learned") else None)
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
            "data": "synthetic (seeded; integer-grid router inputs, N(0,0.02) bf16 expert weights)",
            "config": {**workload_config(args.workload, cfg, cap), "rows": A,
                       "dispatch": ("gathered inside the gate/up GEMM" if gather else "permute copy"),
                       "combine": ("fused into the down GEMM (fp32 atomics into y)" if fused
                                   else "gated rows + ordered combine (bitwise reproducible)"),
                       "out_dtype": args.out_dtype, "rows_dtype": args.rows_dtype,
                       **({"routing": routing} if routing != "learned" else {}),
                       "parallelism": f"replicas x{world} (independent token batches, no collective)",
                       "l2": "flushed before every step (256 MB write)"},
            "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
                    "d2h_bytes_per_step": d2h_bytes, "steps": e2e_steps,
                    "schedule": "two layer instances, copy in / forward / copy out on three streams"},
            "gpu_launches": args.steps * layer.launches_per_forward(True, cfg.T),
            "roofline": {"kernel": ("moe_expert_gate_up_gather (tcgen05 grouped GEMM, gathered rows, SwiGLU)"
                                    if gather else "moe_expert_gate_up (tcgen05 grouped GEMM + SwiGLU)"), **roof},
            "layer_roofline": {"ms": round(roof_ms, 4), "frac": round(roof_ms / ms_per_step, 4),
                               "tokens_per_s": round(cfg.T / (roof_ms / 1e3), 1)},
            "stages_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
            "stage_roofline_ms": {k_: round(v, 4) for k_, v in roof_steps.items()},
            "stage_throughput": thr,
            "alt_form": other,
            "fp4_forms": fp4_forms or None,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


def _oracle_step(cfg, x_np, Wg, off, bias, gu, dn, sh, tokens):
    """One oracle pass over a token sample: routing, dispatch plan, expert FFN, combine."""
    from oracle import moe_oracle as O
    c = dict(T=len(tokens), E=cfg.E, k=cfg.k, score=cfg.score, renormalize=cfg.renormalize, scale=cfg.scale,
             capacity_factor=cfg.capacity_factor)
    xs = x_np[tokens]
    r = O.layer_routing(c, xs, Wg, off, bias)
    out = O.layer_outputs_for_tokens(np.arange(len(tokens)), xs, r, gu, dn, cfg.act == "bf16", shared=sh)
    return out["y"]


def _oracle_setup(cfg):
    """Inputs for the oracle; each expert's weights are widened to float64 when the oracle asks
    for them (the stress workload's experts would take about 40 GB of float64 at once)."""
    from routing_dispatch_expert_moe_b200 import inputs as I
    x_np = I.gen_x(cfg, 0)
    Wg, off, bias = I.gen_router(cfg, 0)
    W_gu, W_dn = I.gen_experts_torch(cfg, 0)
    sh = I.gen_shared(cfg, 0)
    return x_np, Wg, off, bias, (lambda e: W_gu[e].double().numpy()), (lambda e: W_dn[e].double().numpy()), sh


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else (os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_run(cfg, setup, n_tokens, steps, warmup, seed):
    """The oracle as it stands, timed on the host: each step is one pass of the whole layer
    over a fresh random sample of n_tokens tokens of the workload (routing, capacity and the
    dispatch plan of that sample, the SwiGLU experts in float64, the combine).  Returns
    (tokens/s, total seconds, per-step seconds)."""
    rng = np.random.default_rng(seed)
    for _ in range(warmup):
        _oracle_step(cfg, *setup, rng.choice(cfg.T, size=n_tokens, replace=False))
    times = []
    for _ in range(steps):
        tok = rng.choice(cfg.T, size=n_tokens, replace=False)
        t0 = time.perf_counter()
        _oracle_step(cfg, *setup, tok)
        times.append(time.perf_counter() - t0)
    total = float(np.sum(times))
    return n_tokens * steps / total, total, times


def oracle_sample_text(cfg, n_tokens, steps, total_s):
    return (f"{steps} steps of {n_tokens} of {cfg.T} tokens each (fresh random sample per step): routing, "
            f"capacity and dispatch plan of the sample, SwiGLU experts in float64 numpy, combine; {total_s:.1f} s")


def cpu_baseline(cfg, n_tokens=48, budget_s=15.0):
    """The oracle on the host cores, on the same per-step token sample as the reference arm
    (bench.py --impl reference): as many steps as fit in about budget_s seconds."""
    setup = _oracle_setup(cfg)
    _, t1, _ = oracle_sample_run(cfg, setup, n_tokens, 1, 1, seed=1)
    steps = int(max(1, min(200, budget_s / max(t1, 1e-3))))
    value, total, _ = oracle_sample_run(cfg, setup, n_tokens, steps, 0, seed=2)
    return {"value": round(value, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": oracle_sample_text(cfg, n_tokens, steps, total), "host_cpu": _cpu_model(),
            "nproc": os.cpu_count()}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return None
    from oracle import moe_oracle as O
    from routing_dispatch_expert_moe_b200 import inputs as I
    cfg = I.CONFIGS[args.workload]
    setup = _oracle_setup(cfg)
    n = args.ref_tokens
    value, total, _ = oracle_sample_run(cfg, setup, n, args.steps, args.warmup, seed=2)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": workload_config(args.workload, cfg, O.capacity(cfg.T, cfg.E, cfg.k, cfg.capacity_factor, True)),
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
                             "sample": oracle_sample_text(cfg, n, args.steps, total)},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c5_stress")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens", type=int, default=48,
                    help="tokens per oracle step (the reference arm and cpu_baseline time the same sample)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (smaller cases of the same kernels, e.g. for profiler captures)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (smaller cases of the same kernels, e.g. for profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=50, help="steps timed through host buffers")
    ap.add_argument("--combine", choices=["fused", "rows"], default="rows",
                    help="rows: gated rows + ordered combine (reproducible); fused: combine inside the down GEMM")
    ap.add_argument("--dispatch", choices=["auto", "gather", "permute"], default="permute",
                    help="gather: the gate/up GEMM reads token rows through the row map; permute: x_perm copy; "
                         "auto: gather where the gate/up GEMM takes weight-major tiles, else permute")
    ap.add_argument("--out-dtype", choices=["bf16", "f32"], default="bf16",
                    help="dtype of the layer output y (bf16: fp32 sums rounded once at the end)")
    ap.add_argument("--rows-dtype", choices=["f32", "bf16"], default="bf16",
                    help="dtype of the gated expert rows (the combine='rows' form's down GEMM output)")
    ap.add_argument("--routing", choices=["learned", "uniform", "hash", "noisy"], default="learned",
                    help="expert selection: the learned top-k (the layer's definition), forced-uniform, a hash "
                         "of synthetic Zipf token ids, or noisy top-k (softmax workloads); not the reference arm")
    ap.add_argument("--breakdown-steps", type=int, default=100,
                    help="sequential replays for the per-stage split (0 = skip)")
    ap.add_argument("--fp4-steps", type=int, default=30,
                    help="also time the layer with 4-bit (MXFP4, NVFP4) routed experts for this many steps (0 = skip)")
    ap.add_argument("--no-overlap", action="store_true",
                    help="run the router statistics on the main stream after the combine instead of on a "
                         "second graph branch beside the expert GEMMs")
    ap.add_argument("--alt-steps", type=int, default=100,
                    help="also time the other combine form for this many steps (0 = skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference" and args.routing != "learned":
        ap.error("--routing applies to our arm only (the oracle arm times the learned router)")
    out = run_reference(args) if args.impl == "reference" else run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()

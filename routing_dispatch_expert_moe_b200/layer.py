"""MoE-layer forward as a sequence of the library's C-ABI calls.

MoELayer owns preallocated device buffers for a maximum token count and runs, on one
stream with no host synchronisation:

    moe_route -> moe_histogram_scan
      (routing="uniform" / "hash": moe_router_logits -> moe_route_fixed;
       routing="noisy": moe_router_logits for W_g and W_noise -> moe_route_noisy)
      dispatch="permute": -> moe_permute -> moe_expert_gate_up
      dispatch="gather":  -> moe_expert_gate_up_gather (reads x through the row map)
      combine="rows":  -> moe_expert_down (gate fused) [-> shared expert: gate_up/down
                       with E = 1] -> moe_combine
      combine="fused": [-> shared expert, written into y] -> moe_expert_down_combine
    [-> moe_router_stats]

"rows" sums each token's terms in slot order and is bitwise reproducible; "fused" adds
them into y with fp32 atomics inside the down GEMM (no gated-row buffer, no combine
pass), so its y differs from run to run by fp32 rounding only.

Orchestration only: every step runs in the library's CUDA kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import moe as M


@dataclass
class MoEWeights:
    Wg: torch.Tensor                          # [d, E] f32
    W_gu: torch.Tensor                        # [E, 2F, d] act dtype (gate rows, then up rows)
    W_dn: torch.Tensor                        # [E, d, F] act dtype
    logit_offset: Optional[torch.Tensor] = None   # [E] f32
    select_bias: Optional[torch.Tensor] = None    # [E] f32
    W_gu_s: Optional[torch.Tensor] = None     # [1, 2F_s, d] shared expert
    W_dn_s: Optional[torch.Tensor] = None     # [1, d, F_s]
    W_noise: Optional[torch.Tensor] = None    # [d, E] f32: noise router (routing="noisy")
    # 4-bit routed experts (moe.Fp4Weights of W_gu and W_dn, e.g. from moe.quantize_experts_fp4):
    # used in place of W_gu / W_dn by the expert GEMMs (the shared expert stays bf16)
    W_gu_fp4: Optional[object] = None
    W_dn_fp4: Optional[object] = None


class MoELayer:
    def __init__(self, weights: MoEWeights, k: int, T_max: int, score: str = "softmax",
                 renormalize: bool = True, scale: float = 1.0, capacity: int = -1,
                 rows_dtype: torch.dtype = torch.float32, out_dtype: torch.dtype = torch.float32,
                 combine: str = "rows", dispatch: str = "permute", overlap: bool = True,
                 routing: str = "learned", hash_seed: int = 0):
        """rows_dtype: gated expert rows (and the shared expert's output); out_dtype: y.
        fp32 (the default) leaves H as the only bf16 rounding inside the layer.
        combine: "rows" (gated rows + ordered combine) or "fused" (down GEMM adds into an
        fp32 buffer, rounded once to bf16 at the end when out_dtype is bf16).
        dispatch: "permute" (x_perm copy, then the GEMM), "gather" (the GEMM reads the
        token rows through token_of_row; same H bit for bit) or "auto" (gather where the
        gate/up GEMM takes weight-major tiles, moe_gate_up_weight_major; permute otherwise).
        overlap: run the work nothing on the main path waits for (router statistics, and
        clearing y for the fused combine) on a second stream forked from and joined back
        to the caller's stream (one CUDA graph with two branches when captured).
        routing: "learned" (top-k of the router), "uniform" (forced-uniform selection),
        "hash" (experts from a hash of the token ids given to forward, seeded by
        hash_seed) or "noisy" (noisy top-k with weights.W_noise and the standard normal
        draws given to forward; softmax gating).  The fixed rules keep the learned gates
        over the chosen experts; the router statistics always use the router logits."""
        self.fp4 = weights.W_gu_fp4 is not None
        if self.fp4 and (weights.W_dn_fp4 is None or combine != "rows" or dispatch == "gather"
                         or weights.W_gu.dtype != torch.bfloat16):
            raise ValueError("4-bit experts need both W_gu_fp4 and W_dn_fp4, bf16 activations, "
                             "combine='rows' and dispatch='permute' (or 'auto')")
        if routing not in ("learned", "uniform", "hash", "noisy"):
            raise ValueError(f"routing must be learned, uniform, hash or noisy, got {routing!r}")
        if routing != "learned" and weights.select_bias is not None:
            raise ValueError("a selection bias only applies to the learned top-k")
        if routing == "noisy" and (weights.W_noise is None or score != "softmax"):
            raise ValueError("noisy top-k needs weights.W_noise and softmax scoring")
        self.routing, self.hash_seed = routing, hash_seed
        if dispatch not in ("permute", "gather", "auto"):
            raise ValueError(f"dispatch must be 'permute', 'gather' or 'auto', got {dispatch!r}")
        if combine not in ("rows", "fused"):
            raise ValueError(f"combine must be 'rows' or 'fused', got {combine!r}")
        if out_dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("out_dtype must be torch.float32 or torch.bfloat16")
        self.combine_mode = combine
        w = weights
        self.w = w
        self.d, self.E = w.Wg.shape
        self.F = w.W_dn.shape[2]
        self.k, self.T_max = k, T_max
        self.score, self.renormalize, self.scale, self.capacity = score, renormalize, scale, capacity
        self.dtype = w.W_gu.dtype
        self.rows_dtype, self.out_dtype = rows_dtype, out_dtype
        dev = w.Wg.device
        self.device = dev
        E, d, F = self.E, self.d, self.F
        self.rows_max = M.moe_rows_max(T_max, E, k, capacity)
        if dispatch == "auto":
            # gathered where the gate/up GEMM takes weight-major tiles (the token rows are its
            # small operand, read once either way); the permute copy otherwise
            wm = self.dtype == torch.bfloat16 and not self.fp4 and M.moe_gate_up_weight_major(self.rows_max, E)
            dispatch = "gather" if wm else "permute"
        self.dispatch_mode = dispatch
        R = max(self.rows_max, 1)
        f32, i32 = torch.float32, torch.int32
        self.logits = torch.empty((T_max, E), dtype=f32, device=dev)
        self.topk_idx = torch.empty((T_max, k), dtype=i32, device=dev)
        self.topk_gate = torch.empty((T_max, k), dtype=f32, device=dev)
        self.counts = torch.empty(E, dtype=i32, device=dev)
        self.kept = torch.empty(E, dtype=i32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=i32, device=dev)
        self.row_of = torch.empty((T_max, k), dtype=i32, device=dev)
        self.token_of_row = torch.empty(R, dtype=i32, device=dev)
        self.gate_of_row = torch.empty(R, dtype=f32, device=dev)
        self.x_perm = torch.empty((R, d), dtype=self.dtype, device=dev) if dispatch == "permute" else None
        self.h = torch.empty((R, F), dtype=self.dtype, device=dev)
        self.y_perm = torch.empty((R, d), dtype=rows_dtype, device=dev) if combine == "rows" else None
        self.y = torch.empty((T_max, d), dtype=out_dtype, device=dev)
        # the fused combine's fp32 sums: y itself, or a scratch rounded into a bf16 y at the end
        self.y32 = None
        if combine == "fused":
            # a bf16 y: a separate fp32 buffer, zero at rest (the final rounding clears it)
            self.y32 = self.y if out_dtype == torch.float32 else torch.zeros((T_max, d), dtype=f32, device=dev)
        self._y32_at_rest_zero = combine == "fused" and self.y32 is not self.y
        if routing == "noisy":
            self.logits_noise = torch.empty((T_max, E), dtype=f32, device=dev)
            self.H = torch.empty((T_max, E), dtype=f32, device=dev)
        self.load = torch.empty(E, dtype=f32, device=dev)
        self.stats5 = torch.empty(5, dtype=f32, device=dev)
        self.ws = torch.empty(max(M.moe_workspace_bytes(T_max, d, E, k), 16), dtype=torch.uint8, device=dev)
        # the router's exact bf16 split of W_g (and of W_noise), made once here
        self.Wg_split = M.moe_prepare_router_weight(w.Wg)
        self.W_noise_split = M.moe_prepare_router_weight(w.W_noise) if routing == "noisy" else None
        self.overlap = overlap
        if overlap:
            self._side = torch.cuda.Stream(device=dev)
            self._ev_fork, self._ev_routed, self._ev_join = (torch.cuda.Event() for _ in range(3))
        self.has_shared = w.W_gu_s is not None
        if self.has_shared:
            self.F_s = w.W_dn_s.shape[2]
            self.shared_offsets = torch.tensor([0, T_max], dtype=i32, device=dev)
            self.h_s = torch.empty((T_max, self.F_s), dtype=self.dtype, device=dev)
            self.y_s = torch.empty((T_max, d), dtype=rows_dtype, device=dev) if combine == "rows" else None

    # individual steps (so that a caller can time them one by one)
    def route(self, x, stream=None, token_id=None, noise=None):
        T = x.shape[0]
        if self.routing == "learned":
            M.moe_route(x, self.w.Wg, self.k, self.score, self.renormalize, self.scale, self.w.logit_offset,
                        self.w.select_bias, self.logits[:T], self.topk_idx[:T], self.topk_gate[:T], self.ws, stream,
                        Wg_split=self.Wg_split)
            return
        M.moe_router_logits(x, self.w.Wg, self.w.logit_offset, self.logits[:T], self.ws, stream,
                            Wg_split=self.Wg_split)
        if self.routing == "noisy":
            if noise is None:
                raise ValueError("noisy routing needs the standard normal draws (noise=[T, E] f32)")
            M.moe_router_logits(x, self.w.W_noise, None, self.logits_noise[:T], self.ws, stream,
                                Wg_split=self.W_noise_split)
            M.moe_route_noisy(self.logits[:T], self.logits_noise[:T], noise, self.k, self.scale, self.H[:T],
                              self.topk_idx[:T], self.topk_gate[:T], stream)
            return
        if self.routing == "hash" and token_id is None:
            raise ValueError("hash routing needs token_id ([T] int32)")
        M.moe_route_fixed(self.logits[:T], self.k, self.routing, self.score, self.renormalize, self.scale,
                          token_id if self.routing == "hash" else None, self.hash_seed, self.topk_idx[:T],
                          self.topk_gate[:T], stream)

    def histogram_scan(self, T, stream=None):
        M.moe_histogram_scan(self.topk_idx[:T], self.topk_gate[:T], self.E, self.capacity, self.counts, self.kept,
                             self.offsets, self.row_of[:T], self.token_of_row, self.gate_of_row, self.ws, stream)

    def permute(self, x, stream=None):
        M.moe_permute(x, self.row_of[:x.shape[0]], self.rows_max, self.x_perm, stream)

    def gate_up(self, stream=None):
        if self.fp4:
            M.moe_expert_gate_up_fp4(self.x_perm, self.offsets, self.w.W_gu_fp4, self.E, self.F, self.rows_max,
                                     self.h, stream)
            return
        M.moe_expert_gate_up(self.x_perm, self.offsets, self.w.W_gu, self.rows_max, self.h, stream)

    def gate_up_gather(self, x, stream=None):
        M.moe_expert_gate_up_gather(x, self.token_of_row, self.offsets, self.w.W_gu, self.rows_max, self.h, stream)

    def down(self, stream=None):
        if self.fp4:
            M.moe_expert_down_fp4(self.h, self.offsets, self.w.W_dn_fp4, self.E, self.d, self.rows_max,
                                  self.gate_of_row, self.y_perm, stream=stream)
            return
        M.moe_expert_down(self.h, self.offsets, self.w.W_dn, self.rows_max, self.gate_of_row, self.y_perm,
                          stream=stream)

    def shared(self, x, stream=None):
        """Shared expert (weight 1): into y_s ("rows"), or straight into y ("fused")."""
        T = x.shape[0]
        if T != self.T_max:
            self.shared_offsets[1].fill_(T)
        out = self.y_s[:T] if self.combine_mode == "rows" else self.y32[:T]
        M.moe_expert_gate_up(x, self.shared_offsets, self.w.W_gu_s, T, self.h_s[:T], stream)
        M.moe_expert_down(self.h_s[:T], self.shared_offsets, self.w.W_dn_s, T, None, out, stream=stream)

    def down_combine(self, T, stream=None, accumulate=None):
        """accumulate: add onto y as it stands (default: when the shared expert wrote it, or
        when y32 is the zero-at-rest scratch of a bf16 output)."""
        acc = (self.has_shared or self._y32_at_rest_zero) if accumulate is None else accumulate
        M.moe_expert_down_combine(self.h, self.offsets, self.w.W_dn, self.rows_max, self.token_of_row, self.y32[:T],
                                  self.gate_of_row, accumulate=acc, stream=stream)

    def round_output(self, T, stream=None):
        """bf16 y from the fused combine's fp32 sums (the combine's final rounding)."""
        M.moe_round_output(self.y32[:T], self.y[:T], clear=True, stream=stream)

    def combine(self, T, stream=None):
        M.moe_combine(self.y_perm, self.row_of[:T], T, self.rows_max, None,
                      self.y_s[:T] if self.has_shared else None, self.y[:T], stream=stream)

    def stats(self, T, stream=None):
        M.moe_router_stats(self.logits[:T], self.counts, self.kept, self.k, self.score, self.load, self.stats5,
                           self.ws, stream)

    def stages(self, x: torch.Tensor, with_stats: bool = True, token_id=None, noise=None):
        """The forward as (name, fn(stream)) steps in launch order."""
        T = x.shape[0]
        st = [("route", lambda s: self.route(x, s, token_id, noise)),
              ("histogram_scan", lambda s: self.histogram_scan(T, s))]
        if self.dispatch_mode == "permute":
            st += [("permute", lambda s: self.permute(x, s)), ("gate_up", lambda s: self.gate_up(s))]
        else:
            st.append(("gate_up_gather", lambda s: self.gate_up_gather(x, s)))
        if self.combine_mode == "rows":
            st.append(("down", lambda s: self.down(s)))
            if self.has_shared:
                st.append(("shared", lambda s: self.shared(x, s)))
            st.append(("combine", lambda s: self.combine(T, s)))
        else:
            if self.has_shared:
                st.append(("shared", lambda s: self.shared(x, s)))
            st.append(("down_combine", lambda s: self.down_combine(T, s)))
            if self.y32 is not self.y:
                st.append(("round_output", lambda s: self.round_output(T, s)))
        if with_stats:
            st.append(("stats", lambda s: self.stats(T, s)))
        return st

    def forward(self, x: torch.Tensor, stream=None, with_stats: bool = True, marks=None, token_id=None,
                noise=None) -> torch.Tensor:
        """marks: optional {stage name: (event, event)} recorded on the main stream right
        before and after that stage (for timing one kernel inside the real schedule).
        token_id ([T] int32, routing="hash") and noise ([T, E] f32, routing="noisy") are
        that batch's inputs of the routing rule."""
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds T_max={self.T_max}")
        if x.dtype != self.dtype:
            raise ValueError(f"x must be {self.dtype}")
        s = torch.cuda.current_stream() if stream is None else stream

        def run(name, fn):
            m = marks.get(name) if marks else None
            if m is not None:
                m[0].record(s)
            fn(s)
            if m is not None:
                m[1].record(s)

        if not self.overlap:
            for name, fn in self.stages(x, with_stats, token_id, noise):
                run(name, fn)
            return self.y[:T]
        side = self._side
        fused = self.combine_mode == "fused"
        self._ev_fork.record(s)                  # everything the caller queued before (e.g. a read of y)
        side.wait_event(self._ev_fork)
        if fused and not self.has_shared and not self._y32_at_rest_zero:
            M.moe_zero(self.y32[:T], side)       # the fused combine's starting value, off the main path
        run("route", lambda s_: self.route(x, s_, token_id, noise))
        run("histogram_scan", lambda s_: self.histogram_scan(T, s_))
        if with_stats:
            self._ev_routed.record(s)
            side.wait_event(self._ev_routed)
            self.stats(T, side)
        if self.dispatch_mode == "permute":
            run("permute", lambda s_: self.permute(x, s_))
            run("gate_up", lambda s_: self.gate_up(s_))
        else:
            run("gate_up_gather", lambda s_: self.gate_up_gather(x, s_))
        if fused:
            if self.has_shared:
                run("shared", lambda s_: self.shared(x, s_))
            self._ev_join.record(side)
            s.wait_event(self._ev_join)
            run("down_combine", lambda s_: self.down_combine(T, s_, accumulate=True))
            if self.y32 is not self.y:
                run("round_output", lambda s_: self.round_output(T, s_))
        else:
            run("down", lambda s_: self.down(s_))
            if self.has_shared:
                run("shared", lambda s_: self.shared(x, s_))
            run("combine", lambda s_: self.combine(T, s_))
            self._ev_join.record(side)
            s.wait_event(self._ev_join)
        return self.y[:T]

    # ---------------------------------------------------------------- CUDA graph
    def capture(self, x_static: torch.Tensor, with_stats: bool = True, token_id=None, noise=None) -> None:
        """Records one forward over the fixed input buffer x_static into a CUDA graph.

        Replaying it (replay()) runs the same library kernels with no host work per
        step.  Write the next batch into x_static (and token_id / noise, when the routing
        rule reads them) before each replay.  One eager forward runs first so that every
        per-device lookup happens outside the capture.
        """
        self.x_static = x_static
        self.forward(x_static, with_stats=with_stats, token_id=token_id, noise=noise)
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(self.graph, stream=s):
                self.forward(x_static, stream=s, with_stats=with_stats, token_id=token_id, noise=noise)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.y[:self.x_static.shape[0]]

    # library kernels launched by one forward (the scan's workspace memset is not a kernel)
    def _route_launches(self, T: int) -> int:
        """Router kernels: one tensor-core kernel (top-k and gates in its epilogue, plus a
        top-k pass for softmax scores with a selection bias), or the SIMT GEMM and top-k."""
        tc = self.dtype == torch.bfloat16 and T >= 256 and self.d >= 64 and self.E % 4 == 0
        if self.routing == "learned":
            if tc:
                return 2 if (self.score == "softmax" and self.w.select_bias is not None) else 1
            return 2
        gemm = 1                              # the tensor-core or the SIMT logits kernel
        if self.routing == "noisy":
            return 2 * gemm + 2               # two router GEMMs, the noise pass, the top-k
        return gemm + 1                       # the GEMM and the fixed selection

    def launches_per_forward(self, with_stats: bool = True, T: int = None) -> int:
        T = self.T_max if T is None else T
        n = self._route_launches(T) + 2 + 1 + 1 + 1 + 1   # route, scan(2) permute gate_up down combine
        if self.combine_mode == "fused":
            n -= 1                         # down_combine (its zero fill is a memset, not a kernel)
            if self.y32 is not self.y:
                n += 1                     # round_output
        if self.dispatch_mode == "gather":
            n -= 1                         # no permute
        if self.has_shared:
            n += 2
        if with_stats:
            n += 3                         # per-CTA partials, per-expert sums, scalars
        return n

"""Python binding of libmoe_b200.so (include/moe.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensors are torch
CUDA tensors (torch supplies device memory and the current stream); outputs that are
not passed in are allocated with torch.empty.  All arithmetic runs in the library's
CUDA kernels -- there is no CPU or PyTorch fallback: if the shared library is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MOE_B200_LIB", os.path.join(_HERE, "libmoe_b200.so"))

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
SCORE = {"softmax": 0, "sigmoid": 1, "sqrt_softplus": 2}
SELECT = {"uniform": 0, "hash": 1}
FP4 = {"mxfp4": 0, "nvfp4": 1}
DTYPE = {torch.bfloat16: 0, torch.float32: 1}
DEVERR = {0: "none", 1: "expert id out of range", 2: "duplicate expert in a token", 3: "row index out of range",
          4: "scan look-back timeout", 5: "GEMM pipeline timeout"}

_c_void_p, _i32, _i64, _f32, _f64, _size = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                             ctypes.c_double, ctypes.c_size_t)

# name -> (restype, argtypes), mirroring include/moe.h
_SIGNATURES = {
    "moe_version": (_i32, []),
    "moe_status_str": (ctypes.c_char_p, [_i32]),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_capacity": (_i32, [_i32, _i32, _i32, _f64, _i32]),
    "moe_rows_max": (_i64, [_i32, _i32, _i32, _i32]),
    "moe_gate_up_weight_major": (_i32, [_i64, _i32]),
    "moe_route_workspace_bytes": (_size, [_i32, _i32, _i32]),
    "moe_router_weight_bytes": (_size, [_i32, _i32]),
    "moe_prepare_router_weight": (_i32, [_c_void_p, _i32, _i32, _c_void_p, _size, _c_void_p]),
    "moe_route": (_i32, [_c_void_p, _i32, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _i32, _i32, _i32, _i32, _i32,
                         _i32, _f32, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _size, _c_void_p]),
    "moe_router_logits_workspace_bytes": (_size, [_i32, _i32, _i32]),
    "moe_router_logits": (_i32, [_c_void_p, _i32, _c_void_p, _c_void_p, _c_void_p, _i32, _i32, _i32, _c_void_p,
                                 _c_void_p, _size, _c_void_p]),
    "moe_route_fixed": (_i32, [_c_void_p, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _c_void_p, ctypes.c_uint32,
                               _c_void_p, _c_void_p, _c_void_p]),
    "moe_route_noisy": (_i32, [_c_void_p, _c_void_p, _c_void_p, _i32, _i32, _i32, _f32, _c_void_p, _c_void_p,
                               _c_void_p, _c_void_p]),
    "moe_fp4_block_size": (_i32, [_i32]),
    "moe_quantize_fp4_host": (_i32, [_c_void_p, _i64, _i64, _i32, _c_void_p, _c_void_p, _c_void_p, _i32]),
    "moe_dequantize_fp4_host": (_i32, [_c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i32, _c_void_p, _i32]),
    "moe_histogram_scan_workspace_bytes": (_size, [_i32, _i32, _i32]),
    "moe_histogram_scan": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _c_void_p, _c_void_p,
                                  _c_void_p, _c_void_p, _c_void_p, _c_void_p, _size, _c_void_p]),
    "moe_histogram_scan_noalloc": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _c_void_p,
                                          _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "moe_scan_wait_check": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _c_void_p, _c_void_p,
                                   _c_void_p, _c_void_p, _c_void_p, ctypes.c_uint64, _c_void_p, _size, _c_void_p]),
    "moe_histogram_scan_caps": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _i32, _c_void_p, _c_void_p, _c_void_p,
                                       _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _size, _c_void_p]),
    "moe_ep_plan_host": (_i32, [_c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                _c_void_p]),
    "moe_ep_regroup": (_i32, [_c_void_p, _i64, _i32, _c_void_p, _i32, _i32, _c_void_p, _i64, _c_void_p]),
    "moe_ep_dst_base_host": (_i32, [_c_void_p, _i32, _i32, _i32, _i32, _c_void_p]),
    "moe_ep_dispatch": (_i32, [_c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _i32,
                               _i32, _i64, _c_void_p, _c_void_p, _c_void_p]),
    "moe_ep_combine": (_i32, [_c_void_p, _i32, _c_void_p, _i32, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                              _c_void_p, _i32, _i32, _i32, _i32, _i64, _i32, _c_void_p, _c_void_p]),
    "moe_ipc_handle_bytes": (_i32, []),
    "moe_ipc_get_handle": (_i32, [_c_void_p, _c_void_p, ctypes.POINTER(_i64)]),
    "moe_ipc_open_handle": (_i32, [_c_void_p, _i64, ctypes.POINTER(_c_void_p), ctypes.POINTER(_c_void_p)]),
    "moe_ipc_close": (_i32, [_c_void_p]),
    "moe_permute": (_i32, [_c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _i64, _c_void_p, _c_void_p]),
    "moe_expert_gate_up": (_i32, [_c_void_p, _i32, _c_void_p, _i32, _i32, _i32, _i64, _c_void_p, _c_void_p,
                                  _c_void_p]),
    "moe_expert_gate_up_gather": (_i32, [_c_void_p, _i32, _i32, _c_void_p, _c_void_p, _i32, _i32, _i32, _i64,
                                         _c_void_p, _c_void_p, _c_void_p]),
    "moe_expert_down": (_i32, [_c_void_p, _i32, _c_void_p, _i32, _i32, _i32, _i64, _c_void_p, _c_void_p,
                               _i32, _c_void_p, _c_void_p]),
    "moe_grouped_ffn": (_i32, [_c_void_p, _i32, _c_void_p, _i32, _i32, _i32, _i64, _c_void_p, _c_void_p,
                               _c_void_p, _c_void_p, _i32, _c_void_p, _c_void_p]),
    "moe_expert_down_combine": (_i32, [_c_void_p, _i32, _c_void_p, _i32, _i32, _i32, _i64, _c_void_p, _c_void_p,
                                       _c_void_p, _i32, _i32, _c_void_p, _c_void_p]),
    "moe_combine": (_i32, [_c_void_p, _i32, _c_void_p, _c_void_p, _c_void_p, _i32, _i32, _i32, _i64, _i32,
                           _c_void_p, _c_void_p]),
    "moe_router_stats_workspace_bytes": (_size, [_i32, _i32]),
    "moe_router_stats": (_i32, [_c_void_p, _c_void_p, _c_void_p, _i32, _i32, _i32, _i32, _c_void_p, _c_void_p,
                                _c_void_p, _size, _c_void_p]),
    "moe_workspace_bytes": (_size, [_i32, _i32, _i32, _i32]),
    "moe_get_device_error": (_i32, [ctypes.POINTER(_i32), _c_void_p]),
    "moe_zero": (_i32, [_c_void_p, _size, _c_void_p]),
    "moe_round_output": (_i32, [_c_void_p, _i64, _c_void_p, _i32, _c_void_p]),
    "moe_fp4_scales_bytes": (_size, [_i64, _i32, _i32]),
    "moe_prepare_fp4_scales": (_i32, [_c_void_p, _i64, _i32, _i32, _c_void_p, _size, _c_void_p]),
    "moe_expert_gate_up_fp4": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _i32, _i64, _c_void_p, _c_void_p, _i32,
                                      _c_void_p, _c_void_p, _c_void_p]),
    "moe_expert_down_fp4": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _i32, _i64, _c_void_p, _c_void_p, _i32,
                                   _c_void_p, _c_void_p, _i32, _c_void_p, _c_void_p]),
}

_lib = None


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        name = lib().moe_status_str(status).decode()
        extra = ""
        if status == MOE_ERR_CUDA:
            extra = ": " + lib().moe_last_cuda_error().decode()
        super().__init__(f"{fn} failed with {name}{extra}")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is missing: no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not found; build it with "
                               "`python -m routing_dispatch_expert_moe_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return sorted(_SIGNATURES)


# ---------------------------------------------------------------- helpers
def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in DTYPE:
        raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp32)")
    return DTYPE[t.dtype]


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoEError(fn, status)


def _ws(nbytes: int, device, given: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return given
    if given is not None and given.numel() * given.element_size() >= nbytes:
        return given
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- sizes
def moe_capacity(T: int, E: int, k: int, capacity_factor: Optional[float], per_assignment: bool = True) -> int:
    return int(lib().moe_capacity(T, E, k, float(capacity_factor or 0.0), 1 if per_assignment else 0))


def moe_rows_max(T: int, E: int, k: int, capacity: int) -> int:
    return int(lib().moe_rows_max(T, E, k, capacity))


def moe_gate_up_weight_major(rows_max: int, E: int) -> bool:
    """True when the bf16 gate/up GEMMs take weight-major tiles for these sizes."""
    r = int(lib().moe_gate_up_weight_major(rows_max, E))
    if r < 0:
        raise MoEError(f"moe_gate_up_weight_major: invalid sizes rows_max={rows_max}, E={E}")
    return bool(r)


def moe_workspace_bytes(T: int, d: int, E: int, k: int) -> int:
    return int(lib().moe_workspace_bytes(T, d, E, k))


# ---------------------------------------------------------------- the calls
def moe_router_weight_bytes(d: int, E: int) -> int:
    return int(lib().moe_router_weight_bytes(d, E))


def moe_prepare_router_weight(Wg, Wg_split=None, stream=None):
    """The tensor-core router's exact three-term bf16 split of Wg [d, E] f32, made once when
    the weights are loaded.  Returns the uint8 device buffer, or None when the tensor-core
    router does not apply to (d, E) (the router then reads Wg directly)."""
    d, E = Wg.shape
    _need(Wg, "Wg", torch.float32, (d, E))
    nb = moe_router_weight_bytes(d, E)
    if nb == 0:
        return None
    Wg_split = torch.empty(nb, dtype=torch.uint8, device=Wg.device) if Wg_split is None else \
        _need(Wg_split, "Wg_split", torch.uint8)
    if Wg_split.numel() < nb:
        raise ValueError(f"Wg_split must hold {nb} bytes, got {Wg_split.numel()}")
    _check("moe_prepare_router_weight", lib().moe_prepare_router_weight(_p(Wg), d, E, _p(Wg_split), nb,
                                                                        _stream(stream)))
    return Wg_split


def moe_route(x, Wg, k: int, score: str = "softmax", renormalize: bool = True, scale: float = 1.0,
              logit_offset=None, select_bias=None, logits=None, topk_idx=None, topk_gate=None,
              workspace=None, stream=None, Wg_split=None):
    """Router logits, top-k and gates.  Returns (logits [T,E] f32, topk_idx [T,k] i32, topk_gate [T,k] f32).
    Wg_split: moe_prepare_router_weight(Wg)'s buffer (None: the call splits Wg itself)."""
    T, d = x.shape
    E = Wg.shape[1]
    _need(x, "x")
    _need(Wg, "Wg", torch.float32, (d, E))
    if Wg_split is not None:
        _need(Wg_split, "Wg_split", torch.uint8)
    for t, n in ((logit_offset, "logit_offset"), (select_bias, "select_bias")):
        if t is not None:
            _need(t, n, torch.float32, (E,))
    dev = x.device
    logits = torch.empty((T, E), dtype=torch.float32, device=dev) if logits is None else \
        _need(logits, "logits", torch.float32, (T, E))
    topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev) if topk_idx is None else \
        _need(topk_idx, "topk_idx", torch.int32, (T, k))
    topk_gate = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_gate is None else \
        _need(topk_gate, "topk_gate", torch.float32, (T, k))
    nb = int(lib().moe_route_workspace_bytes(T, d, E))
    ws = _ws(nb, dev, workspace)
    _check("moe_route", lib().moe_route(_p(x), _dt(x), _p(Wg), _p(Wg_split), _p(logit_offset), _p(select_bias), T, d,
                                        E, k, SCORE[score], 1 if renormalize else 0, float(scale), _p(logits),
                                        _p(topk_idx), _p(topk_gate), _p(ws), nb, _stream(stream)))
    return logits, topk_idx, topk_gate


def moe_router_logits(x, Wg, logit_offset=None, logits=None, workspace=None, stream=None, Wg_split=None):
    """The router alone: logits [T,E] f32 = x . Wg (+ logit_offset)."""
    T, d = x.shape
    E = Wg.shape[1]
    _need(x, "x")
    _need(Wg, "Wg", torch.float32, (d, E))
    if Wg_split is not None:
        _need(Wg_split, "Wg_split", torch.uint8)
    if logit_offset is not None:
        _need(logit_offset, "logit_offset", torch.float32, (E,))
    dev = x.device
    logits = torch.empty((T, E), dtype=torch.float32, device=dev) if logits is None else \
        _need(logits, "logits", torch.float32, (T, E))
    nb = int(lib().moe_router_logits_workspace_bytes(T, d, E))
    ws = _ws(nb, dev, workspace)
    _check("moe_router_logits", lib().moe_router_logits(_p(x), _dt(x), _p(Wg), _p(Wg_split), _p(logit_offset), T, d,
                                                        E, _p(logits), _p(ws), nb, _stream(stream)))
    return logits


def moe_route_fixed(logits, k: int, rule: str = "uniform", score: str = "softmax", renormalize: bool = True,
                    scale: float = 1.0, token_id=None, seed: int = 0, topk_idx=None, topk_gate=None, stream=None):
    """Forced-uniform or hash selection with the learned gates.  Returns (topk_idx, topk_gate)."""
    T, E = logits.shape
    _need(logits, "logits", torch.float32)
    if rule not in SELECT:
        raise ValueError(f"rule must be one of {sorted(SELECT)}")
    if token_id is not None:
        _need(token_id, "token_id", torch.int32, (T,))
    elif rule == "hash":
        raise ValueError("hash selection needs token_id")
    dev = logits.device
    topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev) if topk_idx is None else \
        _need(topk_idx, "topk_idx", torch.int32, (T, k))
    topk_gate = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_gate is None else \
        _need(topk_gate, "topk_gate", torch.float32, (T, k))
    _check("moe_route_fixed", lib().moe_route_fixed(_p(logits), T, E, k, SCORE[score], 1 if renormalize else 0,
                                                    float(scale), SELECT[rule], _p(token_id),
                                                    int(seed) & 0xFFFFFFFF, _p(topk_idx), _p(topk_gate),
                                                    _stream(stream)))
    return topk_idx, topk_gate


def moe_route_noisy(logits, logits_noise, noise, k: int, scale: float = 1.0, H=None, topk_idx=None,
                    topk_gate=None, stream=None):
    """Noisy top-k gating.  Returns (H [T,E] f32, topk_idx [T,k] i32, topk_gate [T,k] f32)."""
    T, E = logits.shape
    _need(logits, "logits", torch.float32)
    _need(logits_noise, "logits_noise", torch.float32, (T, E))
    _need(noise, "noise", torch.float32, (T, E))
    dev = logits.device
    H = torch.empty((T, E), dtype=torch.float32, device=dev) if H is None else _need(H, "H", torch.float32, (T, E))
    topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev) if topk_idx is None else \
        _need(topk_idx, "topk_idx", torch.int32, (T, k))
    topk_gate = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_gate is None else \
        _need(topk_gate, "topk_gate", torch.float32, (T, k))
    _check("moe_route_noisy", lib().moe_route_noisy(_p(logits), _p(logits_noise), _p(noise), T, E, k, float(scale),
                                                    _p(H), _p(topk_idx), _p(topk_gate), _stream(stream)))
    return H, topk_idx, topk_gate


def _host_ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def moe_quantize_fp4_host(W, fmt: str = "mxfp4", threads: int = 0):
    """4-bit expert weights packed on the host: W [rows, K] (numpy, fp32) ->
    (codes uint8 [rows, K/2], scales uint8 [rows, K/block], tensor_scale float or None)."""
    import numpy as np
    if fmt not in FP4:
        raise ValueError(f"fmt must be one of {sorted(FP4)}")
    W = np.ascontiguousarray(W, dtype=np.float32)
    rows, K = W.shape
    block = int(lib().moe_fp4_block_size(FP4[fmt]))
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, max(K // block, 0)), np.uint8)
    ts = np.ones(1, np.float32)
    _check("moe_quantize_fp4_host", lib().moe_quantize_fp4_host(_host_ptr(W), rows, K, FP4[fmt], _host_ptr(codes),
                                                                _host_ptr(scales), _host_ptr(ts), int(threads)))
    return codes, scales, (float(ts[0]) if fmt == "nvfp4" else None)


def moe_dequantize_fp4_host(codes, scales, tensor_scale, K: int, fmt: str = "mxfp4", threads: int = 0):
    """Inverse of moe_quantize_fp4_host: fp32 W [rows, K] (numpy)."""
    import numpy as np
    if fmt not in FP4:
        raise ValueError(f"fmt must be one of {sorted(FP4)}")
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows = codes.shape[0]
    W = np.empty((rows, K), np.float32)
    ts = np.array([1.0 if tensor_scale is None else tensor_scale], np.float32)
    _check("moe_dequantize_fp4_host", lib().moe_dequantize_fp4_host(_host_ptr(codes), _host_ptr(scales),
                                                                    _host_ptr(ts), rows, K, FP4[fmt],
                                                                    _host_ptr(W), int(threads)))
    return W


class Fp4Weights:
    """One expert weight tensor in a 4-bit format, on the device: codes [rows, K/2] uint8 and
    scales [rows, K/block] uint8 as moe_quantize_fp4_host writes them and, for NVFP4,
    tensor_scale [E] f32 (one per expert).  rows = E * 2F for W_gu (gate rows then up rows
    per expert), E * d for W_dn.  The scales are rearranged once here for the GEMMs
    (moe_prepare_fp4_scales); .scales keeps the packer's layout."""

    def __init__(self, fmt: str, codes, scales, tensor_scale=None, stream=None):
        if fmt not in FP4:
            raise ValueError(f"fmt must be one of {sorted(FP4)}")
        self.fmt, self.codes, self.scales, self.tensor_scale = fmt, codes, scales, tensor_scale
        rows, half = codes.shape
        K = 2 * half
        _need(codes, "codes", torch.uint8)
        _need(scales, "scales", torch.uint8)
        nb = int(lib().moe_fp4_scales_bytes(rows, K, FP4[fmt]))
        if nb == 0:
            raise ValueError("K must be a multiple of 64")
        self.scales_prepared = torch.empty(nb, dtype=torch.uint8, device=codes.device)
        _check("moe_prepare_fp4_scales", lib().moe_prepare_fp4_scales(
            _p(scales), rows, K, FP4[fmt], _p(self.scales_prepared), nb, _stream(stream)))


def quantize_experts_fp4(W, fmt: str = "mxfp4", device="cuda", threads: int = 0) -> Fp4Weights:
    """Packs stacked expert weights W [E, rows_e, K] (torch, any float dtype, on the host)
    with the library's host packer, one expert at a time (NVFP4: one tensor scale per
    expert), and copies the result to the device."""
    import numpy as np
    E, R, K = W.shape
    block = int(lib().moe_fp4_block_size(FP4[fmt]))
    codes = torch.empty((E * R, K // 2), dtype=torch.uint8)
    scales = torch.empty((E * R, K // block), dtype=torch.uint8)
    ts = np.ones(E, np.float32)
    for e in range(E):
        c, sc, t = moe_quantize_fp4_host(W[e].float().numpy(), fmt, threads)
        codes[e * R:(e + 1) * R] = torch.from_numpy(c)
        scales[e * R:(e + 1) * R] = torch.from_numpy(sc)
        if t is not None:
            ts[e] = t
    return Fp4Weights(fmt, codes.to(device), scales.to(device),
                      torch.from_numpy(ts).to(device) if fmt == "nvfp4" else None)


def _need_fp4(w: Fp4Weights, rows: int, K: int, E: int):
    if not isinstance(w, Fp4Weights):
        raise ValueError("expected Fp4Weights")
    block = int(lib().moe_fp4_block_size(FP4[w.fmt]))
    _need(w.codes, "codes", torch.uint8, (rows, K // 2))
    _need(w.scales, "scales", torch.uint8, (rows, K // block))
    if w.fmt == "nvfp4":
        _need(w.tensor_scale, "tensor_scale", torch.float32, (E,))


def moe_expert_gate_up_fp4(x_rows, offsets, W_gu: Fp4Weights, E: int, F: int, rows_max: int, h=None, stream=None):
    """H = silu(X Wg^T) * (X Wu^T) with 4-bit weights W_gu (rows E * 2F, K = d)."""
    d = x_rows.shape[1]
    _need(x_rows, "x_rows", torch.bfloat16)
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need_fp4(W_gu, E * 2 * F, d, E)
    h = torch.empty((max(rows_max, 1), F), dtype=torch.bfloat16, device=x_rows.device) if h is None else \
        _need(h, "h", torch.bfloat16)
    _check("moe_expert_gate_up_fp4", lib().moe_expert_gate_up_fp4(
        _p(x_rows), _p(offsets), E, d, F, rows_max, _p(W_gu.codes), _p(W_gu.scales_prepared), FP4[W_gu.fmt],
        _p(W_gu.tensor_scale), _p(h), _stream(stream)))
    return h


def moe_expert_down_fp4(h, offsets, W_dn: Fp4Weights, E: int, d: int, rows_max: int, gate_of_row=None, y_rows=None,
                        y_dtype=None, stream=None):
    """Gated rows = gate_of_row * (H W_dn^T) with 4-bit weights W_dn (rows E * d, K = F)."""
    F = h.shape[1]
    _need(h, "h", torch.bfloat16)
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need_fp4(W_dn, E * d, F, E)
    if gate_of_row is not None:
        _need(gate_of_row, "gate_of_row", torch.float32)
    y_dtype = y_rows.dtype if y_rows is not None else (y_dtype or torch.float32)
    y_rows = torch.empty((max(rows_max, 1), d), dtype=y_dtype, device=h.device) if y_rows is None else \
        _need(y_rows, "y_rows")
    _check("moe_expert_down_fp4", lib().moe_expert_down_fp4(
        _p(h), _p(offsets), E, d, F, rows_max, _p(W_dn.codes), _p(W_dn.scales_prepared), FP4[W_dn.fmt],
        _p(W_dn.tensor_scale), _p(gate_of_row), _dt(y_rows), _p(y_rows), _stream(stream)))
    return y_rows


def moe_histogram_scan(topk_idx, topk_gate, E: int, capacity: int = -1, counts=None, kept=None, offsets=None,
                       row_of=None, token_of_row=None, gate_of_row=None, workspace=None, stream=None):
    """Returns dict(counts, kept, offsets, row_of, token_of_row, gate_of_row, rows_max)."""
    T, k = topk_idx.shape
    _need(topk_idx, "topk_idx", torch.int32)
    _need(topk_gate, "topk_gate", torch.float32, (T, k))
    dev = topk_idx.device
    rows_max = moe_rows_max(T, E, k, capacity)
    mk = lambda t, shape, dt, n: torch.empty(shape, dtype=dt, device=dev) if t is None else _need(t, n, dt)
    counts = mk(counts, (E,), torch.int32, "counts")
    kept = mk(kept, (E,), torch.int32, "kept")
    offsets = mk(offsets, (E + 1,), torch.int32, "offsets")
    row_of = mk(row_of, (T, k), torch.int32, "row_of")
    token_of_row = mk(token_of_row, (max(rows_max, 1),), torch.int32, "token_of_row")
    gate_of_row = mk(gate_of_row, (max(rows_max, 1),), torch.float32, "gate_of_row")
    nb = int(lib().moe_histogram_scan_workspace_bytes(T, k, E))
    ws = _ws(nb, dev, workspace)
    _check("moe_histogram_scan", lib().moe_histogram_scan(
        _p(topk_idx), _p(topk_gate), T, k, E, capacity, _p(counts), _p(kept), _p(offsets), _p(row_of),
        _p(token_of_row), _p(gate_of_row), _p(ws), nb, _stream(stream)))
    return {"counts": counts, "kept": kept, "offsets": offsets, "row_of": row_of, "token_of_row": token_of_row,
            "gate_of_row": gate_of_row, "rows_max": rows_max}


def moe_histogram_scan_noalloc(topk_idx, topk_gate, E: int, capacity: int, counts, kept, offsets, row_of,
                               token_of_row, gate_of_row, stream=None):
    """moe_histogram_scan without a workspace, for callers that cannot allocate device memory:
    the library's own 4 MiB scratch array is used instead.  Every output buffer must be
    passed in (this wrapper allocates nothing either), all on topk_idx's device, which is
    made current for the call.  Calls that overlap on the GPU race on the shared scratch;
    the first call on a device must come before any stream capture."""
    T, k = topk_idx.shape
    _need(topk_idx, "topk_idx", torch.int32)
    _need(topk_gate, "topk_gate", torch.float32, (T, k))
    rows = max(moe_rows_max(T, E, k, capacity), 1)
    for t, n, dt, shape in ((counts, "counts", torch.int32, (E,)), (kept, "kept", torch.int32, (E,)),
                            (offsets, "offsets", torch.int32, (E + 1,)), (row_of, "row_of", torch.int32, (T, k)),
                            (token_of_row, "token_of_row", torch.int32, None),
                            (gate_of_row, "gate_of_row", torch.float32, None)):
        _need(t, n, dt, shape)
    for t, n in ((token_of_row, "token_of_row"), (gate_of_row, "gate_of_row")):
        if t.numel() < rows:
            raise ValueError(f"{n} must hold at least moe_rows_max(T, E, k, capacity) = {rows} entries, "
                             f"got {t.numel()}")
    dev = topk_idx.device
    for t, n in ((topk_gate, "topk_gate"), (counts, "counts"), (kept, "kept"), (offsets, "offsets"),
                 (row_of, "row_of"), (token_of_row, "token_of_row"), (gate_of_row, "gate_of_row")):
        if t.device != dev:
            raise ValueError(f"{n} is on {t.device}, topk_idx on {dev}: every buffer must be on one device")
    with torch.cuda.device(dev):
        _check("moe_histogram_scan_noalloc", lib().moe_histogram_scan_noalloc(
            _p(topk_idx), _p(topk_gate), T, k, E, capacity, _p(counts), _p(kept), _p(offsets), _p(row_of),
            _p(token_of_row), _p(gate_of_row), _stream(stream)))


def moe_scan_wait_check(topk_idx, topk_gate, E: int, wait_ns: int, capacity: int = -1, stream=None):
    """Diagnostic: the histogram/scan with its first chunk withheld, so that every look-back
    wait runs out after wait_ns and records MOE_DEVERR_SCAN_TIMEOUT (read it with
    moe_get_device_error).  The outputs are not meaningful."""
    T, k = topk_idx.shape
    _need(topk_idx, "topk_idx", torch.int32)
    _need(topk_gate, "topk_gate", torch.float32, (T, k))
    dev = topk_idx.device
    rows = max(moe_rows_max(T, E, k, capacity), 1)
    i32 = torch.int32
    counts, kept = torch.empty(E, dtype=i32, device=dev), torch.empty(E, dtype=i32, device=dev)
    offsets, row_of = torch.empty(E + 1, dtype=i32, device=dev), torch.empty((T, k), dtype=i32, device=dev)
    token_of_row = torch.empty(rows, dtype=i32, device=dev)
    gate_of_row = torch.empty(rows, dtype=torch.float32, device=dev)
    nb = int(lib().moe_histogram_scan_workspace_bytes(T, k, E))
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
    _check("moe_scan_wait_check", lib().moe_scan_wait_check(
        _p(topk_idx), _p(topk_gate), T, k, E, capacity, _p(counts), _p(kept), _p(offsets), _p(row_of),
        _p(token_of_row), _p(gate_of_row), int(wait_ns), _p(ws), nb, _stream(stream)))


def moe_permute(x, row_of, rows_max: int, x_perm=None, stream=None):
    T, d = x.shape
    k = row_of.shape[1]
    _need(x, "x")
    _need(row_of, "row_of", torch.int32, (T, k))
    x_perm = torch.empty((max(rows_max, 1), d), dtype=x.dtype, device=x.device) if x_perm is None else \
        _need(x_perm, "x_perm", x.dtype)
    _check("moe_permute", lib().moe_permute(_p(x), _dt(x), T, d, k, _p(row_of), rows_max, _p(x_perm),
                                            _stream(stream)))
    return x_perm


def moe_expert_gate_up(x_rows, offsets, W_gu, rows_max: int, h=None, stream=None):
    E, F2, d = W_gu.shape
    F = F2 // 2
    _need(x_rows, "x_rows")
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(W_gu, "W_gu", x_rows.dtype)
    h = torch.empty((max(rows_max, 1), F), dtype=x_rows.dtype, device=x_rows.device) if h is None else \
        _need(h, "h", x_rows.dtype)
    _check("moe_expert_gate_up", lib().moe_expert_gate_up(_p(x_rows), _dt(x_rows), _p(offsets), E, d, F, rows_max,
                                                          _p(W_gu), _p(h), _stream(stream)))
    return h


def moe_expert_gate_up_gather(x, token_of_row, offsets, W_gu, rows_max: int, h=None, stream=None):
    """H = silu(X Wg^T) * (X Wu^T) with X[r] = x[token_of_row[r]]: the permute fused into the GEMM."""
    E, F2, d = W_gu.shape
    F = F2 // 2
    _need(x, "x")
    if x.dim() != 2 or x.shape[1] != d:
        raise ValueError(f"x must be [T, {d}]")
    _need(token_of_row, "token_of_row", torch.int32)
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(W_gu, "W_gu", x.dtype)
    h = torch.empty((max(rows_max, 1), F), dtype=x.dtype, device=x.device) if h is None else _need(h, "h", x.dtype)
    _check("moe_expert_gate_up_gather",
           lib().moe_expert_gate_up_gather(_p(x), _dt(x), x.shape[0], _p(token_of_row), _p(offsets), E, d, F,
                                           rows_max, _p(W_gu), _p(h), _stream(stream)))
    return h


def moe_expert_down(h, offsets, W_dn, rows_max: int, gate_of_row=None, y_rows=None, y_dtype=None, stream=None):
    """Gated rows y_rows = gate_of_row * (H W_dn^T) in y_dtype (default: y_rows' dtype, else fp32)."""
    E, d, F = W_dn.shape
    _need(h, "h")
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(W_dn, "W_dn", h.dtype)
    if gate_of_row is not None:
        _need(gate_of_row, "gate_of_row", torch.float32)
    y_dtype = y_rows.dtype if y_rows is not None else (y_dtype or torch.float32)
    y_rows = torch.empty((max(rows_max, 1), d), dtype=y_dtype, device=h.device) if y_rows is None else \
        _need(y_rows, "y_rows")
    _check("moe_expert_down", lib().moe_expert_down(_p(h), _dt(h), _p(offsets), E, d, F, rows_max, _p(W_dn),
                                                    _p(gate_of_row), _dt(y_rows), _p(y_rows), _stream(stream)))
    return y_rows


def moe_round_output(y32, y, clear: bool = False, stream=None):
    """y = bf16_rne(y32): the combine's final rounding of an fp32 sum (clear: zero y32 as it
    is read, ready for the next accumulation)."""
    _need(y32, "y32", torch.float32)
    _need(y, "y", torch.bfloat16, tuple(y32.shape))
    _check("moe_round_output", lib().moe_round_output(_p(y32), y32.numel(), _p(y), 1 if clear else 0,
                                                       _stream(stream)))
    return y


def moe_zero(t, stream=None):
    """Clears a contiguous device tensor with the library's memset (stream-ordered)."""
    _need(t, "t")
    _check("moe_zero", lib().moe_zero(_p(t), t.numel() * t.element_size(), _stream(stream)))
    return t


def moe_expert_down_combine(h, offsets, W_dn, rows_max: int, token_of_row, y, gate_of_row=None,
                            accumulate: bool = False, stream=None):
    """y[token_of_row[r]] += gate_of_row[r] * (H[r] W_dn^T) into fp32 y [T, d] (zeroed first
    unless accumulate); the combine fused into the down GEMM, summed with fp32 atomics."""
    E, d, F = W_dn.shape
    _need(h, "h")
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(W_dn, "W_dn", h.dtype)
    _need(token_of_row, "token_of_row", torch.int32)
    if gate_of_row is not None:
        _need(gate_of_row, "gate_of_row", torch.float32)
    _need(y, "y", torch.float32)
    if y.dim() != 2 or y.shape[1] != d:
        raise ValueError(f"y must be [T, {d}]")
    _check("moe_expert_down_combine",
           lib().moe_expert_down_combine(_p(h), _dt(h), _p(offsets), E, d, F, rows_max, _p(W_dn), _p(gate_of_row),
                                         _p(token_of_row), y.shape[0], 1 if accumulate else 0, _p(y),
                                         _stream(stream)))
    return y


def moe_grouped_ffn(x_rows, offsets, W_gu, W_dn, rows_max: int, gate_of_row=None, h=None, y_rows=None,
                    y_dtype=None, stream=None):
    E, F2, d = W_gu.shape
    F = F2 // 2
    _need(x_rows, "x_rows")
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(W_gu, "W_gu", x_rows.dtype)
    _need(W_dn, "W_dn", x_rows.dtype, (E, d, F))
    dev = x_rows.device
    h = torch.empty((max(rows_max, 1), F), dtype=x_rows.dtype, device=dev) if h is None else _need(h, "h")
    y_dtype = y_rows.dtype if y_rows is not None else (y_dtype or torch.float32)
    y_rows = torch.empty((max(rows_max, 1), d), dtype=y_dtype, device=dev) if y_rows is None else \
        _need(y_rows, "y_rows")
    _check("moe_grouped_ffn", lib().moe_grouped_ffn(_p(x_rows), _dt(x_rows), _p(offsets), E, d, F, rows_max,
                                                    _p(W_gu), _p(W_dn), _p(gate_of_row), _p(h), _dt(y_rows),
                                                    _p(y_rows), _stream(stream)))
    return y_rows


def moe_combine(y_rows, row_of, T: int, rows_max: int, topk_gate=None, shared_y=None, y=None, y_dtype=None,
                stream=None):
    """y[t] = sum_j (g_j) y_rows[row_of[t, j]] (+ shared_y[t]) in y_dtype (default fp32)."""
    d = y_rows.shape[1]
    k = row_of.shape[1]
    _need(y_rows, "y_rows")
    _need(row_of, "row_of", torch.int32, (T, k))
    if shared_y is not None:
        _need(shared_y, "shared_y", y_rows.dtype, (T, d))
    if topk_gate is not None:
        _need(topk_gate, "topk_gate", torch.float32, (T, k))
    y_dtype = y.dtype if y is not None else (y_dtype or torch.float32)
    y = torch.empty((T, d), dtype=y_dtype, device=y_rows.device) if y is None else _need(y, "y")
    _check("moe_combine", lib().moe_combine(_p(y_rows), _dt(y_rows), _p(row_of), _p(topk_gate), _p(shared_y), T, d,
                                            k, rows_max, _dt(y), _p(y), _stream(stream)))
    return y


def moe_router_stats(logits, counts, kept, k: int, score: str = "softmax", load=None, stats5=None, workspace=None,
                     stream=None):
    """Returns (load [E] f32, stats5 [5] f32 = aux, z, dropped, max_over_mean, cv)."""
    T, E = logits.shape
    _need(logits, "logits", torch.float32)
    _need(counts, "counts", torch.int32, (E,))
    _need(kept, "kept", torch.int32, (E,))
    dev = logits.device
    load = torch.empty(E, dtype=torch.float32, device=dev) if load is None else _need(load, "load", torch.float32)
    stats5 = torch.empty(5, dtype=torch.float32, device=dev) if stats5 is None else \
        _need(stats5, "stats5", torch.float32)
    nb = int(lib().moe_router_stats_workspace_bytes(T, E))
    ws = _ws(nb, dev, workspace)
    _check("moe_router_stats", lib().moe_router_stats(_p(logits), _p(counts), _p(kept), T, E, k, SCORE[score],
                                                      _p(load), _p(stats5), _p(ws), nb, _stream(stream)))
    return load, stats5


def moe_get_device_error(stream=None) -> int:
    """Reads and clears the device error word (synchronises the stream); returns the code."""
    code = _i32(0)
    st = lib().moe_get_device_error(ctypes.byref(code), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoEError("moe_get_device_error", st)
    return int(code.value)


# ---------------------------------------------------------------- expert-parallel exchange over peer memory
def moe_ep_dispatch(x, topk_idx, row_of, offsets, dst_base, E: int, G: int, rows_max: int, peer_rows, peer_rows_cap,
                    stream=None):
    """Stores this rank's kept token rows into their owners' expert-major buffers.
    peer_rows: device int64 [G] (buffer addresses), peer_rows_cap: device int64 [G] (rows)."""
    T, d = x.shape
    k = topk_idx.shape[1]
    _need(x, "x")
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    _need(row_of, "row_of", torch.int32, (T, k))
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(dst_base, "dst_base", torch.int32, (E,))
    _need(peer_rows, "peer_rows", torch.int64, (G,))
    _need(peer_rows_cap, "peer_rows_cap", torch.int64, (G,))
    _check("moe_ep_dispatch", lib().moe_ep_dispatch(_p(x), _dt(x), T, d, k, _p(topk_idx), _p(row_of), _p(offsets),
                                                    _p(dst_base), E, G, int(rows_max), _p(peer_rows),
                                                    _p(peer_rows_cap), _stream(stream)))


def moe_ep_combine(peer_rows, rows_dtype, peer_rows_cap, topk_idx, row_of, topk_gate, offsets, dst_base, E: int,
                   G: int, d: int, rows_max: int, y=None, y_dtype=torch.float32, stream=None):
    """y [T, d] = the gated sum of each token's kept rows, read from their owners' buffers."""
    T, k = topk_idx.shape
    dev = topk_idx.device
    if y is None:
        y = torch.empty((T, d), dtype=y_dtype, device=dev)
    _need(y, "y", None, (T, d))
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    _need(row_of, "row_of", torch.int32, (T, k))
    _need(topk_gate, "topk_gate", torch.float32, (T, k))
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(dst_base, "dst_base", torch.int32, (E,))
    _need(peer_rows, "peer_rows", torch.int64, (G,))
    _need(peer_rows_cap, "peer_rows_cap", torch.int64, (G,))
    _check("moe_ep_combine", lib().moe_ep_combine(_p(peer_rows), DTYPE[rows_dtype], _p(peer_rows_cap), G,
                                                  _p(topk_idx), _p(row_of), _p(topk_gate), _p(offsets),
                                                  _p(dst_base), E, T, d, k, int(rows_max), _dt(y), _p(y),
                                                  _stream(stream)))
    return y


def ep_dst_base(counts, g: int, capacity: int):
    """moe_ep_dst_base_host for rank g: counts [G, E] int32 (every rank's per-expert counts)."""
    import numpy as np
    counts = np.ascontiguousarray(counts, np.int32)
    G, E = counts.shape
    out = np.empty(E, np.int32)
    _check("moe_ep_dst_base_host", lib().moe_ep_dst_base_host(ctypes.c_void_p(counts.ctypes.data), G, g, E,
                                                              int(capacity), ctypes.c_void_p(out.ctypes.data)))
    return out


def ipc_handle(t: torch.Tensor):
    """(handle bytes, offset) of the CUDA allocation holding tensor t, for another process."""
    n = int(lib().moe_ipc_handle_bytes())
    buf = ctypes.create_string_buffer(n)
    off = _i64(0)
    _check("moe_ipc_get_handle", lib().moe_ipc_get_handle(_p(t), buf, ctypes.byref(off)))
    return buf.raw, int(off.value)


def ipc_open(handle: bytes, offset: int):
    """Maps another process's allocation: (address, base to pass to ipc_close)."""
    ptr, base = _c_void_p(), _c_void_p()
    _check("moe_ipc_open_handle", lib().moe_ipc_open_handle(handle, int(offset), ctypes.byref(ptr),
                                                            ctypes.byref(base)))
    return int(ptr.value), int(base.value)


def ipc_close(base: int):
    _check("moe_ipc_close", lib().moe_ipc_close(_c_void_p(base)))

"""Beam MoE block forward pass on B200 (sm_100a): Python binding of libbeam_moe.so.

Argument marshalling only: every step of the block runs in the library's CUDA kernels.  PyTorch
provides device memory and the current stream.  There is no CPU fallback: if the library is not
built, importing the binding's functions raises.

The block (Beam launch post, "Welcome Beam" page, section "Mixture of Experts"): sigmoid router over
256 experts, 8 contiguous groups of 32 ranked by the sum of their top-2 scores, 4 groups kept, top 8
experts inside them, router weights normalised to sum 1, expert outputs combined and scaled by 2.5;
each expert a SwiGLU MLP (hidden 5,120, intermediate 2,560).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libbeam_moe.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "beam_moe.h")

OK = 0
ERR_INVALID_CONFIG = 1
ERR_NULL = 2
ERR_MISALIGNED = 3
ERR_WORKSPACE_TOO_SMALL = 4
ERR_UNSUPPORTED_DEVICE = 5
ERR_CUDA = 6
ERR_DEVICE_TIMEOUT = 7
ERR_BAD_INDEX = 8
ERR_INVALID_ARG = 9

WS_ROUTE, WS_PERMUTE, WS_EXPERTS, WS_FORWARD, WS_BLOCK, WS_MXFP8, WS_W4A4, WS_ROUTE_SCREENED = 0, 1, 2, 3, 4, 5, 6, 7


class BeamMoeConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("n_groups", ctypes.c_int32), ("topk_groups", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("group_topn", ctypes.c_int32), ("routed_scale", ctypes.c_float)]


class BeamMoeSublayer(ctypes.Structure):
    _fields_ = [("pre_norm_weight", ctypes.c_void_p), ("post_norm_weight", ctypes.c_void_p),
                ("eps", ctypes.c_float), ("step", ctypes.c_int32)]


class BeamMoeFp8Experts(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_gate_scale", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_up_scale", ctypes.c_void_p), ("w_down", ctypes.c_void_p), ("w_down_scale", ctypes.c_void_p)]


class BeamMoeNvfp4Experts(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_gate", "w_gate_scale", "w_gate_global", "w_up", "w_up_scale",
                                               "w_up_global", "w_down", "w_down_scale", "w_down_global")]


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    hidden: int = 5120
    inter: int = 2560
    n_experts: int = 256
    n_groups: int = 8
    topk_groups: int = 4
    topk: int = 8
    group_topn: int = 2
    routed_scale: float = 2.5

    def c(self) -> BeamMoeConfig:
        return BeamMoeConfig(self.hidden, self.inter, self.n_experts, self.n_groups, self.topk_groups, self.topk,
                             self.group_topn, self.routed_scale)


BEAM_LAYER = LayerConfig()


class BeamMoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


_lib = None
_vp = ctypes.c_void_p
_cfgp = ctypes.POINTER(BeamMoeConfig)


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m group_limited_routing_router_b200.build` (needs nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        L.beam_moe_workspace_size.argtypes = [_cfgp, ctypes.c_int64, ctypes.c_int]
        L.beam_moe_workspace_size.restype = ctypes.c_size_t
        L.beam_moe_route.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp]
        L.beam_moe_route_screened.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                              _vp]
        L.beam_moe_permute.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
        L.beam_moe_experts.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       ctypes.c_size_t, _vp]
        L.beam_moe_forward.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       ctypes.c_size_t, _vp]
        L.beam_moe_forward_profiled.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                _vp, ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_void_p)]
        _f8p = ctypes.POINTER(BeamMoeFp8Experts)
        L.beam_moe_experts_fp8.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f8p, _vp, _vp, ctypes.c_size_t, _vp]
        L.beam_moe_forward_fp8.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f8p, _vp, _vp, _vp, _vp,
                                           ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_void_p)]
        _f4p = ctypes.POINTER(BeamMoeNvfp4Experts)
        L.beam_moe_experts_nvfp4.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f4p, _vp, _vp, ctypes.c_size_t,
                                             _vp]
        L.beam_moe_forward_nvfp4.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f4p, _vp, _vp, _vp, _vp,
                                             ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_void_p)]
        L.beam_moe_block_forward.argtypes = [_cfgp, ctypes.POINTER(BeamMoeSublayer), ctypes.c_int64, _vp, _vp, _vp,
                                             _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
        L.beam_moe_dense_workspace_size.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64]
        L.beam_moe_dense_workspace_size.restype = ctypes.c_size_t
        L.beam_moe_dense_swiglu.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp,
                                            _vp, ctypes.c_size_t, _vp]
        L.beam_moe_dense_swiglu.restype = ctypes.c_int
        L.beam_moe_experts_mxfp8.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f8p, _vp, _vp, ctypes.c_size_t,
                                             _vp]
        L.beam_moe_forward_mxfp8.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f8p, _vp, _vp, _vp, _vp,
                                             ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_void_p)]
        L.beam_moe_experts_w4a4.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f4p, _vp, _vp, ctypes.c_size_t,
                                            _vp]
        L.beam_moe_forward_w4a4.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _f4p, _vp, _vp, _vp, _vp,
                                            ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_void_p)]
        L.beam_moe_gather_rows.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp]
        L.beam_moe_expert_rows_workspace_size.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                          ctypes.c_int64]
        L.beam_moe_expert_rows_workspace_size.restype = ctypes.c_size_t
        L.beam_moe_expert_rows.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, _vp, _vp,
                                           _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
        L.beam_moe_combine.argtypes = [_cfgp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp]
        L.beam_moe_device_status.argtypes = [_vp]
        L.beam_moe_selftest_timeout.argtypes = [ctypes.c_int64, _vp]
        L.beam_moe_strerror.argtypes = [ctypes.c_int]
        L.beam_moe_strerror.restype = ctypes.c_char_p
        for name in ("beam_moe_route", "beam_moe_permute", "beam_moe_experts", "beam_moe_forward",
                     "beam_moe_forward_profiled", "beam_moe_block_forward", "beam_moe_experts_fp8",
                     "beam_moe_forward_fp8", "beam_moe_experts_nvfp4", "beam_moe_forward_nvfp4",
                     "beam_moe_device_status", "beam_moe_gather_rows", "beam_moe_experts_mxfp8", "beam_moe_forward_mxfp8",
                     "beam_moe_experts_w4a4", "beam_moe_forward_w4a4", "beam_moe_expert_rows", "beam_moe_combine",
                     "beam_moe_selftest_timeout"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def declared_symbols() -> list:
    """Entry points declared in include/beam_moe.h."""
    with open(HEADER_PATH) as f:
        return re.findall(r"BEAM_MOE_API\s+[\w\s\*]*?\b(beam_moe_\w+)\s*\(", f.read())


def strerror(code: int) -> str:
    return lib().beam_moe_strerror(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise BeamMoeError(code, where)


def _cfg(cfg) -> BeamMoeConfig:
    if isinstance(cfg, BeamMoeConfig):
        return cfg
    if isinstance(cfg, LayerConfig):
        return cfg.c()
    if isinstance(cfg, dict):
        return LayerConfig(**cfg).c()
    raise TypeError("cfg must be a LayerConfig, a dict of its fields or a BeamMoeConfig")


def _dev(t: Optional[torch.Tensor], name: str, dtype, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def workspace_size(cfg, T: int, which: int) -> int:
    return int(lib().beam_moe_workspace_size(ctypes.byref(_cfg(cfg)), int(T), int(which)))


def _workspace(cfg, T, which, ws, device):
    need = workspace_size(cfg, T, which)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    _dev(ws, "ws", torch.uint8)
    return ws, ws.numel()


def route(cfg, x: torch.Tensor, w_router: torch.Tensor, bias: Optional[torch.Tensor] = None,
          ids: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None, stream=None):
    """Router: returns (topk_ids [T,k] int32, topk_w [T,k] fp32)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
    w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    _check(lib().beam_moe_route(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), _ptr(ids), _ptr(w),
                                _stream(stream)), "beam_moe_route")
    return ids, w


def route_screened(cfg, x: torch.Tensor, w_router: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   ids: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None, ws=None, stream=None):
    """route() with the projection screened on the tensor cores (same outputs): (topk_ids, topk_w)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
    w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_ROUTE_SCREENED, ws, x.device)
    _check(lib().beam_moe_route_screened(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), _ptr(ids),
                                         _ptr(w), _ptr(ws), nbytes, _stream(stream)), "beam_moe_route_screened")
    return ids, w


def permute(cfg, ids: torch.Tensor, ws: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Dispatch order: dict(counts [E] int32, offsets [E+1] int64, row_src [T*k], dest_row [T*k] int32)."""
    c = _cfg(cfg)
    T = ids.shape[0]
    _dev(ids, "ids", torch.int32, (T, c.topk))
    dev = ids.device
    counts = torch.empty(c.n_experts, dtype=torch.int32, device=dev)
    offsets = torch.empty(c.n_experts + 1, dtype=torch.int64, device=dev)
    row_src = torch.empty(max(T * c.topk, 1), dtype=torch.int32, device=dev)
    dest_row = torch.empty(max(T * c.topk, 1), dtype=torch.int32, device=dev)
    ws, nbytes = _workspace(c, T, WS_PERMUTE, ws, dev)
    _check(lib().beam_moe_permute(ctypes.byref(c), T, _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(row_src),
                                  _ptr(dest_row), _ptr(ws), nbytes, _stream(stream)), "beam_moe_permute")
    return dict(counts=counts, offsets=offsets, row_src=row_src[:T * c.topk], dest_row=dest_row[:T * c.topk])


def experts(cfg, x, ids, w, w_gate, w_up, w_down, y=None, ws=None, stream=None) -> torch.Tensor:
    """Expert half for given routing: y [T,H] bf16 = scale * sum_j w[t,j] * E_{ids[t,j]}(x[t])."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    _dev(w_gate, "w_gate", torch.bfloat16, (c.n_experts, c.inter, c.hidden))
    _dev(w_up, "w_up", torch.bfloat16, (c.n_experts, c.inter, c.hidden))
    _dev(w_down, "w_down", torch.bfloat16, (c.n_experts, c.hidden, c.inter))
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    ws, nbytes = _workspace(c, T, WS_EXPERTS, ws, x.device)
    _check(lib().beam_moe_experts(ctypes.byref(c), T, _ptr(x), _ptr(ids), _ptr(w), _ptr(w_gate), _ptr(w_up),
                                  _ptr(w_down), _ptr(y), _ptr(ws), nbytes, _stream(stream)), "beam_moe_experts")
    return y


def forward(cfg, x, w_router, bias, w_gate, w_up, w_down, y=None, ids=None, w=None, ws=None, stream=None,
            return_routing: bool = False):
    """The whole block.  Returns y [T,H] bf16 (and (ids, w) when return_routing)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    _dev(w_gate, "w_gate", torch.bfloat16, (c.n_experts, c.inter, c.hidden))
    _dev(w_up, "w_up", torch.bfloat16, (c.n_experts, c.inter, c.hidden))
    _dev(w_down, "w_down", torch.bfloat16, (c.n_experts, c.hidden, c.inter))
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    if return_routing:
        ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
        w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_FORWARD, ws, x.device)
    _check(lib().beam_moe_forward(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate),
                                  _ptr(w_up), _ptr(w_down), _ptr(y), _ptr(ids), _ptr(w), _ptr(ws), nbytes,
                                  _stream(stream)), "beam_moe_forward")
    return (y, ids, w) if return_routing else y


def gather_rows(cfg, x: torch.Tensor, dest_row: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """Token rows in dispatch order: out[dest_row[t*k + j]] = x[t] -> [T*k, H] bf16."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(dest_row, "dest_row", torch.int32, (T * c.topk,))
    out = torch.empty(T * c.topk, c.hidden, dtype=torch.bfloat16, device=x.device) if out is None else out
    _dev(out, "out", torch.bfloat16, (T * c.topk, c.hidden))
    _check(lib().beam_moe_gather_rows(ctypes.byref(c), T, _ptr(x), _ptr(dest_row), _ptr(out), _stream(stream)),
           "beam_moe_gather_rows")
    return out


def expert_rows(x_rows: torch.Tensor, row_expert: torch.Tensor, w_gate, w_up, w_down,
                out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The experts on rows that each name one (local) expert: [R, H] fp32, unweighted, in row order."""
    R, H = x_rows.shape
    E, I, _ = w_gate.shape
    _dev(x_rows, "x_rows", torch.bfloat16, (R, H))
    _dev(row_expert, "row_expert", torch.int32, (R,))
    _dev(w_gate, "w_gate", torch.bfloat16, (E, I, H))
    _dev(w_up, "w_up", torch.bfloat16, (E, I, H))
    _dev(w_down, "w_down", torch.bfloat16, (E, H, I))
    out = torch.empty(R, H, dtype=torch.float32, device=x_rows.device) if out is None else out
    _dev(out, "out", torch.float32, (R, H))
    need = int(lib().beam_moe_expert_rows_workspace_size(H, I, E, R))
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x_rows.device)
    _dev(ws, "ws", torch.uint8)
    _check(lib().beam_moe_expert_rows(H, I, E, R, _ptr(x_rows), _ptr(row_expert), _ptr(w_gate), _ptr(w_up),
                                      _ptr(w_down), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "beam_moe_expert_rows")
    return out


def combine(cfg, o_rows: torch.Tensor, dest_row: torch.Tensor, w: torch.Tensor, y: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """y [T,H] bf16 = routed_scale * sum_j w[t,j] * o_rows[dest_row[t*k+j]] (FP32, slot order)."""
    c = _cfg(cfg)
    T = w.shape[0]
    _dev(o_rows, "o_rows", torch.float32, (T * c.topk, c.hidden))
    _dev(dest_row, "dest_row", torch.int32, (T * c.topk,))
    _dev(w, "w", torch.float32, (T, c.topk))
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=o_rows.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    _check(lib().beam_moe_combine(ctypes.byref(c), T, _ptr(o_rows), _ptr(dest_row), _ptr(w), _ptr(y),
                                  _stream(stream)), "beam_moe_combine")
    return y


FP8_KEYS = ("q_gate", "s_gate", "q_up", "s_up", "q_down", "s_down")


def _fp8_experts(c: BeamMoeConfig, w8: dict) -> BeamMoeFp8Experts:
    """MXFP8 expert weights: dict of uint8 CUDA tensors q_gate/q_up [E,I,H], q_down [E,H,I] (E4M3 codes)
    and s_gate/s_up [E,H/32,I], s_down [E,I/32,H] (UE8M0 scale codes, K-block-major)."""
    E, H, I = c.n_experts, c.hidden, c.inter
    shapes = dict(q_gate=(E, I, H), q_up=(E, I, H), q_down=(E, H, I),
                  s_gate=(E, H // 32, I), s_up=(E, H // 32, I), s_down=(E, I // 32, H))
    for k in FP8_KEYS:
        if k not in w8:
            raise KeyError(f"FP8 experts need '{k}'")
        _dev(w8[k], k, torch.uint8, shapes[k])
    return BeamMoeFp8Experts(*(w8[k].data_ptr() for k in FP8_KEYS))


def experts_fp8(cfg, x, ids, w, w8: dict, y=None, ws=None, stream=None) -> torch.Tensor:
    """experts() with MXFP8 expert weights (see _fp8_experts for the layout)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    f8 = _fp8_experts(c, w8)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    ws, nbytes = _workspace(c, T, WS_EXPERTS, ws, x.device)
    _check(lib().beam_moe_experts_fp8(ctypes.byref(c), T, _ptr(x), _ptr(ids), _ptr(w), ctypes.byref(f8), _ptr(y),
                                      _ptr(ws), nbytes, _stream(stream)), "beam_moe_experts_fp8")
    return y


def _event_handles(events):
    if events is None:
        return None
    if len(events) != 7:
        raise ValueError("need 7 events")
    handles = (ctypes.c_void_p * 7)()
    for i, e in enumerate(events):
        if e.cuda_event == 0:  # torch creates the CUDA event at its first record
            e.record()
        handles[i] = e.cuda_event
    return handles


def forward_fp8(cfg, x, w_router, bias, w8: dict, y=None, ids=None, w=None, ws=None, stream=None,
                return_routing: bool = False, events=None):
    """forward() with MXFP8 expert weights; `events` (7 torch.cuda.Event, optional) as in forward_profiled."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    f8 = _fp8_experts(c, w8)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    if return_routing:
        ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
        w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_FORWARD, ws, x.device)
    _check(lib().beam_moe_forward_fp8(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), ctypes.byref(f8),
                                      _ptr(y), _ptr(ids), _ptr(w), _ptr(ws), nbytes, _stream(stream),
                                      _event_handles(events)), "beam_moe_forward_fp8")
    return (y, ids, w) if return_routing else y


def experts_mxfp8(cfg, x, ids, w, w8: dict, y=None, ws=None, stream=None) -> torch.Tensor:
    """The expert half on the native FP8 path: MXFP8 weights (as experts_fp8) times MXFP8 activations
    on block-scaled tensor cores (x and h quantised per row in blocks of 32)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    f8 = _fp8_experts(c, w8)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    ws, nbytes = _workspace(c, T, WS_MXFP8, ws, x.device)
    _check(lib().beam_moe_experts_mxfp8(ctypes.byref(c), T, _ptr(x), _ptr(ids), _ptr(w), ctypes.byref(f8), _ptr(y),
                                        _ptr(ws), nbytes, _stream(stream)), "beam_moe_experts_mxfp8")
    return y


def forward_mxfp8(cfg, x, w_router, bias, w8: dict, y=None, ids=None, w=None, ws=None, stream=None,
                  return_routing: bool = False, events=None):
    """forward() on the native FP8 path (see experts_mxfp8); `events` as in forward_fp8."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    f8 = _fp8_experts(c, w8)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    if return_routing:
        ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
        w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_MXFP8, ws, x.device)
    _check(lib().beam_moe_forward_mxfp8(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), ctypes.byref(f8),
                                        _ptr(y), _ptr(ids), _ptr(w), _ptr(ws), nbytes, _stream(stream),
                                        _event_handles(events)), "beam_moe_forward_mxfp8")
    return (y, ids, w) if return_routing else y


NVFP4_KEYS = ("q_gate", "s_gate", "g_gate", "q_up", "s_up", "g_up", "q_down", "s_down", "g_down")


def _nvfp4_experts(c: BeamMoeConfig, w4: dict) -> BeamMoeNvfp4Experts:
    """NVFP4 expert weights: dict of CUDA tensors q_gate/q_up [E,I,H/2], q_down [E,H,I/2] (uint8, two E2M1
    codes per byte, even k in the low nibble); s_gate/s_up [E,H/16,I], s_down [E,I/16,H] (uint8 E4M3
    scale codes); g_gate/g_up/g_down [E] float32 (per-matrix scales)."""
    E, H, I = c.n_experts, c.hidden, c.inter
    shapes = dict(q_gate=(E, I, H // 2), q_up=(E, I, H // 2), q_down=(E, H, I // 2),
                  s_gate=(E, H // 16, I), s_up=(E, H // 16, I), s_down=(E, I // 16, H),
                  g_gate=(E,), g_up=(E,), g_down=(E,))
    for k in NVFP4_KEYS:
        if k not in w4:
            raise KeyError(f"NVFP4 experts need '{k}'")
        _dev(w4[k], k, torch.float32 if k.startswith("g_") else torch.uint8, shapes[k])
    return BeamMoeNvfp4Experts(*(w4[k].data_ptr() for k in NVFP4_KEYS))


def experts_nvfp4(cfg, x, ids, w, w4: dict, y=None, ws=None, stream=None) -> torch.Tensor:
    """experts() with NVFP4 expert weights (see _nvfp4_experts for the layout)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    f4 = _nvfp4_experts(c, w4)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    ws, nbytes = _workspace(c, T, WS_EXPERTS, ws, x.device)
    _check(lib().beam_moe_experts_nvfp4(ctypes.byref(c), T, _ptr(x), _ptr(ids), _ptr(w), ctypes.byref(f4), _ptr(y),
                                        _ptr(ws), nbytes, _stream(stream)), "beam_moe_experts_nvfp4")
    return y


def forward_nvfp4(cfg, x, w_router, bias, w4: dict, y=None, ids=None, w=None, ws=None, stream=None,
                  return_routing: bool = False, events=None):
    """forward() with NVFP4 expert weights; `events` (7 torch.cuda.Event, optional) as in forward_profiled."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    f4 = _nvfp4_experts(c, w4)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    if return_routing:
        ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
        w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_FORWARD, ws, x.device)
    _check(lib().beam_moe_forward_nvfp4(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), ctypes.byref(f4),
                                        _ptr(y), _ptr(ids), _ptr(w), _ptr(ws), nbytes, _stream(stream),
                                        _event_handles(events)), "beam_moe_forward_nvfp4")
    return (y, ids, w) if return_routing else y


def experts_w4a4(cfg, x, ids, w, w4: dict, y=None, ws=None, stream=None) -> torch.Tensor:
    """The expert half on the 4-bit path: NVFP4 weights (as experts_nvfp4) times NVFP4 activations on
    block-scaled tensor cores (x per token with a power-of-two scale, h per row)."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    f4 = _nvfp4_experts(c, w4)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    ws, nbytes = _workspace(c, T, WS_W4A4, ws, x.device)
    _check(lib().beam_moe_experts_w4a4(ctypes.byref(c), T, _ptr(x), _ptr(ids), _ptr(w), ctypes.byref(f4), _ptr(y),
                                       _ptr(ws), nbytes, _stream(stream)), "beam_moe_experts_w4a4")
    return y


def forward_w4a4(cfg, x, w_router, bias, w4: dict, y=None, ids=None, w=None, ws=None, stream=None,
                 return_routing: bool = False, events=None):
    """forward() on the 4-bit path (see experts_w4a4); `events` as in forward_fp8."""
    c = _cfg(cfg)
    T = x.shape[0]
    _dev(x, "x", torch.bfloat16, (T, c.hidden))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    f4 = _nvfp4_experts(c, w4)
    y = torch.empty(T, c.hidden, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, c.hidden))
    if return_routing:
        ids = torch.empty(T, c.topk, dtype=torch.int32, device=x.device) if ids is None else ids
        w = torch.empty(T, c.topk, dtype=torch.float32, device=x.device) if w is None else w
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_W4A4, ws, x.device)
    _check(lib().beam_moe_forward_w4a4(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), ctypes.byref(f4),
                                       _ptr(y), _ptr(ids), _ptr(w), _ptr(ws), nbytes, _stream(stream),
                                       _event_handles(events)), "beam_moe_forward_w4a4")
    return (y, ids, w) if return_routing else y


def block_forward(cfg, stream_in, pre_norm_weight, post_norm_weight, eps: float, step: int, w_router, bias,
                  w_gate, w_up, w_down, stream_out=None, u=None, ids=None, w=None, ws=None, stream=None):
    """One MoE sublayer on the residual stream (pre-norm, block, post-norm, scaled residual).

    Returns stream_out [T,H] bf16 (pass stream_out=stream_in to update in place); `u`, `ids`, `w`,
    when given, receive the pre-norm activation and the routing."""
    c = _cfg(cfg)
    T = stream_in.shape[0]
    _dev(stream_in, "stream_in", torch.bfloat16, (T, c.hidden))
    _dev(pre_norm_weight, "pre_norm_weight", torch.float32, (c.hidden,))
    _dev(post_norm_weight, "post_norm_weight", torch.float32, (c.hidden,))
    _dev(w_router, "w_router", torch.float32, (c.n_experts, c.hidden))
    _dev(bias, "bias", torch.float32, (c.n_experts,))
    _dev(w_gate, "w_gate", torch.bfloat16, (c.n_experts, c.inter, c.hidden))
    _dev(w_up, "w_up", torch.bfloat16, (c.n_experts, c.inter, c.hidden))
    _dev(w_down, "w_down", torch.bfloat16, (c.n_experts, c.hidden, c.inter))
    stream_out = torch.empty_like(stream_in) if stream_out is None else stream_out
    _dev(stream_out, "stream_out", torch.bfloat16, (T, c.hidden))
    _dev(u, "u", torch.bfloat16, (T, c.hidden))
    _dev(ids, "ids", torch.int32, (T, c.topk))
    _dev(w, "w", torch.float32, (T, c.topk))
    ws, nbytes = _workspace(c, T, WS_BLOCK, ws, stream_in.device)
    sub = BeamMoeSublayer(pre_norm_weight.data_ptr(), post_norm_weight.data_ptr(), float(eps), int(step))
    _check(lib().beam_moe_block_forward(ctypes.byref(c), ctypes.byref(sub), T, _ptr(stream_in), _ptr(w_router),
                                        _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(stream_out),
                                        _ptr(u), _ptr(ids), _ptr(w), _ptr(ws), nbytes, _stream(stream)),
           "beam_moe_block_forward")
    return stream_out


def dense_workspace_size(hidden: int, inter: int, T: int) -> int:
    return int(lib().beam_moe_dense_workspace_size(int(hidden), int(inter), int(T)))


def dense_swiglu(x, w_gate, w_up, w_down, y=None, ws=None, stream=None):
    """Dense SwiGLU MLP: y = W_down (SiLU(W_gate x) * (W_up x)), x [T,H] bf16, weights [I,H]/[H,I] bf16."""
    T, H = x.shape
    I = w_gate.shape[0]
    _dev(x, "x", torch.bfloat16, (T, H))
    _dev(w_gate, "w_gate", torch.bfloat16, (I, H))
    _dev(w_up, "w_up", torch.bfloat16, (I, H))
    _dev(w_down, "w_down", torch.bfloat16, (H, I))
    y = torch.empty(T, H, dtype=torch.bfloat16, device=x.device) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, H))
    need = dense_workspace_size(H, I, T)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device) if ws is None else ws
    _dev(ws, "ws", torch.uint8)
    _check(lib().beam_moe_dense_swiglu(H, I, T, _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(y), _ptr(ws),
                                       ws.numel(), _stream(stream)), "beam_moe_dense_swiglu")
    return y


STAGES = ("router", "dispatch", "gather", "gate_up_swiglu", "down", "combine")


def forward_profiled(cfg, x, w_router, bias, w_gate, w_up, w_down, events, y, ids, w, ws, stream=None):
    """forward() that records the 7 torch.cuda.Event objects in `events` around its stages (see
    beam_moe_forward_profiled); all buffers are caller-provided so nothing is allocated per call."""
    c = _cfg(cfg)
    T = x.shape[0]
    handles = _event_handles(events)
    _check(lib().beam_moe_forward_profiled(ctypes.byref(c), T, _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate),
                                           _ptr(w_up), _ptr(w_down), _ptr(y), _ptr(ids), _ptr(w), _ptr(ws),
                                           ws.numel(), _stream(stream), handles), "beam_moe_forward_profiled")
    return y


def device_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(lib().beam_moe_device_status(_stream(stream)))


def selftest_timeout(timeout_us: int, stream=None):
    _check(lib().beam_moe_selftest_timeout(int(timeout_us), _stream(stream)), "beam_moe_selftest_timeout")

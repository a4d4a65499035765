"""CPU oracle of the Beam MoE block forward pass (plain FP64 C via ctypes, numpy glue).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline and
reference arm use it.  The CUDA product path never imports it, and it imports nothing from the
product package.  All arithmetic lives in beam_oracle.c; this module only marshals arrays.

Functions, in the order of the Beam launch post's description of the block ("Welcome Beam" page,
section "Mixture of Experts"):
  router_scores  - sigmoid scores of all experts (FP64 logits)
  select         - group-limited top-k: group score = sum of the top-2, keep 4 of 8 groups, top 8
  route          - router_scores + select
  permute        - stable (expert, token) grouping of the T*k routed pairs
  expert_mlp     - one SwiGLU expert on a set of rows
  combine        - routed_scale * sum_j w_j * expert_j(x)
  forward        - the whole block on host tensors
  forward_tokens - the whole block for a subset of tokens, fetching one expert's weights at a time
  rmsnorm        - the sublayer norm (section "Residual Stream": normalised before and after)
  scaled_residual- stream update sqrt((k-1)/k) * stream + z / sqrt(k) (same section)
  block_forward  - pre-norm -> block -> post-norm -> scaled residual
  quant_mxfp8_rows, expert_mlp_mx8, experts_tokens_mx8
                 - the block-scaled FP8 path: MXFP8 activations (x and h) around the FP8 experts
  quant_nvfp4_rows, expert_mlp_w4a4, experts_tokens_w4a4
                 - the 4-bit path: NVFP4 activations (x and h) around NVFP4 experts
"""
from __future__ import annotations

import ctypes
import os
from typing import Callable, Optional, Sequence

import numpy as np

from . import build as _build

_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_router_scores.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _fp, _dp, _dp]
        L.oracle_router_scores.restype = None
        L.oracle_select.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, _dp, _fp, _i32p, _i32p, _dp, _dp]
        L.oracle_select.restype = ctypes.c_int
        L.oracle_permute.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _i64p, _i32p, _i32p]
        L.oracle_permute.restype = ctypes.c_int
        L.oracle_expert_mlp.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _u16p, _u16p, _u16p, _dp]
        L.oracle_expert_mlp.restype = None
        L.oracle_combine.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp, _dp, _dp]
        L.oracle_combine.restype = None
        L.oracle_rmsnorm.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, _dp, ctypes.c_double, _dp]
        L.oracle_rmsnorm.restype = None
        L.oracle_scaled_residual.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, _dp, ctypes.c_int, _dp]
        L.oracle_scaled_residual.restype = ctypes.c_int
        L.oracle_dequant_mxfp8.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_uint8),
                                           ctypes.POINTER(ctypes.c_uint8), _u16p]
        L.oracle_dequant_mxfp8.restype = ctypes.c_int
        L.oracle_dequant_nvfp4.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_uint8),
                                           ctypes.POINTER(ctypes.c_uint8), ctypes.c_double, _dp]
        L.oracle_dequant_nvfp4.restype = ctypes.c_int
        L.oracle_expert_mlp_f64.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _dp, _dp, _dp, _dp]
        L.oracle_expert_mlp_f64.restype = None
        L.oracle_quant_mxfp8_rows.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, ctypes.POINTER(ctypes.c_uint8),
                                              ctypes.POINTER(ctypes.c_uint8), _dp]
        L.oracle_quant_mxfp8_rows.restype = ctypes.c_int
        L.oracle_expert_mlp_mx8.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _u16p, _u16p, _u16p,
                                            _dp]
        L.oracle_expert_mlp_mx8.restype = ctypes.c_int
        L.oracle_quant_nvfp4_rows.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, ctypes.c_int,
                                              ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint8), _dp, _dp]
        L.oracle_quant_nvfp4_rows.restype = ctypes.c_int
        L.oracle_expert_mlp_w4a4.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _dp, _dp, _dp, _dp]
        L.oracle_expert_mlp_w4a4.restype = ctypes.c_int
        L.oracle_expert_mlp_w4a4_env.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _dp, _dp, _dp,
                                                 ctypes.c_double, _dp, _dp]
        L.oracle_expert_mlp_w4a4_env.restype = ctypes.c_int
        L.oracle_quant_nvfp4_rows_alt.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, ctypes.c_int,
                                                  ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint8), _dp,
                                                  _dp, ctypes.c_double, _dp]
        L.oracle_quant_nvfp4_rows_alt.restype = ctypes.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _ptr(a: Optional[np.ndarray], typ):
    if a is None:
        return ctypes.cast(None, typ)
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(typ)


def bf16_bits(t) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 torch tensor (or pass-through of a uint16 array)."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def router_scores(x_bits: np.ndarray, w_router: np.ndarray, return_logits: bool = False):
    """Sigmoid scores [T,E] fp64 (and the FP64 logits) of x [T,H] (bf16 bits) under W_r [E,H] fp32."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w_router = np.ascontiguousarray(w_router, dtype=np.float32)
    T, H = x_bits.shape
    E = w_router.shape[0]
    assert w_router.shape[1] == H
    score = np.empty((T, E), dtype=np.float64)
    logit = np.empty((T, E), dtype=np.float64) if return_logits else None
    lib().oracle_router_scores(T, H, E, _ptr(x_bits, _u16p), _ptr(w_router, _fp), _ptr(logit, _dp), _ptr(score, _dp))
    return (score, logit) if return_logits else score


def select(score: np.ndarray, layer: dict, bias: Optional[np.ndarray] = None):
    """Group-limited top-k on scores [T,E].  Returns dict(ids, ids64, weight, margin)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    T, E = score.shape
    k = layer["topk"]
    ids = np.empty((T, k), dtype=np.int32)
    ids64 = np.empty((T, k), dtype=np.int32)
    weight = np.empty((T, k), dtype=np.float64)
    margin = np.empty((T, 3), dtype=np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = lib().oracle_select(T, E, layer["n_groups"], layer["topk_groups"], k, layer["group_topn"],
                             _ptr(score, _dp), _ptr(b, _fp), _ptr(ids, _i32p), _ptr(ids64, _i32p),
                             _ptr(weight, _dp), _ptr(margin, _dp))
    if rc != 0:
        raise ValueError(f"oracle_select rejected the configuration (rc={rc})")
    return dict(ids=ids, ids64=ids64, weight=weight, margin=margin)


def route(x_bits: np.ndarray, w_router: np.ndarray, layer: dict, bias: Optional[np.ndarray] = None):
    score = router_scores(x_bits, w_router)
    out = select(score, layer, bias)
    out["score"] = score
    return out


def permute(ids: np.ndarray, n_experts: int):
    """Stable grouping by expert.  Returns dict(counts, offsets, row_src, dest_row)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(n_experts, dtype=np.int32)
    offsets = np.empty(n_experts + 1, dtype=np.int64)
    row_src = np.empty(T * k, dtype=np.int32)
    dest_row = np.empty(T * k, dtype=np.int32)
    rc = lib().oracle_permute(T, k, n_experts, _ptr(ids, _i32p), _ptr(counts, _i32p), _ptr(offsets, _i64p),
                              _ptr(row_src, _i32p), _ptr(dest_row, _i32p))
    if rc != 0:
        raise ValueError("oracle_permute: id out of range")
    return dict(counts=counts, offsets=offsets, row_src=row_src, dest_row=dest_row)


def expert_mlp(x_rows_bits: np.ndarray, wg_bits: np.ndarray, wu_bits: np.ndarray, wd_bits: np.ndarray) -> np.ndarray:
    """SwiGLU expert on rows [n,H] (bf16 bits); weights bf16 bits; returns [n,H] fp64."""
    x_rows_bits = np.ascontiguousarray(x_rows_bits, dtype=np.uint16)
    n, H = x_rows_bits.shape
    I = wg_bits.shape[0]
    assert wg_bits.shape == (I, H) and wu_bits.shape == (I, H) and wd_bits.shape == (H, I)
    out = np.empty((n, H), dtype=np.float64)
    if n == 0:
        return out
    lib().oracle_expert_mlp(n, H, I, _ptr(x_rows_bits, _u16p), _ptr(np.ascontiguousarray(wg_bits), _u16p),
                            _ptr(np.ascontiguousarray(wu_bits), _u16p), _ptr(np.ascontiguousarray(wd_bits), _u16p),
                            _ptr(out, _dp))
    return out


def combine(expert_out: np.ndarray, weight: np.ndarray, routed_scale: float) -> np.ndarray:
    """y [T,H] = routed_scale * sum_j weight[t,j] expert_out[t,j,:] (fp64)."""
    expert_out = np.ascontiguousarray(expert_out, dtype=np.float64)
    weight = np.ascontiguousarray(weight, dtype=np.float64)
    T, k, H = expert_out.shape
    y = np.empty((T, H), dtype=np.float64)
    lib().oracle_combine(T, k, H, float(routed_scale), _ptr(expert_out, _dp), _ptr(weight, _dp), _ptr(y, _dp))
    return y


ExpertFetch = Callable[[int], Sequence[np.ndarray]]


def experts_tokens(x_bits: np.ndarray, ids: np.ndarray, weight: np.ndarray, fetch: ExpertFetch,
                   n_experts: int, routed_scale: float) -> np.ndarray:
    """Expert half of the block for the given rows: x_bits [n,H], ids/weight [n,k].

    `fetch(e)` returns (W_gate[e], W_up[e], W_down[e]) as bf16 bit arrays; it is called once per
    expert that any of the rows uses, so the full weight set never has to sit in host memory.
    """
    n, H = x_bits.shape
    k = ids.shape[1]
    out = np.zeros((n, k, H), dtype=np.float64)
    for e in range(n_experts):
        rows, slots = np.nonzero(ids == e)
        if rows.size == 0:
            continue
        wg, wu, wd = fetch(e)
        out[rows, slots, :] = expert_mlp(x_bits[rows], wg, wu, wd)
    return combine(out, weight, routed_scale)


def forward(x_bits: np.ndarray, w_router: np.ndarray, bias: Optional[np.ndarray], fetch: ExpertFetch,
            layer: dict, tokens: Optional[np.ndarray] = None):
    """The whole block.  Routing for all T tokens; expert outputs for `tokens` (default: all).

    Returns dict(route=..., tokens=..., y=[len(tokens),H] fp64).
    """
    r = route(x_bits, w_router, layer, bias)
    T = x_bits.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    y = experts_tokens(np.ascontiguousarray(x_bits[tok]), r["ids"][tok], r["weight"][tok], fetch,
                       layer["n_experts"], layer["routed_scale"])
    return dict(route=r, tokens=tok, y=y)


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis in FP64: x / sqrt(mean(x^2) + eps) * g."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    T, H = x.shape
    g = np.ascontiguousarray(g, dtype=np.float64)
    assert g.shape == (H,)
    out = np.empty_like(x)
    lib().oracle_rmsnorm(T, H, _ptr(x, _dp), _ptr(g, _dp), float(eps), _ptr(out, _dp))
    return out


def scaled_residual(stream: np.ndarray, z: np.ndarray, step: int) -> np.ndarray:
    """sqrt((k-1)/k) * stream + z / sqrt(k) for residual step k >= 2 (the embedding is step 1)."""
    stream = np.ascontiguousarray(stream, dtype=np.float64)
    z = np.ascontiguousarray(z, dtype=np.float64)
    assert stream.shape == z.shape
    T, H = stream.shape
    out = np.empty_like(stream)
    if lib().oracle_scaled_residual(T, H, _ptr(stream, _dp), _ptr(z, _dp), int(step), _ptr(out, _dp)) != 0:
        raise ValueError("residual step must be >= 2")
    return out


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round FP64 values to bf16 directly (8 significant bits, ties to even) and return the bit patterns."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                              # v = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)    # np.rint rounds half to even
    f = r.astype(np.float32)                        # exact: r has at most 8 significant bits
    return np.ascontiguousarray((f.view(np.uint32) >> 16).astype(np.uint16))


def block_forward(stream_bits: np.ndarray, g_pre: np.ndarray, g_post: np.ndarray, eps: float, step: int,
                  w_router: np.ndarray, bias, fetch: ExpertFetch, layer: dict, tokens=None):
    """The MoE sublayer with its norms and residual update.

    u = bf16(RMSNorm(stream) * g_pre)      (the block's bf16 input activation)
    y = MoE block of u                     (routing on all tokens, experts on `tokens`)
    out = sqrt((k-1)/k) * stream + RMSNorm(y) * g_post / sqrt(k)
    Returns dict(u_bits, route, tokens, y, out) with out in FP64 for the chosen tokens.
    """
    s64 = bf16_bits_to_f64(stream_bits)
    u_bits = f64_to_bf16_bits(rmsnorm(s64, g_pre, eps))
    f = forward(u_bits, w_router, bias, fetch, layer, tokens)
    tok = f["tokens"]
    z = rmsnorm(f["y"], g_post, eps)
    out = scaled_residual(s64[tok], z, step)
    return dict(u_bits=u_bits, route=f["route"], tokens=tok, y=f["y"], out=out)


def dequant_mxfp8(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Exact MXFP8 dequantisation to bf16 bits: q [rows,K] E4M3 codes, scale [K/32,rows] UE8M0 codes."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.uint8)
    rows, K = q.shape
    assert scale.shape == (K // 32, rows)
    out = np.empty((rows, K), dtype=np.uint16)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    if lib().oracle_dequant_mxfp8(rows, K, q.ctypes.data_as(u8p), scale.ctypes.data_as(u8p), _ptr(out, _u16p)) != 0:
        raise ValueError("MXFP8 weights with a NaN code or a value bf16 cannot hold exactly")
    return out


def dequant_nvfp4(q: np.ndarray, scale: np.ndarray, global_scale: float) -> np.ndarray:
    """NVFP4 dequantisation to fp64: q [rows,K/2] packed E2M1 codes (even k in the low nibble),
    scale [K/16,rows] E4M3 codes, one FP32 global scale."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.uint8)
    rows, K2 = q.shape
    K = 2 * K2
    assert scale.shape == (K // 16, rows)
    out = np.empty((rows, K), dtype=np.float64)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    if lib().oracle_dequant_nvfp4(rows, K, q.ctypes.data_as(u8p), scale.ctypes.data_as(u8p),
                                  ctypes.c_double(float(global_scale)), _ptr(out, _dp)) != 0:
        raise ValueError("NVFP4 scale code with the sign bit set, or NaN")
    return out


def expert_mlp_f64(x_rows_bits: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """SwiGLU expert on rows [n,H] (bf16 bits) with fp64 weights; returns [n,H] fp64."""
    x_rows_bits = np.ascontiguousarray(x_rows_bits, dtype=np.uint16)
    n, H = x_rows_bits.shape
    I = wg.shape[0]
    assert wg.shape == (I, H) and wu.shape == (I, H) and wd.shape == (H, I)
    out = np.empty((n, H), dtype=np.float64)
    if n == 0:
        return out
    lib().oracle_expert_mlp_f64(n, H, I, _ptr(x_rows_bits, _u16p),
                                *(_ptr(np.ascontiguousarray(w, dtype=np.float64), _dp) for w in (wg, wu, wd)),
                                _ptr(out, _dp))
    return out


def experts_tokens_f64(x_bits: np.ndarray, ids: np.ndarray, weight: np.ndarray, fetch,
                       n_experts: int, routed_scale: float) -> np.ndarray:
    """experts_tokens with fetch(e) returning fp64 weights (W_gate[e], W_up[e], W_down[e])."""
    n, H = x_bits.shape
    k = ids.shape[1]
    out = np.zeros((n, k, H), dtype=np.float64)
    for e in range(n_experts):
        rows, slots = np.nonzero(ids == e)
        if rows.size == 0:
            continue
        wg, wu, wd = fetch(e)
        out[rows, slots, :] = expert_mlp_f64(x_bits[rows], wg, wu, wd)
    return combine(out, weight, routed_scale)


def quant_mxfp8_rows(v: np.ndarray):
    """MXFP8 activation rows (blocks of 32 along the last axis): returns (codes [rows,K] uint8,
    scale codes [rows,K/32] uint8, dequantised values [rows,K] fp64)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, K = v.shape
    q = np.empty((rows, K), dtype=np.uint8)
    sc = np.empty((rows, K // 32), dtype=np.uint8)
    deq = np.empty((rows, K), dtype=np.float64)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    if lib().oracle_quant_mxfp8_rows(rows, K, _ptr(v, _dp), q.ctypes.data_as(u8p), sc.ctypes.data_as(u8p),
                                     _ptr(deq, _dp)) != 0:
        raise ValueError("MXFP8 activations: K not a multiple of 32, or a scale outside UE8M0")
    return q, sc, deq


def expert_mlp_mx8(x_rows_bits: np.ndarray, wg_bits: np.ndarray, wu_bits: np.ndarray, wd_bits: np.ndarray):
    """The block-scaled FP8 path's SwiGLU expert: MXFP8 x, then h quantised to MXFP8 before the down
    projection (FP64 on the dequantised values); weights as bf16 bits.  Returns [n,H] fp64."""
    x_rows_bits = np.ascontiguousarray(x_rows_bits, dtype=np.uint16)
    n, H = x_rows_bits.shape
    I = wg_bits.shape[0]
    assert wg_bits.shape == (I, H) and wu_bits.shape == (I, H) and wd_bits.shape == (H, I)
    out = np.empty((n, H), dtype=np.float64)
    if n == 0:
        return out
    if lib().oracle_expert_mlp_mx8(n, H, I, _ptr(x_rows_bits, _u16p), _ptr(np.ascontiguousarray(wg_bits), _u16p),
                                   _ptr(np.ascontiguousarray(wu_bits), _u16p),
                                   _ptr(np.ascontiguousarray(wd_bits), _u16p), _ptr(out, _dp)) != 0:
        raise ValueError("MXFP8 activations: a scale outside UE8M0")
    return out


def experts_tokens_mx8(x_bits: np.ndarray, ids: np.ndarray, weight: np.ndarray, fetch: ExpertFetch,
                       n_experts: int, routed_scale: float) -> np.ndarray:
    """experts_tokens of the block-scaled FP8 path (expert_mlp_mx8 per expert)."""
    n, H = x_bits.shape
    k = ids.shape[1]
    out = np.zeros((n, k, H), dtype=np.float64)
    for e in range(n_experts):
        rows, slots = np.nonzero(ids == e)
        if rows.size == 0:
            continue
        out[rows, slots, :] = expert_mlp_mx8(x_bits[rows], *fetch(e))
    return combine(out, weight, routed_scale)


def quant_nvfp4_rows(v: np.ndarray, per_row_scale: bool = True):
    """NVFP4 activation rows (blocks of 16 along the last axis): returns (E2M1 codes [rows,K] uint8 (one
    per element), E4M3 scale codes [rows,K/16] uint8, row scales [rows] fp64, dequantised [rows,K])."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, K = v.shape
    q = np.empty((rows, K), dtype=np.uint8)
    sc = np.empty((rows, K // 16), dtype=np.uint8)
    g = np.empty(rows, dtype=np.float64)
    deq = np.empty((rows, K), dtype=np.float64)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    if lib().oracle_quant_nvfp4_rows(rows, K, _ptr(v, _dp), int(per_row_scale), q.ctypes.data_as(u8p),
                                     sc.ctypes.data_as(u8p), _ptr(g, _dp), _ptr(deq, _dp)) != 0:
        raise ValueError("NVFP4 activations: K not a multiple of 16")
    return q, sc, g, deq


def quant_nvfp4_rows_alt(v: np.ndarray, per_row_scale: bool, eps: float) -> np.ndarray:
    """For each element of quant_nvfp4_rows(v), the largest change of its dequantised value that a
    quantiser deciding on values within eps (relative to the block) could legitimately make."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, K = v.shape
    g = np.empty(rows, dtype=np.float64)
    deq = np.empty((rows, K), dtype=np.float64)
    alt = np.empty((rows, K), dtype=np.float64)
    if lib().oracle_quant_nvfp4_rows_alt(rows, K, _ptr(v, _dp), int(per_row_scale), None, None, _ptr(g, _dp),
                                         _ptr(deq, _dp), float(eps), _ptr(alt, _dp)) != 0:
        raise ValueError("NVFP4 activations: K not a multiple of 16")
    return alt


def expert_mlp_w4a4(x_rows_bits: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, eps=None):
    """The 4-bit path's SwiGLU expert: NVFP4 x (per-row power-of-two scale), h quantised to NVFP4 (row
    scale 1) before the down projection; FP64 weights (dequantised NVFP4).  Returns [n,H] fp64; with
    eps, also the envelope |W_d| alt(h) of quantisation decisions on h taken within eps of a boundary."""
    x_rows_bits = np.ascontiguousarray(x_rows_bits, dtype=np.uint16)
    n, H = x_rows_bits.shape
    I = wg.shape[0]
    assert wg.shape == (I, H) and wu.shape == (I, H) and wd.shape == (H, I)
    out = np.empty((n, H), dtype=np.float64)
    env = np.zeros((n, H), dtype=np.float64) if eps is not None else None
    if n > 0 and lib().oracle_expert_mlp_w4a4_env(
            n, H, I, _ptr(x_rows_bits, _u16p),
            *(_ptr(np.ascontiguousarray(w, dtype=np.float64), _dp) for w in (wg, wu, wd)),
            float(eps or 0.0), _ptr(out, _dp), _ptr(env, _dp)) != 0:
        raise ValueError("4-bit expert: hidden and inter must be multiples of 16")
    return out if eps is None else (out, env)


def experts_tokens_w4a4(x_bits: np.ndarray, ids: np.ndarray, weight: np.ndarray, fetch,
                        n_experts: int, routed_scale: float, eps=None):
    """experts_tokens of the 4-bit path (expert_mlp_w4a4 per expert; fetch gives FP64 weights).  With
    eps, returns (y, envelope of y): routed_scale * sum_j weight_j * envelope_j."""
    n, H = x_bits.shape
    k = ids.shape[1]
    out = np.zeros((n, k, H), dtype=np.float64)
    env = np.zeros((n, k, H), dtype=np.float64) if eps is not None else None
    for e in range(n_experts):
        rows, slots = np.nonzero(ids == e)
        if rows.size == 0:
            continue
        r = expert_mlp_w4a4(x_bits[rows], *fetch(e), eps=eps)
        if eps is None:
            out[rows, slots, :] = r
        else:
            out[rows, slots, :], env[rows, slots, :] = r
    y = combine(out, weight, routed_scale)
    return y if eps is None else (y, combine(env, np.abs(weight), abs(routed_scale)))

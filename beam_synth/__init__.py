"""Seeded synthetic inputs for the Beam MoE block (shared by the tests, the bench and the oracle's callers).

This module draws random numbers and nothing else: it holds none of the routing or expert arithmetic.
Both the CUDA path and the CPU oracle read the tensors it returns; neither is imported here.

Workloads follow the shapes the Beam launch post gives for one MoE layer ("Welcome Beam" page,
section "Mixture of Experts": 256 experts in 8 groups of 32, keep 4 groups, 8 routed experts,
SwiGLU intermediate 2,560; section "Attention": hidden size 5,120).  Distributions are synthetic:

* x ~ N(0, 1), rounded to bf16; optionally a seeded fraction of rows multiplied by a constant
  (outlier rows) before rounding;
* router weight W_r ~ N(0, 1/H) in fp32, selection bias b = 0 unless a stored bias is named;
* expert weights W_gate, W_up ~ N(0, 1/H), W_down ~ N(0, 1/I), rounded to bf16
  (fan-in scaling).

Every tensor (and every expert of a weight tensor) has its own sub-seed derived from
(seed, tensor id, expert): x from the workload seed, W_r and the experts from the layer's weight
seed (the Beam-shaped workloads are batches through one shared layer).  Values depend on the generator device: the CPU generator
(Mersenne twister) and the CUDA generator (Philox) give different streams for one seed, so a
workload states where each tensor is drawn (`expert_device`).  x and W_r are always drawn on the
CPU; expert weights at Beam size are drawn on the GPU (20 GB would take minutes on the host) and
the oracle reads back the experts it needs.
"""
from __future__ import annotations

import dataclasses
import os
from typing import Optional

import numpy as np
import torch

_TENSOR_IDS = {"x": 1, "router": 2, "gate": 3, "up": 4, "down": 5, "outlier": 6, "perm": 7, "sample": 8}

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden")


def sub_seed(seed: int, tensor: str, expert: int = 0) -> int:
    """Deterministic 63-bit sub-seed for (workload seed, tensor, expert)."""
    v = (seed * 1_000_003 + _TENSOR_IDS[tensor] * 10_007 + expert * 7919 + 12345) & ((1 << 63) - 1)
    return v


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    hidden: int
    inter: int
    n_experts: int
    n_groups: int
    topk_groups: int
    topk: int
    group_topn: int = 2
    routed_scale: float = 2.5
    seed: int = 1000
    outlier_frac: float = 0.0
    outlier_scale: float = 30.0
    bias: str = "zero"            # "zero" or the name of a stored bias file under tests/golden/
    expert_device: str = "cpu"    # where expert weights are drawn ("cpu" or "cuda")
    weight_seed: Optional[int] = None  # seed of the layer parameters (W_r, experts); default: seed
    description: str = ""

    @property
    def wseed(self) -> int:
        return self.seed if self.weight_seed is None else self.weight_seed

    @property
    def layer(self) -> dict:
        return dict(hidden=self.hidden, inter=self.inter, n_experts=self.n_experts,
                    n_groups=self.n_groups, topk_groups=self.topk_groups, topk=self.topk,
                    group_topn=self.group_topn, routed_scale=self.routed_scale)

    def with_T(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)


# Beam-shaped workloads are batches through ONE layer: they share the layer parameters (seed 999)
# and differ in T, x and the selection bias.
_BEAM = dict(hidden=5120, inter=2560, n_experts=256, n_groups=8, topk_groups=4, topk=8,
             group_topn=2, routed_scale=2.5, expert_device="cuda", weight_seed=999)

# The five Beam workloads (tiny brute-force case, decode, prefill, skewed routing, long prefill).
WORKLOADS = {
    "tiny": Workload("tiny", T=64, hidden=128, inter=64, n_experts=16, n_groups=4, topk_groups=2,
                     topk=4, seed=1000,
                     description="T=64, hidden 128, 16 experts in 4 groups of 4, keep 2, top-4, I=64"),
    "decode": Workload("decode", T=256, seed=1001, **_BEAM,
                       description="Beam layer, T=256 decode batch, zero bias"),
    "prefill": Workload("prefill", T=4096, seed=1002, **_BEAM,
                        description="Beam layer, T=4096 prefill chunk, zero bias"),
    "skew": Workload("skew", T=16384, seed=1003, bias="skew_bias_beam.txt", **_BEAM,
                     description="Beam layer, T=16384, bias calibrated to Zipf(1.1) expert popularity"),
    "long": Workload("long", T=65536, seed=1004, outlier_frac=0.01, outlier_scale=30.0, **_BEAM,
                     description="Beam layer, T=65536, 1% of rows x30 (outliers)"),
}

# Mid-size cases for parity at sizes the oracle finishes in seconds: several M/N/K tiles, ragged tails.
PARITY_CASES = {
    "mid_a": Workload("mid_a", T=333, hidden=512, inter=384, n_experts=32, n_groups=4, topk_groups=2,
                      topk=4, seed=2001, description="3 gate/up tiles, 4 down tiles, ragged tokens"),
    "mid_b": Workload("mid_b", T=1000, hidden=1024, inter=512, n_experts=64, n_groups=8, topk_groups=4,
                      topk=8, seed=2002, description="Beam group structure scaled down, ~125 rows/expert"),
    "mid_c": Workload("mid_c", T=77, hidden=320, inter=192, n_experts=24, n_groups=3, topk_groups=2,
                      topk=6, group_topn=3, routed_scale=1.0, seed=2003,
                      description="H, I not multiples of 128; group_topn=3; scale 1"),
    "mid_skew": Workload("mid_skew", T=700, hidden=256, inter=128, n_experts=64, n_groups=8,
                         topk_groups=4, topk=8, seed=2004, bias="skew_bias_mid.txt",
                         description="stored bias: Zipf-like popularity, some experts never chosen"),
    "mid_big_expert": Workload("mid_big_expert", T=600, hidden=256, inter=256, n_experts=8,
                               n_groups=2, topk_groups=1, topk=2, seed=2005,
                               description="~150 rows/expert: several token tiles per expert"),
    "beam_small_T": Workload("beam_small_T", T=40, seed=2006, **_BEAM,
                             description="Beam shapes with T=40: most experts get 0 or 1 token"),
}


# Dense SwiGLU MLP of Beam's first three layers.  The intermediate size is not on the pages; this
# build reads it as 20,480 (= 8 x 2,560, the MoE's active width), which also makes the page's
# "8B" non-expert parameters add up (tests/test_closed_forms.py).
DENSE = {
    "dense_prefill": Workload("dense_prefill", T=4096, hidden=5120, inter=20480, n_experts=1, n_groups=1,
                              topk_groups=1, topk=1, seed=3001, expert_device="cuda",
                              description="dense SwiGLU, T=4096, hidden 5120, intermediate 20480"),
    "dense_mid": Workload("dense_mid", T=300, hidden=512, inter=1024, n_experts=1, n_groups=1, topk_groups=1,
                          topk=1, seed=3002, description="dense SwiGLU, ragged T, several tiles"),
}


def get(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name in DENSE:
        return DENSE[name]
    return PARITY_CASES[name]


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_x(wl: Workload, T: Optional[int] = None, seed_offset: int = 0) -> torch.Tensor:
    """x [T, H] bf16 on the CPU: N(0,1); a seeded fraction of rows scaled by outlier_scale."""
    T = wl.T if T is None else T
    g = _gen(sub_seed(wl.seed + seed_offset, "x"), "cpu")
    x = torch.randn(T, wl.hidden, generator=g, dtype=torch.float32)
    if wl.outlier_frac > 0 and T > 0:
        n_out = int(round(wl.outlier_frac * T))
        go = _gen(sub_seed(wl.seed + seed_offset, "outlier"), "cpu")
        rows = torch.randperm(T, generator=go)[:n_out]
        x[rows] *= wl.outlier_scale
    return x.to(torch.bfloat16)


def outlier_rows(wl: Workload, T: Optional[int] = None, seed_offset: int = 0) -> np.ndarray:
    """Indices of the rows make_x scaled (empty when the workload has none)."""
    T = wl.T if T is None else T
    if wl.outlier_frac <= 0 or T == 0:
        return np.zeros(0, dtype=np.int64)
    n_out = int(round(wl.outlier_frac * T))
    go = _gen(sub_seed(wl.seed + seed_offset, "outlier"), "cpu")
    return np.sort(torch.randperm(T, generator=go)[:n_out].numpy())


def make_router(wl: Workload) -> torch.Tensor:
    """W_r [E, H] fp32 on the CPU, N(0, 1/H)."""
    g = _gen(sub_seed(wl.wseed, "router"), "cpu")
    return torch.randn(wl.n_experts, wl.hidden, generator=g, dtype=torch.float32) * (1.0 / wl.hidden) ** 0.5


def load_bias(wl: Workload) -> Optional[torch.Tensor]:
    """Selection bias [E] fp32 or None (zero bias)."""
    if wl.bias == "zero":
        return None
    path = os.path.join(GOLDEN_DIR, wl.bias)
    vals = [float(v) for v in _read_numbers(path)]
    if len(vals) != wl.n_experts:
        raise ValueError(f"{path}: {len(vals)} values, expected {wl.n_experts}")
    return torch.tensor(vals, dtype=torch.float32)


def _read_numbers(path: str):
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield from line.split()


def make_expert(wl: Workload, e: int, device: Optional[str] = None):
    """(W_gate[e] [I,H], W_up[e] [I,H], W_down[e] [H,I]) bf16, drawn on `device`."""
    device = wl.expert_device if device is None else device
    H, I = wl.hidden, wl.inter
    out = []
    for name, shape, fan_in in (("gate", (I, H), H), ("up", (I, H), H), ("down", (H, I), I)):
        g = _gen(sub_seed(wl.wseed, name, e), device)
        w = torch.randn(*shape, generator=g, dtype=torch.float32, device=device) * (1.0 / fan_in) ** 0.5
        out.append(w.to(torch.bfloat16))
    return tuple(out)


def make_experts(wl: Workload, device: Optional[str] = None):
    """Full expert weights (W_gate [E,I,H], W_up [E,I,H], W_down [E,H,I]) bf16 on the generator device."""
    device = wl.expert_device if device is None else device
    E, H, I = wl.n_experts, wl.hidden, wl.inter
    wg = torch.empty(E, I, H, dtype=torch.bfloat16, device=device)
    wu = torch.empty(E, I, H, dtype=torch.bfloat16, device=device)
    wd = torch.empty(E, H, I, dtype=torch.bfloat16, device=device)
    for e in range(E):
        g_, u_, d_ = make_expert(wl, e, device)
        wg[e].copy_(g_)
        wu[e].copy_(u_)
        wd[e].copy_(d_)
    return wg, wu, wd


def sample_tokens(wl: Workload, n: int, T: Optional[int] = None, include=None) -> np.ndarray:
    """A seeded sorted sample of n token indices in [0, T), plus the indices in `include`."""
    T = wl.T if T is None else T
    g = _gen(sub_seed(wl.seed, "sample"), "cpu")
    idx = torch.randperm(T, generator=g)[: min(n, T)].numpy()
    if include is not None and len(include):
        idx = np.union1d(idx, np.asarray(include, dtype=np.int64))
    return np.sort(idx.astype(np.int64))


def quantize_mxfp8(w: torch.Tensor):
    """Synthetic FP8 checkpoint: w [..., rows, K] (bf16) -> (q [..., rows, K] E4M3 codes (uint8),
    scale [..., K/32, rows] UE8M0 codes (uint8)).

    Input preparation only (the OCP MXFP8 layout): each block of 32 consecutive K elements of a row
    gets the power-of-two scale 2^(c-127) with c = ceil(log2(amax / 448)) + 127, so the block's
    largest magnitude maps to at most 448 (E4M3's largest finite value); elements are rounded to
    E4M3 (nearest even).  All-zero blocks get c = 0."""
    *lead, rows, K = w.shape
    assert K % 32 == 0
    if len(lead) == 1 and lead[0] > 8:  # bound the FP32 temporaries: a few experts at a time
        parts = [quantize_mxfp8(w[i:i + 8]) for i in range(0, lead[0], 8)]
        return torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])
    wf = w.float().reshape(*lead, rows, K // 32, 32)
    amax = wf.abs().amax(-1)
    e = torch.ceil(torch.log2(torch.clamp(amax, min=1e-38) / 448.0))
    code = torch.where(amax > 0, torch.clamp(e + 127, 1, 254), torch.zeros_like(e))
    q = (wf / torch.exp2(code - 127).unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    scale = code.to(torch.uint8).transpose(-1, -2).contiguous()  # [..., K/32, rows]
    return q.reshape(*lead, rows, K).contiguous(), scale


def make_experts_fp8(wl: Workload, device: Optional[str] = None):
    """MXFP8 version of make_experts: dict with q_gate, s_gate, q_up, s_up, q_down, s_down."""
    return quantize_experts(*make_experts(wl, device))


def quantize_experts(wg: torch.Tensor, wu: torch.Tensor, wd: torch.Tensor):
    """quantize_mxfp8 of the three expert weight tensors, as the dict make_experts_fp8 returns."""
    out = {}
    for name, w in (("gate", wg), ("up", wu), ("down", wd)):
        out["q_" + name], out["s_" + name] = quantize_mxfp8(w)
    return out


_E2M1_MID = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _e2m1_codes(v: torch.Tensor) -> torch.Tensor:
    """Round to the nearest E2M1 value (0, 0.5, 1, 1.5, 2, 3, 4, 6; ties to the even code) -> 4-bit codes."""
    a = v.abs().clamp(max=6.0)
    mid = _E2M1_MID.to(v.device)
    lower = (a.unsqueeze(-1) > mid).sum(-1)                       # codes 0..7 by strict midpoints
    tie = (lower < 7) & (a == mid[lower.clamp(max=6)])
    code = lower + (tie & (lower % 2 == 1)).to(lower.dtype)
    return (code | ((v < 0).to(code.dtype) << 3)).to(torch.uint8)


def quantize_nvfp4(w: torch.Tensor):
    """Synthetic NVFP4 checkpoint: w [n, rows, K] (bf16) -> (q [n, rows, K/2] uint8, two E2M1 codes per
    byte, even k in the low nibble; scale [n, K/16, rows] E4M3 codes; global [n] fp32).

    Input preparation only (NVIDIA's NVFP4 layout): per matrix a global scale amax / (6 * 448); per
    block of 16 consecutive K elements an E4M3 scale amax_block / (6 * global), rounded to nearest
    even; elements rounded to the nearest E2M1 value of w / (scale * global)."""
    n, rows, K = w.shape
    assert K % 16 == 0
    if n > 8:  # bound the FP32 temporaries: a few matrices at a time
        parts = [quantize_nvfp4(w[i:i + 8]) for i in range(0, n, 8)]
        return tuple(torch.cat([p[j] for p in parts]) for j in range(3))
    wf = w.float()
    amax = wf.abs().amax(dim=(-1, -2))
    glob = torch.where(amax > 0, amax / (6.0 * 448.0), torch.ones_like(amax))
    blk = wf.reshape(n, rows, K // 16, 16)
    s = (blk.abs().amax(-1) / (6.0 * glob[:, None, None])).clamp(max=448.0)
    s_code = s.to(torch.float8_e4m3fn)
    sv = s_code.float()
    denom = (sv * glob[:, None, None]).unsqueeze(-1)
    v = torch.where(denom > 0, blk / torch.where(denom > 0, denom, torch.ones_like(denom)), torch.zeros_like(blk))
    codes = _e2m1_codes(v).reshape(n, rows, K)
    q = (codes[..., 0::2] | (codes[..., 1::2] << 4)).contiguous()
    scale = s_code.view(torch.uint8).transpose(-1, -2).contiguous()    # [n, K/16, rows]
    return q, scale, glob.float()


def quantize_experts_nvfp4(wg: torch.Tensor, wu: torch.Tensor, wd: torch.Tensor):
    """quantize_nvfp4 of the three expert weight tensors: dict q_/s_/g_ for gate, up, down."""
    out = {}
    for name, w in (("gate", wg), ("up", wu), ("down", wd)):
        out["q_" + name], out["s_" + name], out["g_" + name] = quantize_nvfp4(w)
    return out

"""Helpers for the GPU-vs-oracle parity tests.

Routing protocol (the pages fix no tie rule; the oracle's reading is lower index first):
  * the oracle gives, per token, FP64 decision margins: the 4th-vs-5th group score, the
    8th-vs-9th selection value inside the kept groups, and the smallest gap between consecutive
    chosen values;
  * tokens whose group and expert margins are >= 1e-6 must have exactly the oracle's expert SET,
    and, if the order margin is also >= 1e-6, exactly its slot order; their weights match within
    1e-6 (compared per expert id);
  * tokens below a margin are excluded from the bit-exact comparison, counted, and must still be a
    valid choice: at most topk_groups groups, whose total group score is within 1e-6 of the best
    possible, and experts whose total selection value is within 1e-6 of the best inside them.
Output protocol: |y_gpu - y_oracle| <= 2e-2 * RMS(y_oracle) + half_ulp_bf16(y_oracle) elementwise over
the compared tokens.  The second term is the rounding of the exact result to the BF16 output format
itself (up to 2^-8 |y|, about 0.02 RMS at the 5-sigma elements of a 21M-element output), which no
BF16 output can avoid; the raw max |err| / RMS is reported beside it.
"""
from __future__ import annotations

import numpy as np
import torch

import beam_synth as bs
import oracle

MARGIN = 1e-6
Y_TOL = 2e-2


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda", non_blocking=False).contiguous()


class Case:
    """Inputs of one workload on the GPU plus what the oracle needs on the host."""

    def __init__(self, wl: bs.Workload, T=None, weights=None):
        self.wl = wl
        self.T = wl.T if T is None else T
        self.layer = wl.layer
        x = bs.make_x(wl, T=self.T)
        self.x_bits = oracle.bf16_bits(x)
        self.x = to_dev(x)
        W = bs.make_router(wl)
        self.w_router_np = W.numpy()
        self.w_router = to_dev(W)
        b = bs.load_bias(wl)
        self.bias_np = None if b is None else b.numpy()
        self.bias = None if b is None else to_dev(b)
        if weights is None:
            wg, wu, wd = bs.make_experts(wl)
            weights = (to_dev(wg), to_dev(wu), to_dev(wd))
        self.wg, self.wu, self.wd = weights
        self._route = None

    def fetch(self, e: int):
        return (oracle.bf16_bits(self.wg[e]), oracle.bf16_bits(self.wu[e]), oracle.bf16_bits(self.wd[e]))

    def oracle_route(self):
        if self._route is None:
            self._route = oracle.route(self.x_bits, self.w_router_np, self.layer, self.bias_np)
        return self._route

    def oracle_y(self, ids: np.ndarray, w: np.ndarray, tokens: np.ndarray) -> np.ndarray:
        return oracle.experts_tokens(np.ascontiguousarray(self.x_bits[tokens]), ids[tokens], w[tokens], self.fetch,
                                     self.layer["n_experts"], self.layer["routed_scale"])


def compare_routing(r: dict, layer: dict, ids_gpu: np.ndarray, w_gpu: np.ndarray, bias=None,
                    margin_tol: float = MARGIN, weight_tol: float = 1e-6) -> dict:
    ids_o, w_o, margin, score = r["ids"], r["weight"], r["margin"], r["score"]
    T, k = ids_o.shape
    sel_clear = (margin[:, 0] >= margin_tol) & (margin[:, 1] >= margin_tol)
    order_clear = sel_clear & (margin[:, 2] >= margin_tol)
    # exact slot order where the order is decided by more than the margin
    bad = np.nonzero(np.any(ids_gpu[order_clear] != ids_o[order_clear], axis=1))[0]
    assert bad.size == 0, f"slot order differs on {bad.size} clear tokens, e.g. token {np.nonzero(order_clear)[0][bad[0]]}"
    # exact expert sets on every selection-clear token
    so = np.sort(ids_o, axis=1)
    sg = np.sort(ids_gpu, axis=1)
    bad = np.nonzero(np.any(so[sel_clear] != sg[sel_clear], axis=1))[0]
    assert bad.size == 0, f"expert sets differ on {bad.size} clear tokens"
    # weights per expert id
    oo = np.argsort(ids_o, axis=1)
    og = np.argsort(ids_gpu, axis=1)
    wo = np.take_along_axis(w_o, oo, 1)
    wg = np.take_along_axis(w_gpu.astype(np.float64), og, 1)
    dw = np.abs(wo - wg)[sel_clear]
    assert dw.size == 0 or dw.max() <= weight_tol, f"weight error {dw.max():.3g}"
    # every token: distinct ids, weights sum to 1
    assert np.all(np.diff(sg, axis=1) > 0), "repeated expert id"
    np.testing.assert_allclose(w_gpu.sum(1), 1.0, atol=1e-5)
    # excluded tokens: the GPU's choice must be (near-)optimal
    E, G, kg = layer["n_experts"], layer["n_groups"], layer["topk_groups"]
    per = E // G
    sel64 = score + (0.0 if bias is None else bias.astype(np.float64)[None, :])
    excl = np.nonzero(~sel_clear)[0]
    for t in excl:
        v = sel64[t].reshape(G, per)
        gs = np.sort(v, axis=1)[:, ::-1][:, :layer["group_topn"]].sum(1)
        best_groups_total = np.sort(gs)[::-1][:kg].sum()
        gpu_groups = set((ids_gpu[t] // per).tolist())
        assert len(gpu_groups) <= kg
        rest = [g for g in np.argsort(-gs, kind="stable") if g not in gpu_groups]
        S = sorted(gpu_groups) + rest[:kg - len(gpu_groups)]
        assert gs[S].sum() >= best_groups_total - margin_tol, f"token {t}: group choice not optimal"
        cand = np.concatenate([sel64[t, g * per:(g + 1) * per] for g in S])
        best_k = np.sort(cand)[::-1][:k].sum()
        assert sel64[t, ids_gpu[t]].sum() >= best_k - margin_tol, f"token {t}: expert choice not optimal"
    set_equal = np.all(so == sg, axis=1)
    return dict(n_tokens=T, n_excluded=int((~sel_clear).sum()), n_order_excluded=int((sel_clear & ~order_clear).sum()),
                n_excluded_same_set=int((~sel_clear & set_equal).sum()), set_equal=set_equal,
                n_near_miss=int((np.min(margin[:, :2], axis=1) < 1e-5).sum() - (~sel_clear).sum()))


def half_ulp_bf16(y: np.ndarray) -> np.ndarray:
    """Half a BF16 unit in the last place at |y| (8 significant bits): 2^(floor(log2|y|) - 8)."""
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def compare_y(y_gpu: np.ndarray, y_or: np.ndarray, what: str = "y") -> dict:
    y_gpu = y_gpu.astype(np.float64)
    err = np.abs(y_gpu - y_or)
    rms = float(np.sqrt(np.mean(y_or ** 2))) if y_or.size else 0.0
    max_err = float(err.max()) if err.size else 0.0
    excess = err - half_ulp_bf16(y_or)
    max_excess = float(excess.max()) if err.size else 0.0
    assert max_excess <= Y_TOL * rms, \
        f"{what}: max(|err| - half ulp) {max_excess:.4g} > {Y_TOL} * RMS {rms:.4g} (raw max|err| {max_err:.4g})"
    row_rms = np.sqrt(np.mean(y_or ** 2, axis=1)) if y_or.size else np.zeros(0)
    row_ok = np.all(excess <= Y_TOL * row_rms[:, None] + 1e-30, axis=1) if y_or.size else np.zeros(0, bool)
    return dict(max_err=max_err, rms=rms, rel=max_err / rms if rms else 0.0,
                rel_excess=max_excess / rms if rms else 0.0,
                rows_within_own_rms=float(row_ok.mean()) if row_ok.size else 1.0)

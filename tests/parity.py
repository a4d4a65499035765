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
    possible, and experts whose total selection value is within 1e-6 of the best inside them.  The
    output of every excluded token whose set differs is still checked: the oracle recomputes it from
    the GPU's expert ids (oracle_y_checked).

Output protocol (compare_y), for y_gpu (BF16) against the oracle's FP64 y, per token t (one output
row) with tol_t = 2e-2 * RMS(y_oracle[t]):
  * literal bound where BF16 can meet it: on every element whose BF16 spacing is fine enough that
    rounding alone uses at most a quarter of the budget (half a BF16 ulp of y_oracle <= tol_t / 4,
    which holds for |y_oracle| below 1.28 to 2.56 row RMS, by where the binades fall), the literal
    |y_gpu - y_oracle| <= tol_t;
  * every element: y_gpu must be the round-to-nearest BF16 value of some v with
    |v - y_oracle| <= tol_t, i.e. the distance from y_oracle to y_gpu's BF16 rounding interval is at
    most tol_t.  Where |y_oracle| is above ~5 row RMS, half a BF16 ulp is itself more than 1e-2 RMS
    (above 8 RMS more than 2e-2 RMS), so the raw difference of a correctly rounded output can exceed
    the bound with no error in the computation at all;
  * "the output RMS" is read per token: each token's output row is checked at its own scale.  On
    batches whose rows share one scale this is the whole-output rule; on the long batch, whose 1%
    of x30 outlier rows carry ~900x larger outputs, the whole-output RMS (~90x a normal row's)
    would leave the normal rows essentially unchecked, while the per-token rule checks every row
    at its own scale;
  * paths that quantise h inside the layer (the 4-bit path) take a per-element slack from the oracle:
    the output change that E2M1/E4M3 decisions within the oracle's tolerance of a rounding boundary
    could make (oracle.expert_mlp_w4a4 with eps), since the GPU decides them on FP32 values;
  * reported, not enforced: the raw max |y_gpu - y_oracle| / RMS of the whole output (the literal
    quantity), the distance rule against the whole-output RMS, the difference from bf16(y_oracle),
    and how many elements differ from bf16(y_oracle) by more than 2e-2 RMS and by exactly one BF16
    step (an FP32 result and the exact one on opposite sides of a rounding midpoint: one step is
    0.031 RMS at |y| in [4, 8) RMS).
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
    """Inputs of one workload on the GPU plus what the oracle needs on the host.

    weights: the experts as GPU tensors (drawn here when None); host: the same weights as host bf16
    bit arrays (the oracle then reads them instead of copying each expert back from the GPU)."""

    def __init__(self, wl: bs.Workload, T=None, weights=None, host=None):
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
        self.host = host
        self._route = None

    def fetch(self, e: int):
        if self.host is not None:
            return tuple(h[e] for h in self.host)
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


def oracle_weights_for(score: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """The oracle's normalised weights for a given choice of experts: its FP64 sigmoid scores of those
    experts divided by their sum (the normalisation step, applied to another expert set)."""
    s = np.take_along_axis(score, ids.astype(np.int64), 1)
    return s / s.sum(1, keepdims=True)


def oracle_y_checked(route: dict, st: dict, ids_gpu: np.ndarray, tokens: np.ndarray, y_oracle_route: np.ndarray,
                     y_of) -> np.ndarray:
    """Oracle outputs for `tokens` to compare with a GPU forward pass: the oracle's own outputs
    (y_oracle_route, rows aligned with tokens) where the GPU chose the oracle's expert set, and, for
    excluded tokens where it chose another valid set, the oracle recomputed on the GPU's ids with
    the oracle's weights for them.  y_of(ids, w, tokens) runs the oracle's expert half."""
    y = np.array(y_oracle_route, copy=True)
    diff = np.nonzero(~st["set_equal"][tokens])[0]
    if diff.size:
        tk = tokens[diff]
        ids = np.zeros_like(route["ids"])
        w = np.zeros_like(route["weight"])
        ids[tk] = ids_gpu[tk]
        w[tk] = oracle_weights_for(route["score"][tk], ids_gpu[tk])
        y[diff] = y_of(ids, w, tk)
    return y


def bf16_interval(y_gpu: np.ndarray):
    """Lower and upper ends of the set of real values that round (to nearest) to each BF16 value:
    the value +- half the spacing to its lower / upper BF16 neighbour."""
    b = oracle.f64_to_bf16_bits(y_gpu).astype(np.int32)  # exact: y_gpu already holds BF16 values
    mag = b & 0x7FFF
    sign = np.where(b & 0x8000, -1.0, 1.0)
    up = oracle.bf16_bits_to_f64(np.minimum(mag + 1, 0x7F7F).astype(np.uint16))
    dn = oracle.bf16_bits_to_f64(np.maximum(mag - 1, 0).astype(np.uint16))
    a = oracle.bf16_bits_to_f64(mag.astype(np.uint16))
    half_up = (up - a) / 2
    half_dn = np.where(mag == 0, half_up, (a - dn) / 2)
    lo_mag, hi_mag = a - half_dn, a + half_up
    lo = np.where(sign > 0, lo_mag, -hi_mag)
    hi = np.where(sign > 0, hi_mag, -lo_mag)
    return lo, hi


def half_ulp_bf16(y: np.ndarray) -> np.ndarray:
    """Half a BF16 unit in the last place at |y| (8 significant bits): 2^(floor(log2|y|) - 8)."""
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def compare_y(y_gpu: np.ndarray, y_or: np.ndarray, what: str = "y", slack=None) -> dict:
    """slack (optional, same shape): per element, the output change the oracle allows for quantisation
    decisions it finds within its tolerance of a rounding boundary (the 4-bit path's h); added to the
    bound of both rules, its largest ratio to the token's RMS reported."""
    y_gpu = y_gpu.astype(np.float64)
    if y_or.size == 0:
        return dict(max_err=0.0, rms=0.0, rel=0.0, rel_row=0.0, rel_dist_row=0.0, rel_dist=0.0, rel_vs_bf16=0.0,
                    n_over_vs_bf16=0, n_one_step=0, n_elements=0)
    err = np.abs(y_gpu - y_or)
    rms = float(np.sqrt(np.mean(y_or ** 2)))
    row_rms = np.sqrt(np.mean(y_or ** 2, axis=1, keepdims=True))
    tol = Y_TOL * row_rms + (0.0 if slack is None else slack)
    assert np.all(row_rms > 0), f"{what}: a token's output is exactly zero"
    # literal bound per token, wherever BF16 rounding alone takes at most a quarter of it
    fine = half_ulp_bf16(y_or) <= 0.25 * tol
    ratio_fine = np.where(fine, err / tol, 0.0)
    worst = float(ratio_fine.max())
    t_w = int(np.unravel_index(np.argmax(ratio_fine), err.shape)[0])
    assert worst <= 1.0, (f"{what}: token {t_w}: max |err| {worst * Y_TOL:.4g} x its RMS > {Y_TOL} on the elements "
                          f"with fine BF16 spacing")
    # everywhere: distance from y_oracle to the BF16 rounding interval of y_gpu, per token
    lo, hi = bf16_interval(y_gpu)
    dist = np.maximum(0.0, np.maximum(lo - y_or, y_or - hi))
    dist_ratio = float((dist / tol).max())
    assert dist_ratio <= 1.0, (f"{what}: y_oracle lies {dist_ratio * Y_TOL:.4g} x the token's RMS from the BF16 "
                               f"rounding interval of y_gpu (> {Y_TOL})")
    # reported: the whole-output quantities and the comparison against the oracle rounded to BF16
    yb = oracle.bf16_bits_to_f64(oracle.f64_to_bf16_bits(y_or))
    eb = np.abs(y_gpu - yb)
    over = eb > Y_TOL * rms
    bg = oracle.f64_to_bf16_bits(y_gpu).astype(np.int32)
    bo = oracle.f64_to_bf16_bits(y_or).astype(np.int32)
    one_step = over & (np.abs(bg - bo) == 1)
    extra = {} if slack is None else dict(slack_row=float((slack / row_rms).max()), n_slack=int((slack > 0).sum()))
    return dict(**extra, max_err=float(err.max()), rms=rms, rel=float(err.max()) / rms,
                rel_row=float((err / (Y_TOL * row_rms)).max()) * Y_TOL,
                rel_fine_row=worst * Y_TOL, rel_dist_row=dist_ratio * Y_TOL, rel_dist=float(dist.max()) / rms,
                rel_vs_bf16=float(eb.max()) / rms, n_over_vs_bf16=int(over.sum()), n_one_step=int(one_step.sum()),
                n_elements=int(y_or.size))

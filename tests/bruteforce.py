"""Brute-force statement of group-limited routing, used only to pin the oracle.

It reads the method as an optimisation over subsets instead of a sequence of sorts:
  * a group's score is the largest sum over all group_topn-subsets of the group's selection values;
  * the kept groups are the topk_groups-subset of groups with the largest total group score;
  * the experts are the topk-subset of the kept groups' experts with the largest total value;
  * slots list the chosen experts by descending value (lower index first on ties).
With continuous random inputs (no ties) this equals the sort-based description on the Beam
launch pages ('Welcome Beam' page, section 'Mixture of Experts'); enumerating every subset makes
the equivalence a check rather than an assumption.  Pure Python: tiny inputs only.
"""
from __future__ import annotations

import itertools
import math

import numpy as np


def sigmoid64(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def route_token(sel: np.ndarray, score: np.ndarray, E: int, G: int, topk_groups: int, topk: int, group_topn: int):
    per = E // G
    gscore = []
    for g in range(G):
        vals = sel[g * per:(g + 1) * per]
        gscore.append(max(sum(c) for c in itertools.combinations(vals.tolist(), group_topn)))
    best_groups = max(itertools.combinations(range(G), topk_groups), key=lambda s: sum(gscore[g] for g in s))
    cand = [e for g in best_groups for e in range(g * per, (g + 1) * per)]
    best = max(itertools.combinations(cand, topk), key=lambda s: sum(sel[e] for e in s))
    ids = sorted(best, key=lambda e: (-sel[e], e))
    den = sum(score[e] for e in ids)
    w = [score[e] / den for e in ids]
    return ids, w, sorted(best_groups)


def route(x: np.ndarray, w_router: np.ndarray, E: int, G: int, topk_groups: int, topk: int, group_topn: int,
          bias=None):
    """x [T,H] float64 (already exact bf16 values), w_router [E,H]; returns ids [T,k], w [T,k], groups."""
    logits = x.astype(np.float64) @ w_router.astype(np.float64).T
    score = sigmoid64(logits)
    sel = score + (0.0 if bias is None else np.asarray(bias, dtype=np.float64)[None, :])
    out_ids, out_w, out_g = [], [], []
    for t in range(x.shape[0]):
        ids, w, g = route_token(sel[t], score[t], E, G, topk_groups, topk, group_topn)
        out_ids.append(ids)
        out_w.append(w)
        out_g.append(g)
    return np.array(out_ids, dtype=np.int64), np.array(out_w), out_g


def n_subsets(E: int, G: int, topk_groups: int, topk: int) -> int:
    return math.comb(G, topk_groups) * math.comb(topk_groups * E // G, topk)


def margins(sel: np.ndarray, E: int, G: int, topk_groups: int, topk: int, group_topn: int):
    """The decision margins of one token stated as smallest gaps between what was chosen and what was
    not: the smallest kept-minus-dropped group score, the smallest chosen-minus-unchosen value among
    the kept groups' experts, and the smallest gap between consecutive slots (inf where nothing is
    compared).  Group scores by subset enumeration."""
    per = E // G
    gscore = [max(sum(c) for c in itertools.combinations(sel[g * per:(g + 1) * per].tolist(), group_topn))
              for g in range(G)]
    ids, _, kept = route_token(sel, sel, E, G, topk_groups, topk, group_topn)
    dropped = [g for g in range(G) if g not in kept]
    m_group = min((gscore[a] - gscore[b] for a in kept for b in dropped), default=math.inf)
    cand = [e for g in kept for e in range(g * per, (g + 1) * per)]
    m_expert = min((sel[a] - sel[b] for a in ids for b in cand if b not in ids), default=math.inf)
    m_order = min((sel[ids[j]] - sel[ids[j + 1]] for j in range(topk - 1)), default=math.inf)
    return m_group, m_expert, m_order

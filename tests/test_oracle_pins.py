"""Pins of the CPU oracle against facts that do not come from the oracle itself.

The Beam pages print no worked numeric example of the layer, so the oracle is pinned by:
  * brute-force enumeration of every group / expert subset on tiny inputs (tests/bruteforce.py);
  * hand-derived cases with closed-form sigmoid values (tests/golden/hand_routing_cases.json);
  * special cases that reduce to library routines (plain top-k, a single SwiGLU expert in torch
    float64, a stable argsort for the dispatch order);
  * invariants and metamorphic relations (permutation equivariance, exact power-of-two scaling,
    group relabelling).
A separate test (test_oracle_mutants.py) plants mistakes in copies of the oracle and checks that
these pins catch each one.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import beam_synth as bs
import oracle
from tests import bruteforce

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny_inputs(seed: int, T: int = 64, wl_name: str = "tiny"):
    wl = bs.get(wl_name)
    wl = bs.Workload(**{**wl.__dict__, "seed": seed, "T": T})
    x = bs.make_x(wl)
    W = bs.make_router(wl)
    return wl, x, W


@pytest.mark.parametrize("with_bias", [False, True])
def test_bruteforce_tiny(with_bias):
    """Sort-based oracle == subset enumeration on the tiny layer (E=16, G=4, keep 2, k=4), 20 seeds."""
    rng = np.random.default_rng(7)
    n_cmp = 0
    for seed in range(100, 120):
        wl, x, W = tiny_inputs(seed)
        L = wl.layer
        bias = rng.normal(0, 0.05, size=wl.n_experts).astype(np.float32) if with_bias else None
        xb = oracle.bf16_bits(x)
        r = oracle.route(xb, W.numpy(), L, bias)
        ids_bf, w_bf, groups_bf = bruteforce.route(oracle.bf16_bits_to_f64(xb), W.numpy(), L["n_experts"],
                                                   L["n_groups"], L["topk_groups"], L["topk"], L["group_topn"],
                                                   bias)
        np.testing.assert_array_equal(r["ids64"], ids_bf)
        np.testing.assert_allclose(r["weight"][r["ids"] == r["ids64"]].ravel(),
                                   w_bf[r["ids"] == r["ids64"]].ravel(), rtol=0, atol=1e-12)
        clear = np.all(r["margin"] >= 1e-6, axis=1)
        np.testing.assert_array_equal(r["ids"][clear], ids_bf[clear])
        n_cmp += int(clear.sum())
    assert n_cmp > 0.9 * 20 * 64



@pytest.mark.parametrize("with_bias", [False, True])
def test_margins_are_the_smallest_chosen_minus_unchosen_gaps(with_bias):
    """The FP64 decision margins (group, expert, slot order) equal the smallest gaps between what was
    chosen and what was not, found by subset enumeration on the tiny layer; a margin that compares
    the wrong ranks or the wrong sets would let near-ties through the bit-exact checks."""
    rng = np.random.default_rng(8)
    for seed in range(130, 140):
        wl, x, W = tiny_inputs(seed)
        L = wl.layer
        bias = rng.normal(0, 0.05, size=wl.n_experts).astype(np.float32) if with_bias else None
        xb = oracle.bf16_bits(x)
        r = oracle.route(xb, W.numpy(), L, bias)
        score = bruteforce.sigmoid64(oracle.bf16_bits_to_f64(xb) @ W.numpy().astype(np.float64).T)
        sel = score + (0.0 if bias is None else bias.astype(np.float64)[None, :])
        want = np.array([bruteforce.margins(sel[t], L["n_experts"], L["n_groups"], L["topk_groups"], L["topk"],
                                            L["group_topn"]) for t in range(wl.T)])
        np.testing.assert_allclose(r["margin"], want, rtol=0, atol=1e-12)



@pytest.mark.parametrize("E,G,kg,k,gn", [
    (16, 4, 2, 4, 1), (16, 4, 2, 4, 3), (16, 4, 3, 6, 4), (16, 8, 3, 5, 2), (12, 3, 1, 3, 2),
    (24, 6, 4, 7, 3), (16, 2, 1, 8, 8), (16, 4, 4, 4, 2)])
def test_select_matches_bruteforce_across_layouts(E, G, kg, k, gn):
    """The selection step on scores drawn directly (continuous, so no ties) for layouts other than
    Beam's: group sizes 2-8, one to all groups kept, group scores over the top 1 to 8 members, k from
    3 to 8 -- against subset enumeration, with and without a selection bias."""
    rng = np.random.default_rng(E * 1000 + G * 100 + kg * 10 + k + gn)
    L = dict(n_experts=E, n_groups=G, topk_groups=kg, topk=k, group_topn=gn)
    for with_bias in (False, True):
        score = rng.uniform(0.01, 0.99, (24, E))
        bias = rng.normal(0, 0.1, E).astype(np.float32) if with_bias else None
        r = oracle.select(score, L, bias)
        sel = score + (0.0 if bias is None else bias.astype(np.float64)[None, :])
        for t in range(score.shape[0]):
            ids, w, _ = bruteforce.route_token(sel[t], score[t], E, G, kg, k, gn)
            assert r["ids64"][t].tolist() == ids
            if np.all(r["margin"][t] >= 1e-6):
                assert r["ids"][t].tolist() == ids
                np.testing.assert_allclose(r["weight"][t], w, rtol=0, atol=1e-12)


def test_hand_cases():
    with open(os.path.join(GOLDEN, "hand_routing_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        E = c["E"]
        x = torch.ones(1, 1, dtype=torch.bfloat16)
        W = np.array(c["logits"], dtype=np.float32).reshape(E, 1)
        layer = dict(n_experts=E, n_groups=c["G"], topk_groups=c["topk_groups"], topk=c["topk"],
                     group_topn=c["group_topn"])
        bias = None if c["bias"] is None else np.array(c["bias"], dtype=np.float32)
        r = oracle.route(oracle.bf16_bits(x), W, layer, bias)
        assert r["ids"][0].tolist() == c["expected_ids"], c["name"]
        assert r["ids64"][0].tolist() == c["expected_ids"], c["name"]
        s = [1.0 / (1.0 + math.exp(-c["logits"][e])) for e in c["expected_ids"]]
        w = [v / sum(s) for v in s]
        np.testing.assert_allclose(r["weight"][0], w, rtol=0, atol=1e-15, err_msg=c["name"])


def test_invariants_beam_groups():
    """k distinct ids, all inside <= topk_groups groups, weights sum to 1 (Beam group structure)."""
    wl = bs.Workload("inv", T=300, hidden=256, inter=64, n_experts=256, n_groups=8, topk_groups=4, topk=8, seed=31)
    x, W = bs.make_x(wl), bs.make_router(wl)
    r = oracle.route(oracle.bf16_bits(x), W.numpy(), wl.layer)
    ids, w = r["ids"], r["weight"]
    assert ids.shape == (300, 8)
    for t in range(300):
        assert len(set(ids[t].tolist())) == 8
        groups = set((ids[t] // 32).tolist())
        assert len(groups) <= 4
        # the kept groups are the 4 best by top-2 sum; every chosen expert's group is among them
        sc = r["score"][t]
        gs = [np.sort(sc[g * 32:(g + 1) * 32])[-2:].sum() for g in range(8)]
        best4 = set(np.argsort(-np.array(gs), kind="stable")[:4].tolist())
        assert groups <= best4
        # slot order: descending score
        assert np.all(np.diff(sc[ids[t]]) <= 0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(w > 0)


def test_all_groups_kept_is_plain_topk():
    """topk_groups = n_groups reduces to sigmoid top-k (torch.topk in float64 as the library check)."""
    wl = bs.Workload("pt", T=200, hidden=128, inter=64, n_experts=64, n_groups=8, topk_groups=8, topk=6, seed=32)
    x, W = bs.make_x(wl), bs.make_router(wl)
    r = oracle.route(oracle.bf16_bits(x), W.numpy(), wl.layer)
    xs = torch.from_numpy(oracle.bf16_bits_to_f64(oracle.bf16_bits(x)))
    sc = torch.sigmoid(xs @ W.double().T)
    top = torch.topk(sc, 6, dim=1).indices.numpy()
    np.testing.assert_array_equal(r["ids64"], top)
    np.testing.assert_allclose(r["score"], sc.numpy(), rtol=1e-15, atol=1e-15)


def _expert_fetch(wg, wu, wd):
    return lambda e: (oracle.bf16_bits(wg[e]), oracle.bf16_bits(wu[e]), oracle.bf16_bits(wd[e]))


def _torch_expert(x64, wg, wu, wd):
    g = x64 @ wg.double().T
    u = x64 @ wu.double().T
    return (torch.nn.functional.silu(g) * u) @ wd.double().T


def test_single_expert_matches_torch_float64():
    wl = bs.get("mid_c")
    x = bs.make_x(wl, T=9)
    wg, wu, wd = bs.make_expert(wl, 3, "cpu")
    out = oracle.expert_mlp(oracle.bf16_bits(x), oracle.bf16_bits(wg), oracle.bf16_bits(wu), oracle.bf16_bits(wd))
    ref = _torch_expert(x.double(), wg, wu, wd).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_k1_is_scaled_single_expert():
    """With one routed expert the normalised weight is 1 and y = routed_scale * E_e(x)."""
    wl = bs.Workload("k1", T=20, hidden=128, inter=64, n_experts=16, n_groups=4, topk_groups=2, topk=1,
                     routed_scale=2.5, seed=33)
    x, W = bs.make_x(wl), bs.make_router(wl)
    wg, wu, wd = bs.make_experts(wl, "cpu")
    f = oracle.forward(oracle.bf16_bits(x), W.numpy(), None, _expert_fetch(wg, wu, wd), wl.layer)
    np.testing.assert_array_equal(f["route"]["weight"], 1.0)
    x64 = x.double()
    for t in range(wl.T):
        e = int(f["route"]["ids"][t, 0])
        ref = 2.5 * _torch_expert(x64[t:t + 1], wg[e], wu[e], wd[e]).numpy()[0]
        np.testing.assert_allclose(f["y"][t], ref, rtol=1e-12, atol=1e-12)


def test_forward_matches_torch_float64_composition():
    """Whole block on mid_a == torch float64 composition of the pinned pieces (ids from brute force)."""
    wl = bs.get("mid_a").with_T(40)
    x, W = bs.make_x(wl), bs.make_router(wl)
    wg, wu, wd = bs.make_experts(wl, "cpu")
    L = wl.layer
    f = oracle.forward(oracle.bf16_bits(x), W.numpy(), None, _expert_fetch(wg, wu, wd), L)
    x64 = x.double()
    ids_bf, w_bf, _ = bruteforce.route(x64.numpy(), W.numpy(), L["n_experts"], L["n_groups"], L["topk_groups"],
                                       L["topk"], L["group_topn"])
    np.testing.assert_array_equal(f["route"]["ids"], ids_bf)
    y = np.zeros((wl.T, wl.hidden))
    for t in range(wl.T):
        for j in range(wl.topk):
            e = ids_bf[t, j]
            y[t] += w_bf[t, j] * _torch_expert(x64[t:t + 1], wg[e], wu[e], wd[e]).numpy()[0]
    np.testing.assert_allclose(f["y"], L["routed_scale"] * y, rtol=1e-10, atol=1e-12)


def test_token_permutation_equivariance():
    wl = bs.get("mid_a").with_T(50)
    x, W = bs.make_x(wl), bs.make_router(wl)
    wg, wu, wd = bs.make_experts(wl, "cpu")
    fetch = _expert_fetch(wg, wu, wd)
    p = np.random.default_rng(3).permutation(wl.T)
    a = oracle.forward(oracle.bf16_bits(x), W.numpy(), None, fetch, wl.layer)
    b = oracle.forward(oracle.bf16_bits(x[torch.from_numpy(p)]), W.numpy(), None, fetch, wl.layer)
    np.testing.assert_array_equal(a["route"]["ids"][p], b["route"]["ids"])
    np.testing.assert_allclose(a["y"][p], b["y"], rtol=1e-13, atol=1e-13)


def test_down_projection_scaling_is_exact():
    """Scaling W_down by 2 (exact in bf16) scales y by exactly 2; scaling W_up by 2 does too."""
    wl = bs.get("mid_a").with_T(30)
    x, W = bs.make_x(wl), bs.make_router(wl)
    wg, wu, wd = bs.make_experts(wl, "cpu")
    xb = oracle.bf16_bits(x)
    a = oracle.forward(xb, W.numpy(), None, _expert_fetch(wg, wu, wd), wl.layer)["y"]
    b = oracle.forward(xb, W.numpy(), None, _expert_fetch(wg, wu, wd * 2), wl.layer)["y"]
    c = oracle.forward(xb, W.numpy(), None, _expert_fetch(wg, wu * 2, wd), wl.layer)["y"]
    np.testing.assert_array_equal(b, 2 * a)
    np.testing.assert_allclose(c, 2 * a, rtol=1e-14, atol=0)


def test_group_relabelling_permutes_ids():
    """Swapping whole expert groups in W_r relabels the chosen ids the same way."""
    wl = bs.Workload("rl", T=120, hidden=128, inter=64, n_experts=64, n_groups=8, topk_groups=4, topk=8, seed=34)
    x, W = bs.make_x(wl), bs.make_router(wl)
    per = 8
    gperm = np.array([3, 0, 7, 5, 1, 2, 6, 4])
    eperm = np.concatenate([np.arange(g * per, (g + 1) * per) for g in gperm])  # new expert i = old eperm[i]
    a = oracle.route(oracle.bf16_bits(x), W.numpy(), wl.layer)
    b = oracle.route(oracle.bf16_bits(x), np.ascontiguousarray(W.numpy()[eperm]), wl.layer)
    inv = np.empty_like(eperm)
    inv[eperm] = np.arange(len(eperm))
    clear = np.all(a["margin"] >= 1e-6, axis=1)
    np.testing.assert_array_equal(inv[a["ids"]][clear], b["ids"][clear])


def test_permute_matches_stable_argsort():
    rng = np.random.default_rng(5)
    for T, k, E in ((1, 1, 1), (7, 3, 5), (300, 8, 64), (1000, 4, 16)):
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        p = oracle.permute(ids, E)
        np.testing.assert_array_equal(p["counts"], np.bincount(ids.ravel(), minlength=E))
        np.testing.assert_array_equal(p["offsets"], np.concatenate([[0], np.cumsum(np.bincount(ids.ravel(), minlength=E))]))
        order = np.argsort(ids.ravel(), kind="stable")
        np.testing.assert_array_equal(p["row_src"], order)
        np.testing.assert_array_equal(p["dest_row"][p["row_src"]], np.arange(T * k))
        # within an expert, tokens increase
        tok = p["row_src"] // k
        for e in range(E):
            seg = tok[p["offsets"][e]:p["offsets"][e + 1]]
            assert np.all(np.diff(seg) > 0)


def test_permute_empty_and_bad_ids():
    p = oracle.permute(np.zeros((0, 8), dtype=np.int32), 256)
    assert p["offsets"][-1] == 0 and p["counts"].sum() == 0
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 9]], dtype=np.int32), 8)


def test_combine_weighted_sum():
    rng = np.random.default_rng(9)
    out = rng.normal(size=(5, 3, 7))
    w = rng.random((5, 3))
    y = oracle.combine(out, w, 2.5)
    np.testing.assert_allclose(y, 2.5 * np.einsum("tj,tjh->th", w, out), rtol=1e-14, atol=1e-14)


def test_select_rejects_bad_configs():
    sc = np.full((2, 16), 0.5)
    for bad in (dict(n_groups=3), dict(topk_groups=5), dict(group_topn=5), dict(topk=9)):
        L = dict(n_experts=16, n_groups=4, topk_groups=2, topk=4, group_topn=2)
        L.update(bad)
        with pytest.raises(ValueError):
            oracle.select(sc, L)


def test_saturated_scores_tie_to_lower_index():
    """Scores that round to 1.0 in FP32 tie; the FP32 decision takes the lowest indices."""
    E = 16
    W = np.zeros((E, 1), dtype=np.float32)
    W[[3, 6, 9, 12, 13], 0] = [40.0, 35.0, 30.0, 25.0, 45.0]   # all sigmoid -> 1.0f
    x = torch.ones(1, 1, dtype=torch.bfloat16)
    L = dict(n_experts=E, n_groups=4, topk_groups=2, topk=2, group_topn=2)
    r = oracle.route(oracle.bf16_bits(x), W, L)
    # FP32: groups 0..3 top-2 sums: g0 = 1+0.5, g1 = 1+0.5, g2 = 1+0.5, g3 = 1+1 -> keep g3, then g0 (tie, lower)
    assert r["ids"][0].tolist() == [3, 12]
    # FP64: sigmoid(40) and sigmoid(45) are 1.0 exactly, sigmoid(25) = 1 - 1.4e-11: groups g3, g0 again,
    # experts e3 and e13 tie at 1.0 (lower index first), e12 is third.
    assert r["ids64"][0].tolist() == [3, 13]
    assert r["margin"][0, 1] < 1e-6   # the expert margin flags the near-tie
    assert r["margin"][0, 2] < 1e-6   # the order margin flags the exact tie

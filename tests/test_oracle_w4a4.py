"""Pins of the oracle's NVFP4 activations (4-bit path), checked against an exhaustive nearest search on
the E2M1 grid, torch's float8 E4M3 cast and a torch float64 composition, none of it the oracle's code.

Reading (the pages give no recipe): activations are quantised per row with a power-of-two row scale g
(the smallest bringing the row's largest magnitude to at most 6 x 448; 1 for h), one E4M3 scale per
16 elements (the nearest E4M3 value to amax / (6 g)) and E2M1 elements (nearest, ties to even,
saturating at 6).
"""
import numpy as np
import torch

import oracle

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _nearest_e2m1(m: np.ndarray) -> np.ndarray:
    """Nearest grid value by exhaustive search; ties to the even code (index)."""
    d = np.abs(m[..., None] - E2M1)
    best = d.min(-1, keepdims=True)
    cand = np.where(d == best, np.arange(8), 99)
    idx = np.where((cand % 2 == 0) & (cand < 99), cand, 99).min(-1)        # an even tie winner if any
    idx = np.where(idx == 99, cand.min(-1), idx)
    return E2M1[idx]


def _ref_quant(v: np.ndarray, per_row: bool):
    rows, K = v.shape
    amax_row = np.abs(v).max(1)
    g = np.ones(rows)
    if per_row:
        e = np.floor(np.log2(np.maximum(amax_row, 1e-300) / 2688.0)) - 2
        for _ in range(6):
            e = np.where(amax_row > 2688.0 * np.exp2(e), e + 1, e)
        g = np.where(amax_row > 0, np.exp2(e), 1.0)
    blk = v.reshape(rows, K // 16, 16)
    a = np.minimum(np.abs(blk).max(-1) / (6 * g[:, None]), 448.0)
    s = torch.from_numpy(a).to(torch.float8_e4m3fn).double().numpy()
    with np.errstate(divide="ignore", invalid="ignore"):
        m = np.where(s[..., None] > 0, np.abs(blk) / (s[..., None] * g[:, None, None]), 0.0)
    q = np.sign(blk) * _nearest_e2m1(np.minimum(m, 6.0))
    return (q * s[..., None] * g[:, None, None]).reshape(rows, K), g


def _rows(seed, rows=12, K=256):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, K)) * np.exp(rng.standard_normal((rows, 1)) * 3)
    v[0, :16] = 0.0
    v[1, 16:32] *= 1e-5
    v[2, :] = np.round(v[2, :] * 4) / 4   # values on quarter steps: E2M1 ties after scaling
    return v


def test_nvfp4_rows_match_exhaustive_search_and_torch_e4m3():
    for seed in range(4):
        v = _rows(seed)
        for per_row in (True, False):
            q, sc, g, deq = oracle.quant_nvfp4_rows(v, per_row)
            ref, gref = _ref_quant(v, per_row)
            np.testing.assert_array_equal(g, gref)
            np.testing.assert_array_equal(deq, ref)
            if per_row:
                top = np.abs(v).max(1) / g
                assert np.all(top <= 2688.0) and np.all(top[np.abs(v).max(1) > 0] > 1344.0)


def test_codes_decode_to_the_dequantised_values():
    v = _rows(9)
    q, sc, g, deq = oracle.quant_nvfp4_rows(v, True)
    mag = E2M1[q & 7] * np.where(q & 8, -1.0, 1.0)
    s = torch.from_numpy(sc.view(np.int8)).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(mag * s.repeat(16, axis=1) * g[:, None], deq)


def test_expert_w4a4_matches_torch_float64_composition():
    """Two weight scales: O(1) intermediate values, and ~1e-4 ones whose 16-blocks fall below E4M3's
    normal range under the row scale 1 that h uses (where a per-row power of two would differ)."""
    rng = np.random.default_rng(11)
    n, H, I = 7, 256, 128
    x = torch.from_numpy(rng.standard_normal((n, H))).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    for scale in (1.0, 1e-2):
        wg, wu = (rng.standard_normal((I, H)) / 16 * scale for _ in range(2))
        wd = rng.standard_normal((H, I)) / 11
        got = oracle.expert_mlp_w4a4(bits, wg, wu, wd)
        xq, _ = _ref_quant(x.double().numpy(), True)
        g = xq @ wg.T
        u = xq @ wu.T
        h = torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u
        hq, _ = _ref_quant(h, False)
        ref = hq @ wd.T
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_alternative_quantisation_envelope():
    """alt: 0 without tolerance; one E2M1 step at an element exactly on a rounding midpoint; the other
    scale's dequantisation for a block whose amax/6 sits on an E4M3 midpoint; 0 far from boundaries."""
    v = np.zeros((3, 16))
    v[0, 0], v[0, 1], v[0, 2] = 6.0, 2.5, 1.1                  # scale 1: 2.5 is the midpoint of 2 and 3
    v[1, 0], v[1, 1] = 6.0 * 1.0625, 1.0                        # amax / 6 = 1.0625: E4M3 midpoint of 1 and 1.125
    v[2, 0], v[2, 1] = 6.0, 1.1                                 # nothing near a boundary
    assert np.all(oracle.quant_nvfp4_rows_alt(v, False, 0.0) == 0.0)
    alt = oracle.quant_nvfp4_rows_alt(v, False, 1e-6)
    assert alt[0, 1] == 1.0 and alt[0, 2] == 0.0 and alt[0, 0] == 0.0
    _, _, _, deq = oracle.quant_nvfp4_rows(v[1:2], False)
    s_other = 1.125 if deq[0, 0] == 6.0 else 1.0                 # the scale not taken
    q_other = _nearest_e2m1(np.minimum(np.abs(v[1]) / s_other, 6.0)) * s_other
    np.testing.assert_allclose(alt[1], np.abs(q_other - deq[0]), rtol=0, atol=0)
    assert np.all(alt[2] == 0.0)


def _boundary_rows(seed, rows=48, K=64, eps=1e-3):
    """Rows whose 16-blocks sit on or near the quantiser's decision boundaries: a third of the blocks
    have amax / 6 exactly on an E4M3 midpoint (the scale can round either way), a third within eps / 4
    of one; elements on E2M1 midpoints under the block's scale or under the neighbouring scale, near
    them, or uniform.  Returns the rows and each block's E4M3 scale (torch's cast)."""
    rng = np.random.default_rng(seed)
    codes = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    grid = np.unique(codes[(codes >= 0.5) & (codes <= 4.0)])
    mids = (E2M1[1:] + E2M1[:-1]) / 2
    v = np.zeros((rows, K))
    for r in range(rows):
        for b in range(K // 16):
            kind = (r * (K // 16) + b) % 3
            j = rng.integers(0, len(grid) - 1)
            mid = (grid[j] + grid[j + 1]) / 2
            a = (mid, mid * (1 + rng.choice([-1, 1]) * eps / 4), rng.uniform(0.5, 4.0))[kind]
            s = torch.tensor(a).to(torch.float8_e4m3fn).double().item()
            other = (grid[j + 1] if s == grid[j] else grid[j]) if kind < 2 else s
            m = np.stack([rng.choice(mids, 16) * s, rng.choice(mids, 16) * other,
                          rng.choice(mids, 16) * s * (1 + rng.uniform(-2, 2, 16) * eps), rng.uniform(0, 6 * a, 16)])
            blk = m[rng.integers(0, 4, 16), np.arange(16)] * rng.choice([-1, 1], 16)
            blk[rng.integers(0, 16)] = 6 * a * rng.choice([-1, 1])
            v[r, b * 16:(b + 1) * 16] = blk
    amax = np.abs(v).reshape(rows, K // 16, 16).max(-1)
    return v, torch.from_numpy(amax / 6).to(torch.float8_e4m3fn).double().numpy()


def test_envelope_bounds_every_perturbed_quantisation():
    """alt as a bound: quantising v + d, with every |d| at most half the tolerance (eps / 2 of the
    block's largest element 6 s), changes no dequantised element by more than alt(v, eps) — on rows
    built to sit on the decision boundaries, where the block scale and the codes do flip, alone and
    together.  The perturbed quantisation is this file's own (exhaustive E2M1 search, torch's E4M3)."""
    eps = 1e-3
    v, s_blk = _boundary_rows(5, eps=eps)
    alt = oracle.quant_nvfp4_rows_alt(v, False, eps)
    deq0, _ = _ref_quant(v, False)
    np.testing.assert_array_equal(oracle.quant_nvfp4_rows(v, False)[3], deq0)
    budget = np.repeat((eps / 2) * 6 * s_blk, 16, axis=1)
    rng = np.random.default_rng(6)
    changed = scale_flips = 0
    for _ in range(150):
        w = v + rng.uniform(-1, 1, v.shape) * budget
        deq1, _ = _ref_quant(w, False)
        diff = np.abs(deq1 - deq0)
        assert np.all(diff <= alt), f"{int((diff > alt).sum())} elements moved beyond the envelope"
        changed += int((diff > 0).sum())
        s1 = torch.from_numpy(np.abs(w).reshape(s_blk.shape + (16,)).max(-1) / 6).to(torch.float8_e4m3fn)
        scale_flips += int((s1.double().numpy() != s_blk).sum())
    assert changed > 10_000 and scale_flips > 1_000   # the boundaries were really crossed


def test_expert_envelope_bounds_a_perturbed_h():
    """The expert's envelope env = |W_d| alt(h): perturb h (computed here by a torch float64
    composition) by at most half the tolerance per element, quantise it with this file's quantiser,
    project, and the output moves by no more than env.  eps = 1e-2 so that many decisions flip."""
    rng = np.random.default_rng(12)
    n, H, I, eps = 7, 256, 128, 1e-2
    x = torch.from_numpy(rng.standard_normal((n, H))).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    wg, wu = (rng.standard_normal((I, H)) / 16 for _ in range(2))
    wd = rng.standard_normal((H, I)) / 11
    out, env = oracle.expert_mlp_w4a4(bits, wg, wu, wd, eps=eps)
    xq, _ = _ref_quant(x.double().numpy(), True)
    h = torch.nn.functional.silu(torch.from_numpy(xq @ wg.T)).numpy() * (xq @ wu.T)
    hq, _ = _ref_quant(h, False)
    np.testing.assert_allclose(out, hq @ wd.T, rtol=1e-12, atol=1e-12 * np.abs(out).max())
    s_blk = torch.from_numpy(np.abs(h).reshape(n, I // 16, 16).max(-1) / 6).to(torch.float8_e4m3fn)
    budget = np.repeat((eps / 2) * 6 * s_blk.double().numpy(), 16, axis=1)
    slack = 1e-12 * (np.abs(hq) @ np.abs(wd).T).max()    # rounding of the two FP64 projections
    moved = 0
    for _ in range(40):
        hq1, _ = _ref_quant(h + rng.uniform(-1, 1, h.shape) * budget, False)
        moved += int((hq1 != hq).sum())
        assert np.all(np.abs(hq1 @ wd.T - out) <= env + slack)
    assert moved > 100

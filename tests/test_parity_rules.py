"""The GPU parity tests' own yardsticks, checked on the CPU: the BF16 rounding interval and half-ulp
helpers against torch's round-to-nearest-even BF16 cast; compare_y's pass rule on outputs whose
error is known (a correctly rounded oracle passes; an error planted past the per-token bound fails;
an outlier row's scale does not loosen a normal row's bound); and compare_routing's rule on
hand-made scores (planted wrong ids, slot order and weights fail; either side of a tie passes)."""
import numpy as np
import pytest
import torch

from tests import parity


def _bf16(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v).to(torch.bfloat16).double().numpy()


def _values(seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(4000) * np.exp2(rng.integers(-20, 20, 4000))
    p2 = np.exp2(rng.integers(-20, 20, 200)) * rng.choice([-1.0, 1.0], 200)
    return np.concatenate([v, p2, p2 * (1 + 2.0 ** -9), p2 * (1 - 2.0 ** -10), [0.0, 1.0, -1.0]])


def test_bf16_interval_is_exactly_the_set_that_rounds_there():
    v = _values(1)
    y = _bf16(v)
    lo, hi = parity.bf16_interval(y)
    assert np.all(lo <= v) and np.all(v <= hi)
    # just inside the ends rounds to y, just outside rounds elsewhere (torch's RNE cast decides; the
    # points sit 2^-10 of the interval's width from its ends, exact in FP32, so the cast's passage
    # through FP32 rounds nothing)
    nz = y != 0
    d = (hi - lo) * 2.0 ** -10
    inner_lo, inner_hi, outer_lo, outer_hi = lo + d, hi - d, lo - d, hi + d
    np.testing.assert_array_equal(_bf16(inner_lo)[nz], y[nz])
    np.testing.assert_array_equal(_bf16(inner_hi)[nz], y[nz])
    assert np.all(_bf16(outer_lo)[nz] != y[nz]) and np.all(_bf16(outer_hi)[nz] != y[nz])
    # at a power of two the spacing below is half the spacing above
    lo1, hi1 = parity.bf16_interval(np.array([1.0]))
    assert hi1[0] - 1.0 == 2.0 ** -8 and 1.0 - lo1[0] == 2.0 ** -9


def test_half_ulp_is_half_the_spacing_above():
    y = _bf16(_values(2))
    y = y[y != 0]
    up = np.abs(y) * (1 + 2.0 ** -7)    # at least one BF16 step above |y|
    nxt = np.array([float(torch.nextafter(torch.tensor(a, dtype=torch.bfloat16),
                                          torch.tensor(b, dtype=torch.bfloat16)))
                    for a, b in zip(np.abs(y), up)])
    np.testing.assert_array_equal(parity.half_ulp_bf16(y), (nxt - np.abs(y)) / 2)


def _rows(seed: int, T: int = 16, H: int = 512):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((T, H))
    y[3] *= 900.0     # an outlier row, as on the long batch
    return y


def test_compare_y_accepts_the_rounded_oracle():
    y_or = _rows(3)
    r = parity.compare_y(_bf16(y_or), y_or)
    assert r["rel_vs_bf16"] == 0.0 and r["n_over_vs_bf16"] == 0
    # rounding alone: at most half a BF16 step, 2^-8 of |y| at most
    assert r["rel_row"] <= (np.abs(y_or) / np.sqrt(np.mean(y_or ** 2, axis=1, keepdims=True))).max() * 2.0 ** -8


@pytest.mark.parametrize("row,scale,passes", [
    (5, 0.021, False),   # a normal row, just past 2e-2 of its own RMS
    (5, 0.015, True),
    (3, 0.021, False),   # the outlier row at its own scale
    (3, 0.5, False),     # ... and far past it
])
def test_compare_y_planted_errors(row, scale, passes):
    y_or = _rows(4)
    y_gpu = _bf16(y_or)
    rms_row = np.sqrt(np.mean(y_or[row] ** 2))
    j = int(np.argmin(np.abs(y_or[row])))          # a small element: fine BF16 spacing, literal rule
    y_gpu[row, j] = _bf16(np.array([y_or[row, j] + scale * rms_row]))[0]
    if passes:
        parity.compare_y(y_gpu, y_or)
    else:
        with pytest.raises(AssertionError):
            parity.compare_y(y_gpu, y_or)


def test_outlier_row_does_not_loosen_a_normal_row():
    """An error of 0.5 of a normal row's RMS is far below 2e-2 of the whole output's RMS (dominated
    by the x900 row) but fails the per-token rule."""
    y_or = _rows(5)
    whole = np.sqrt(np.mean(y_or ** 2))
    rms_row = np.sqrt(np.mean(y_or[7] ** 2))
    assert 0.5 * rms_row < 2e-2 * whole
    y_gpu = _bf16(y_or)
    j = int(np.argmin(np.abs(y_or[7])))
    y_gpu[7, j] = _bf16(np.array([y_or[7, j] + 0.5 * rms_row]))[0]
    with pytest.raises(AssertionError):
        parity.compare_y(y_gpu, y_or)


def test_large_elements_judged_by_their_rounding_interval():
    """At |y| ~ 6 row RMS half a BF16 step exceeds 1e-2 RMS: a correctly rounded value passes, and the
    neighbour two steps away (outside the interval by more than the bound) fails."""
    y_or = _rows(6)
    row = 9
    rms_row = np.sqrt(np.mean(y_or[row] ** 2))
    y_or[row, 0] = 6.1 * rms_row
    y_gpu = _bf16(y_or)
    parity.compare_y(y_gpu, y_or)
    step = 2 * parity.half_ulp_bf16(y_gpu[row, :1])[0]
    y_bad = y_gpu.copy()
    y_bad[row, 0] += 2 * step
    assert (y_bad[row, 0] - step / 2) - y_or[row, 0] > 2e-2 * rms_row   # y_oracle that far below the interval
    with pytest.raises(AssertionError):
        parity.compare_y(y_bad, y_or)


# ---- routing rule (compare_routing) on hand-made scores, tiny layer -------------------------------
_L = dict(n_experts=16, n_groups=4, topk_groups=2, topk=4, group_topn=2)


def _route(score: np.ndarray) -> dict:
    import oracle
    r = oracle.select(score, _L)
    r["score"] = score
    return r


def _scores(seed: int, T: int = 32) -> np.ndarray:
    return np.random.default_rng(seed).uniform(0.05, 0.95, (T, 16))


def test_routing_rule_accepts_the_oracle_and_rejects_planted_mistakes():
    sc = _scores(7)
    r = _route(sc)
    ids, w = r["ids"].copy(), r["weight"].astype(np.float32)
    out = parity.compare_routing(r, _L, ids, w)
    assert out["n_excluded"] == 0 and out["set_equal"].all()
    # another expert of a kept group in the last slot
    bad = ids.copy()
    kept = np.unique(ids[0] // 4)
    bad[0, 3] = [e for g in kept for e in range(4 * g, 4 * g + 4) if e not in ids[0]][0]
    with pytest.raises(AssertionError):
        parity.compare_routing(r, _L, bad, w)
    # two slots swapped on a token whose order is clear
    assert r["margin"][1, 2] >= parity.MARGIN
    bad = ids.copy()
    bad[1, [0, 1]] = bad[1, [1, 0]]
    with pytest.raises(AssertionError):
        parity.compare_routing(r, _L, bad, w)
    # a weight off by 1e-5
    wb = w.copy()
    wb[2, 0] += 1e-5
    wb[2, 1] -= 1e-5
    with pytest.raises(AssertionError):
        parity.compare_routing(r, _L, ids, wb)


def test_routing_rule_on_a_tie():
    """Token 0's 4th and 5th best experts tie: either is a correct choice, a clearly worse one is not."""
    sc = _scores(8, T=4)
    sc[0] = [0.90, 0.80, 0.10, 0.10, 0.95, 0.60, 0.60, 0.10, 0.20, 0.20, 0.20, 0.20, 0.30, 0.10, 0.10, 0.30]
    r = _route(sc)
    assert r["margin"][0, 1] == 0.0
    ids, w = r["ids"].copy(), r["weight"].astype(np.float32)
    assert sorted(ids[0].tolist()) == [0, 1, 4, 5]            # the tie goes to the lower index
    alt = ids.copy()
    alt[0] = [4, 0, 1, 6]                                      # the other expert of the tie
    out = parity.compare_routing(r, _L, alt, w)
    assert out["n_excluded"] == 1 and not out["set_equal"][0]
    worse = ids.copy()
    worse[0] = [4, 0, 1, 2]                                    # 0.10 instead of 0.60
    with pytest.raises(AssertionError):
        parity.compare_routing(r, _L, worse, w)

"""The whole block (beam_moe_forward) vs the CPU oracle: routing bit-exact outside near-ties, output
within 2e-2 * RMS on every token whose expert set matches the oracle's (all non-excluded tokens)."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
from tests import parity

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "mid_a", "mid_b", "mid_c", "mid_skew", "mid_big_expert", "beam_small_T"]


def _forward(case):
    y, ids, w = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd,
                           return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    return y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


def _check(case, tokens=None):
    y, ids, w = _forward(case)
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = np.arange(case.T) if tokens is None else tokens
    tok = tok[st["set_equal"][tok]]  # tokens whose expert set is the oracle's
    yo = case.oracle_y(r["ids"], r["weight"], tok)
    sy = parity.compare_y(y[tok], yo, case.wl.name)
    return st, sy, y


@pytest.mark.parametrize("name", SMALL)
def test_forward_small(name, beam_weights):
    wl = bs.get(name)
    case = parity.Case(wl, weights=beam_weights if wl.expert_device == "cuda" else None)
    st, sy, _ = _check(case)
    print(f"{name}: excluded {st['n_excluded']}, {sy}")


@pytest.mark.parametrize("name,n_sample", [("decode", 32), ("prefill", 24), ("skew", 24), ("long", 16)])
def test_forward_full_size_sampled(name, n_sample, beam_weights):
    wl = bs.get(name)
    case = parity.Case(wl, weights=beam_weights)
    tok = bs.sample_tokens(wl, n_sample, include=bs.outlier_rows(wl)[:16])
    st, sy, y = _check(case, tok)
    assert np.isfinite(y).all()
    print(f"{name}: excluded {st['n_excluded']} same-set {st['n_excluded_same_set']}: {sy}")


def test_forward_without_routing_outputs_matches(beam_weights):
    case = parity.Case(bs.get("beam_small_T"), weights=beam_weights)
    y1, _, _ = _forward(case)
    y2 = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd)
    assert np.array_equal(y1, y2.float().cpu().numpy())


def test_forward_deterministic(beam_weights):
    case = parity.Case(bs.get("prefill"), weights=beam_weights)
    a = _forward(case)
    b = _forward(case)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_forward_zero_tokens(beam_weights):
    wl = bs.get("prefill")
    x = torch.zeros(0, wl.hidden, dtype=torch.bfloat16, device="cuda")
    case = parity.Case(bs.get("beam_small_T"), weights=beam_weights)
    y = bm.forward(case.layer, x, case.w_router, None, case.wg, case.wu, case.wd)
    assert y.shape == (0, wl.hidden)
    assert bm.device_status() == bm.OK


def test_bounded_wait_reports_timeout():
    """A device wait that nothing ends gives up after ~2 ms and reports, leaving the context usable."""
    bm.selftest_timeout(2000)
    assert bm.device_status() == bm.ERR_DEVICE_TIMEOUT
    assert bm.device_status() == bm.OK
    x = torch.ones(4, device="cuda")
    assert x.sum().item() == 4.0

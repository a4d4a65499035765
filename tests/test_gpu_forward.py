"""The whole block (beam_moe_forward) vs the CPU oracle.

Routing bit-exact on every token outside near-ties (compare_routing).  Outputs (parity.compare_y) on
every token of the small cases and on the full-size token samples (all 256 decode tokens, 512 of the
prefill batch, 4096 of the skewed and of the long batch plus every outlier row): tokens whose expert
set is the oracle's against the oracle's own outputs, and excluded tokens where the GPU chose another
valid set against the oracle recomputed on the GPU's ids, so no sampled token goes unchecked."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
from tests import fullsize, parity

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "mid_a", "mid_b", "mid_c", "mid_skew", "mid_big_expert", "beam_small_T"]


def _forward(case):
    y, ids, w = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd,
                           return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    return y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name", SMALL)
def test_forward_small(name, beam_weights):
    wl = bs.get(name)
    case = parity.Case(wl, weights=beam_weights if wl.expert_device == "cuda" else None)
    y, ids, w = _forward(case)
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = np.arange(case.T)
    yo = parity.oracle_y_checked(r, st, ids, tok, case.oracle_y(r["ids"], r["weight"], tok), case.oracle_y)
    sy = parity.compare_y(y[tok], yo, name)
    print(f"{name}: excluded {st['n_excluded']} (other set {st['n_excluded'] - st['n_excluded_same_set']}), {sy}")


@pytest.mark.parametrize("name", fullsize.FULL)
def test_forward_full_size(name, bank):
    case = bank.case(name)
    y, ids, w = _forward(case)
    assert np.isfinite(y).all()
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = fullsize.sample(name)
    yo = parity.oracle_y_checked(r, st, ids, tok, bank.oracle_y("bf16", name), bank.y_of("bf16", name))
    sy = parity.compare_y(y[tok], yo, name)
    n_other = int((~st["set_equal"][tok]).sum())
    print(f"{name}: {len(tok)} tokens compared, excluded {st['n_excluded']} of {case.T} "
          f"({n_other} sampled with another valid set, recomputed on the GPU's ids): {sy}")


def test_forward_without_routing_outputs_matches(bank):
    case = bank.case("decode")
    y1, _, _ = _forward(case)
    y2 = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd)
    assert np.array_equal(y1, y2.float().cpu().numpy())


def test_forward_deterministic(bank):
    case = bank.case("prefill")
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

"""Expert half (dispatch, gate/up + SwiGLU GEMM, down GEMM, combine) vs the CPU oracle, on the
oracle's own routing, under the output protocol of tests/parity.py (compare_y)."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
from tests import fullsize, parity

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "mid_a", "mid_b", "mid_c", "mid_skew", "mid_big_expert", "beam_small_T"]


def _experts(case, ids_np, w_np):
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).cuda()
    w = torch.from_numpy(np.ascontiguousarray(w_np, dtype=np.float32)).cuda()
    y = bm.experts(case.layer, case.x, ids, w, case.wg, case.wu, case.wd)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    return y.float().cpu().numpy()


@pytest.mark.parametrize("name", SMALL)
def test_experts_small(name, beam_weights):
    wl = bs.get(name)
    case = parity.Case(wl, weights=beam_weights if wl.expert_device == "cuda" else None)
    r = case.oracle_route()
    y = _experts(case, r["ids"], r["weight"])
    tok = np.arange(wl.T)
    st = parity.compare_y(y, case.oracle_y(r["ids"], r["weight"], tok), name)
    print(f"{name}: {st}")


@pytest.mark.parametrize("name", fullsize.FULL)
def test_experts_full_size(name, bank):
    """The expert half on the oracle's routing at full size; outputs on the workload's token sample."""
    case = bank.case(name)
    r = case.oracle_route()
    y = _experts(case, r["ids"], r["weight"])
    assert np.isfinite(y).all()
    tok = fullsize.sample(name)
    st = parity.compare_y(y[tok], bank.oracle_y("bf16", name), name)
    print(f"{name}: {len(tok)} tokens: {st}")


def test_experts_k1_and_ragged_tokens():
    wl = bs.Workload("k1", T=131, hidden=256, inter=192, n_experts=16, n_groups=4, topk_groups=2, topk=1, seed=77)
    case = parity.Case(wl)
    r = case.oracle_route()
    y = _experts(case, r["ids"], r["weight"])
    parity.compare_y(y, case.oracle_y(r["ids"], r["weight"], np.arange(wl.T)), "k1")


def test_experts_deterministic(bank):
    case = bank.case("prefill")
    r = case.oracle_route()
    a = _experts(case, r["ids"], r["weight"])
    b = _experts(case, r["ids"], r["weight"])
    assert np.array_equal(a, b)

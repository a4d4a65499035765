"""Expert parallelism on one GPU with N ranks emulated phase by phase (group_limited_routing_router_b200/ep.py).

Each emulated rank owns E/N experts (views of the shared layer's weight tensors) and a contiguous slice
of the tokens; it routes its own tokens, gathers its rows in dispatch order (beam_moe_gather_rows),
runs its experts on the rows it receives (beam_moe_expert_rows) and combines the outputs that come
back (beam_moe_combine).  The exchanges are concatenations of row blocks in one process, so no
kernel waits on another rank's.  Expected: the whole batch's output bit-identical to beam_moe_forward
on one device ("Welcome Beam" page, section "Multi-GPU and multi-node": the same experts, placed on
different devices, compute the same layer).
"""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
from group_limited_routing_router_b200 import ep
from tests import parity

pytestmark = pytest.mark.gpu


def _run(case, world):
    ranks = ep.gpu_ranks(case.layer, case.w_router, case.bias, case.wg, case.wu, case.wd, world)
    T = case.T
    xs = [case.x[r * T // world:(r + 1) * T // world].contiguous() for r in range(world)]
    ys = ep.forward_emulated(ranks, xs)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    return torch.cat(ys), ranks


@pytest.mark.parametrize("name,world", [("prefill", 2), ("prefill", 8), ("decode", 8), ("skew", 4)])
def test_ep_emulated_equals_one_device_forward(name, world, bank):
    case = bank.case(name)
    y_ep, ranks = _run(case, world)
    y1 = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd)
    torch.cuda.synchronize()
    assert torch.equal(y_ep.view(torch.int16), y1.view(torch.int16))
    sent = sum(sum(r.send_splits()) for r in ranks)
    assert sent == case.T * case.layer["topk"]


@pytest.mark.parametrize("name,world", [("mid_b", 4), ("mid_skew", 2), ("tiny", 4)])
def test_ep_emulated_small_against_oracle(name, world):
    case = parity.Case(bs.get(name))
    y_ep, _ = _run(case, world)
    y1 = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd)
    torch.cuda.synchronize()
    assert torch.equal(y_ep.view(torch.int16), y1.view(torch.int16))
    r = case.oracle_route()
    tok = np.arange(case.T)
    ids, w = bm.route(case.layer, case.x, case.w_router, case.bias)
    st = parity.compare_routing(r, case.layer, ids.cpu().numpy(), w.cpu().numpy(), case.bias_np)
    yo = parity.oracle_y_checked(r, st, ids.cpu().numpy(), tok, case.oracle_y(r["ids"], r["weight"], tok),
                                 case.oracle_y)
    print(name, parity.compare_y(y_ep.float().cpu().numpy(), yo, name))


def test_expert_rows_matches_forward_rows(bank):
    """beam_moe_expert_rows on rows given in an arbitrary order: each output row is its expert's FP32
    output, the same whatever the row order (rows are shuffled, then un-shuffled)."""
    case = bank.case("decode")
    ids, w = bm.route(case.layer, case.x, case.w_router, case.bias)
    p = bm.permute(case.layer, ids)
    rows = bm.gather_rows(case.layer, case.x, p["dest_row"])
    counts = p["counts"].cpu().numpy()
    row_expert = torch.from_numpy(np.repeat(np.arange(256), counts).astype(np.int32)).cuda()
    o = bm.expert_rows(rows, row_expert, case.wg, case.wu, case.wd)
    perm = torch.randperm(rows.shape[0], generator=torch.Generator().manual_seed(3)).cuda()
    o2 = bm.expert_rows(rows[perm].contiguous(), row_expert[perm].contiguous(), case.wg, case.wu, case.wd)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    assert torch.equal(o[perm], o2)
    y = bm.combine(case.layer, o, p["dest_row"], w)
    y1 = bm.forward(case.layer, case.x, case.w_router, case.bias, case.wg, case.wu, case.wd)
    assert torch.equal(y.view(torch.int16), y1.view(torch.int16))

"""Dispatch kernels vs the CPU oracle: counts, offsets, row_src and dest_row bit-exact.
Inputs are expert ids from the oracle's routing or from a seeded generator, never from the GPU."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def _check(layer, ids_np):
    p = bm.permute(layer, torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).cuda())
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    ref = oracle.permute(ids_np.astype(np.int32), layer["n_experts"])
    for key in ("counts", "offsets", "row_src", "dest_row"):
        np.testing.assert_array_equal(p[key].cpu().numpy(), ref[key], err_msg=key)
    return ref


@pytest.mark.parametrize("name", ["tiny", "mid_a", "mid_b", "mid_c", "mid_skew", "mid_big_expert"])
def test_permute_oracle_ids(name):
    wl = bs.get(name)
    case = parity.Case(wl)
    _check(case.layer, case.oracle_route()["ids"])


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (255, 8, 256), (257, 8, 256), (4096, 8, 256), (65536, 8, 256),
                                   (1000, 1, 4), (3000, 16, 64), (777, 3, 5)])
def test_permute_random_ids(T, k, E):
    rng = np.random.default_rng(T * 31 + k)
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k]  # k distinct experts per token
    layer = dict(hidden=64, inter=64, n_experts=E, n_groups=1, topk_groups=1, topk=k, group_topn=1, routed_scale=1.0)
    _check(layer, ids)


def test_permute_extreme_skew():
    """Every token picks experts 0..7: 248 experts stay empty, 8 take all T rows."""
    T = 5000
    ids = np.tile(np.arange(8), (T, 1))
    layer = bs.WORKLOADS["prefill"].layer
    ref = _check(layer, ids)
    assert (ref["counts"][8:] == 0).all() and (ref["counts"][:8] == T).all()


def test_permute_zero_tokens():
    layer = bs.WORKLOADS["prefill"].layer
    p = bm.permute(layer, torch.zeros(0, 8, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert p["counts"].sum().item() == 0 and p["offsets"].abs().sum().item() == 0


def test_permute_bad_index_sets_status():
    layer = bs.WORKLOADS["prefill"].layer
    ids = torch.zeros(10, 8, dtype=torch.int32)
    ids[:] = torch.arange(8)
    ids[3, 5] = 300  # outside [0, 256)
    bm.permute(layer, ids.cuda())
    assert bm.device_status() == bm.ERR_BAD_INDEX
    assert bm.device_status() == bm.OK  # cleared by the read


def test_permute_deterministic():
    rng = np.random.default_rng(1)
    ids = torch.from_numpy(np.argsort(rng.random((20000, 256)), axis=1)[:, :8].astype(np.int32)).cuda()
    layer = bs.WORKLOADS["prefill"].layer
    a = bm.permute(layer, ids)
    b = bm.permute(layer, ids)
    for k in a:
        assert torch.equal(a[k], b[k])

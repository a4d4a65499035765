"""The native FP8 path (beam_moe_experts_mxfp8 / beam_moe_forward_mxfp8): MXFP8 expert weights times
MXFP8 activations on block-scaled tensor cores (tcgen05.mma kind::mxf8f6f4), against the oracle's
block-scaled FP8 expert (oracle.expert_mlp_mx8: x and h quantised per row in blocks of 32, FP64 on the
dequantised values) on the same checkpoint codes.

Protocol as for bf16 (tests/parity.py): routing bit-exact outside near-ties, outputs under compare_y.
The GPU quantises h from FP32 values, the oracle from FP64 ones; an E4M3 code can differ where the two
straddle a rounding midpoint (a few in 10^5 elements, one E4M3 step of one of the 2560 terms of an
output), which the output bound absorbs.
"""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
import oracle
from tests import fullsize, parity

pytestmark = pytest.mark.gpu

SMALL = ["mid_a", "mid_b", "mid_skew", "mid_big_expert", "beam_small_T"]  # hidden, inter multiples of 128


class Mx8Case(parity.Case):
    def __init__(self, wl, weights=None, w8=None):
        super().__init__(wl, weights=weights)
        self.w8 = bs.quantize_experts(self.wg, self.wu, self.wd) if w8 is None else w8

    def fetch(self, e: int):
        return tuple(oracle.dequant_mxfp8(self.w8["q_" + n][e].cpu().numpy(), self.w8["s_" + n][e].cpu().numpy())
                     for n in ("gate", "up", "down"))

    def oracle_y(self, ids, w, tokens):
        return oracle.experts_tokens_mx8(np.ascontiguousarray(self.x_bits[tokens]), ids[tokens], w[tokens],
                                         self.fetch, self.layer["n_experts"], self.layer["routed_scale"])


def _case(name, bank):
    wl = bs.get(name)
    if wl.expert_device == "cuda":
        return Mx8Case(wl, weights=bank.gpu, w8=bank.fp8())
    return Mx8Case(wl)


def _experts(case, ids_np, w_np, w8):
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).cuda()
    w = torch.from_numpy(np.ascontiguousarray(w_np, dtype=np.float32)).cuda()
    y = bm.experts_mxfp8(case.layer, case.x, ids, w, w8)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    return y.float().cpu().numpy()


@pytest.mark.parametrize("name", SMALL)
def test_mxfp8_experts_small(name, bank):
    case = _case(name, bank)
    r = case.oracle_route()
    y = _experts(case, r["ids"], r["weight"], case.w8)
    st = parity.compare_y(y, case.oracle_y(r["ids"], r["weight"], np.arange(case.T)), name)
    print(f"{name}: {st}")


@pytest.mark.parametrize("name", ["mid_b", "beam_small_T"])
def test_mxfp8_forward_small(name, bank):
    case = _case(name, bank)
    y, ids, w = bm.forward_mxfp8(case.layer, case.x, case.w_router, case.bias, case.w8, return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y, ids, w = y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = np.arange(case.T)
    yo = parity.oracle_y_checked(r, st, ids, tok, case.oracle_y(r["ids"], r["weight"], tok), case.oracle_y)
    print(f"{name}: {parity.compare_y(y, yo, name)}")


@pytest.mark.parametrize("name", list(fullsize.SAMPLE_LOWP))
def test_mxfp8_forward_full_size(name, bank):
    case = bank.case(name)
    y, ids, w = bm.forward_mxfp8(case.layer, case.x, case.w_router, case.bias, bank.fp8(), return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y, ids, w = y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()
    assert np.isfinite(y).all()
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = fullsize.sample(name, "mxfp8")
    yo = parity.oracle_y_checked(r, st, ids, tok, bank.oracle_y("mxfp8", name), bank.y_of("mxfp8", name))
    print(f"{name}: {len(tok)} tokens: {parity.compare_y(y[tok], yo, name)}")


def test_mxfp8_experts_equal_forward_and_deterministic(bank):
    case = bank.case("prefill")
    y1, ids, w = bm.forward_mxfp8(case.layer, case.x, case.w_router, case.bias, bank.fp8(), return_routing=True)
    y2 = bm.experts_mxfp8(case.layer, case.x, ids, w, bank.fp8())
    y3 = bm.forward_mxfp8(case.layer, case.x, case.w_router, case.bias, bank.fp8())
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))


def test_mxfp8_rejects_shapes_not_multiple_of_128():
    wl = bs.get("mid_c")  # hidden 320, inter 192
    case = Mx8Case(wl)
    with pytest.raises(bm.BeamMoeError) as e:
        bm.forward_mxfp8(case.layer, case.x, case.w_router, case.bias, case.w8)
    assert e.value.code == bm.ERR_INVALID_CONFIG

"""The 4-bit path (beam_moe_experts_w4a4 / beam_moe_forward_w4a4): NVFP4 expert weights times NVFP4
activations on block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4), against the oracle's 4-bit
expert (oracle.expert_mlp_w4a4: x quantised per token with a power-of-two scale, h per row with scale
1, FP64 on the dequantised values) on the same checkpoint codes.

Protocol as for bf16 (tests/parity.py): routing bit-exact outside near-ties, outputs under compare_y.
x's codes are decided identically on both sides (exact power-of-two scales, single roundings of
bf16 values).  h is quantised from FP32 values on the GPU and from FP64 ones in the oracle: where an
E2M1 code or a block's E4M3 scale is decided within EPS (relative to the block) of a rounding
boundary, either result is correct, and the oracle's envelope of those alternatives (|W_down| times
the change of h~, through the combine) is added to the bound as slack; its size is printed.
"""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
import oracle
from tests import fullsize, parity

pytestmark = pytest.mark.gpu

# relative error of the GPU's FP32 h (tensor-core FP32 accumulation over up to 5120 products, SwiGLU
# in FP32) that the near-boundary envelope allows for
EPS = 3e-5

SMALL = ["mid_b", "mid_big_expert", "beam_small_T"]  # hidden, inter multiples of 256


class W4Case(parity.Case):
    def __init__(self, wl, weights=None, w4=None):
        super().__init__(wl, weights=weights)
        self.w4 = bs.quantize_experts_nvfp4(self.wg, self.wu, self.wd) if w4 is None else w4

    def fetch64(self, e: int):
        return tuple(oracle.dequant_nvfp4(self.w4["q_" + n][e].cpu().numpy(), self.w4["s_" + n][e].cpu().numpy(),
                                          float(self.w4["g_" + n][e].cpu())) for n in ("gate", "up", "down"))

    def oracle_y(self, ids, w, tokens, eps=None):
        return oracle.experts_tokens_w4a4(np.ascontiguousarray(self.x_bits[tokens]), ids[tokens], w[tokens],
                                          self.fetch64, self.layer["n_experts"], self.layer["routed_scale"], eps)


def _case(name, bank):
    wl = bs.get(name)
    if wl.expert_device == "cuda":
        return W4Case(wl, weights=bank.gpu, w4=bank.nvfp4())
    return W4Case(wl)


@pytest.mark.parametrize("name", SMALL)
def test_w4a4_experts_small(name, bank):
    case = _case(name, bank)
    r = case.oracle_route()
    ids = torch.from_numpy(np.ascontiguousarray(r["ids"], dtype=np.int32)).cuda()
    w = torch.from_numpy(np.ascontiguousarray(r["weight"], dtype=np.float32)).cuda()
    y = bm.experts_w4a4(case.layer, case.x, ids, w, case.w4)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    yo, env = case.oracle_y(r["ids"], r["weight"], np.arange(case.T), EPS)
    st = parity.compare_y(y.float().cpu().numpy(), yo, name, slack=env)
    print(f"{name}: {st}")


@pytest.mark.parametrize("name", list(fullsize.SAMPLE_LOWP))
def test_w4a4_forward_full_size(name, bank):
    case = bank.case(name)
    y, ids, w = bm.forward_w4a4(case.layer, case.x, case.w_router, case.bias, bank.nvfp4(), return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y, ids, w = y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()
    assert np.isfinite(y).all()
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = fullsize.sample(name, "w4a4")
    assert st["set_equal"][tok].all()  # (no near-tie tokens at decode/prefill: the envelope is per oracle set)
    yo, env = bank.oracle_y("w4a4", name)
    print(f"{name}: {len(tok)} tokens: {parity.compare_y(y[tok], yo, name, slack=env)}")


def test_w4a4_deterministic_and_rejects_shapes(bank):
    case = bank.case("decode")
    a = bm.forward_w4a4(case.layer, case.x, case.w_router, case.bias, bank.nvfp4())
    b = bm.forward_w4a4(case.layer, case.x, case.w_router, case.bias, bank.nvfp4())
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    wl = bs.get("mid_a")  # hidden 512, inter 384
    small = W4Case(wl)
    with pytest.raises(bm.BeamMoeError) as e:
        bm.forward_w4a4(small.layer, small.x, small.w_router, small.bias, small.w4)
    assert e.value.code == bm.ERR_INVALID_CONFIG

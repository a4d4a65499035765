"""The MoE sublayer on the residual stream (beam_moe_block_forward) vs the oracle's block step:
pre-norm (RMSNorm, bf16 activation), block, post-norm, scaled residual update ("Welcome Beam" page,
section "Residual Stream").

Protocol, derived from the arithmetic:
  * u (the pre-norm output) is computed in FP32 on the GPU and in FP64 by the oracle, then rounded to
    bf16; the two roundings can differ by one ulp where the exact value lies within FP32 error of a
    bf16 midpoint (a few elements in 10^4).  u must match within one ulp everywhere.
  * one ulp on one element of u moves a router score by at most ~2e-5 at these scales
    (|W_r| ~ 0.014, |u| ~ 3, ulp 2^-8 |u|, sigmoid slope <= 1/4), so routing on the block is compared
    with a 1e-4 decision margin instead of 1e-6, and the normalised weights (scores / their sum) within
    1e-4 instead of 1e-6; excluded tokens are still checked for validity.
  * stream_out on every token whose expert set matches: |err| <= 2e-2 * RMS(z) / sqrt(k) + half a bf16
    ulp of the oracle value, z the post-norm block output (RMS ~ 1), i.e. the block tolerance carried
    through the residual weight.
"""
import math

import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

BLOCK_MARGIN = 1e-4


def _norm_weights(H, seed):
    rng = np.random.default_rng(seed)
    return (1 + 0.1 * rng.normal(size=H)).astype(np.float32), (1 + 0.1 * rng.normal(size=H)).astype(np.float32)


def _run(case, step, tokens=None, in_place=False):
    H = case.layer["hidden"]
    g_pre, g_post = _norm_weights(H, case.wl.seed)
    s_in = case.x.clone()
    u = torch.empty_like(s_in)
    ids = torch.empty(case.T, case.layer["topk"], dtype=torch.int32, device="cuda")
    w = torch.empty(case.T, case.layer["topk"], dtype=torch.float32, device="cuda")
    out = s_in if in_place else None
    out = bm.block_forward(case.layer, s_in, torch.from_numpy(g_pre).cuda(), torch.from_numpy(g_post).cuda(), 1e-6,
                           step, case.w_router, case.bias, case.wg, case.wu, case.wd, stream_out=out, u=u, ids=ids,
                           w=w)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    ob = oracle.block_forward(case.x_bits, g_pre.astype(np.float64), g_post.astype(np.float64), 1e-6, step,
                              case.w_router_np, case.bias_np, case.fetch, case.layer, tokens)
    return out, u, ids, w, ob


def _check(case, step, tokens=None, in_place=False):
    out, u, ids, w, ob = _run(case, step, tokens, in_place)
    # pre-norm output: within one bf16 ulp
    ug = oracle.bf16_bits_to_f64(oracle.bf16_bits(u))
    uo = oracle.bf16_bits_to_f64(ob["u_bits"])
    ulp = 2 * parity.half_ulp_bf16(uo)
    assert np.all(np.abs(ug - uo) <= ulp * (1 + 1e-12)), "pre-norm output beyond one bf16 ulp"
    frac_diff = float((ug != uo).mean())
    assert frac_diff < 1e-3
    st = parity.compare_routing(ob["route"], case.layer, ids.cpu().numpy(), w.cpu().numpy(), case.bias_np,
                                margin_tol=BLOCK_MARGIN, weight_tol=BLOCK_MARGIN)
    tok = ob["tokens"]
    keep = st["set_equal"][tok]
    og = oracle.bf16_bits_to_f64(oracle.bf16_bits(out))[tok][keep]
    oo = ob["out"][keep]
    s64 = oracle.bf16_bits_to_f64(case.x_bits)[tok][keep]
    z = (oo - math.sqrt((step - 1) / step) * s64) * math.sqrt(step)
    rms_z = float(np.sqrt((z ** 2).mean()))
    err = np.abs(og - oo) - parity.half_ulp_bf16(oo)
    tol = 2e-2 * rms_z / math.sqrt(step)
    assert err.max() <= tol, f"stream_out error {err.max():.3g} > {tol:.3g}"
    print(f"{case.wl.name} k={step}: u ulp diffs {frac_diff:.2e}, excluded {st['n_excluded']}, "
          f"max excess {err.max() / (rms_z / math.sqrt(step)):.4f} x RMS(z)/sqrt(k)")


@pytest.mark.parametrize("name", ["mid_a", "mid_b", "mid_c", "mid_skew"])
@pytest.mark.parametrize("step", [7, 105])
def test_block_small(name, step):
    _check(parity.Case(bs.get(name)), step)


def test_block_beam_small_T(beam_weights):
    _check(parity.Case(bs.get("beam_small_T"), weights=beam_weights), 9)


def test_block_prefill_sampled(bank):
    wl = bs.get("prefill")
    _check(bank.case("prefill"), 11, tokens=bs.sample_tokens(wl, 64))


def test_block_in_place_equals_out_of_place():
    case = parity.Case(bs.get("mid_b"))
    a = _run(case, 5)[0].clone()
    b = _run(case, 5, in_place=True)[0]
    assert torch.equal(a, b)

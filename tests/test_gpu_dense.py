"""Dense SwiGLU MLP (beam_moe_dense_swiglu) vs the oracle's SwiGLU expert applied to every row
("The first 3 layers use a dense SwiGLU MLP": 'Welcome Beam' page, section 'Mixture of Experts')."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def _check(name, n_sample=None):
    wl = bs.get(name)
    x = bs.make_x(wl)
    wg, wu, wd = (t[0] for t in bs.make_experts(wl))
    y = bm.dense_swiglu(x.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    tok = np.arange(wl.T) if n_sample is None else bs.sample_tokens(wl, n_sample)
    xb = oracle.bf16_bits(x)
    yo = oracle.expert_mlp(np.ascontiguousarray(xb[tok]), oracle.bf16_bits(wg), oracle.bf16_bits(wu),
                           oracle.bf16_bits(wd))
    st = parity.compare_y(y.float().cpu().numpy()[tok], yo, name)
    print(f"{name}: {st}")


def test_dense_mid():
    _check("dense_mid")


def test_dense_beam_prefill_sampled():
    _check("dense_prefill", n_sample=12)


def test_dense_single_and_ragged_tokens():
    for T in (1, 7, 65):
        wl = bs.get("dense_mid").with_T(T)
        x = bs.make_x(wl)
        wg, wu, wd = (t[0] for t in bs.make_experts(wl))
        y = bm.dense_swiglu(x.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
        yo = oracle.expert_mlp(oracle.bf16_bits(x), oracle.bf16_bits(wg), oracle.bf16_bits(wu), oracle.bf16_bits(wd))
        parity.compare_y(y.float().cpu().numpy(), yo, f"T={T}")

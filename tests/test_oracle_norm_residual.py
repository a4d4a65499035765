"""Pins of the oracle's sublayer norm and scaled residual ("Welcome Beam" page, section "Residual
Stream": every sublayer is normalised before and after; at step k the stream keeps weight
sqrt((k-1)/k) and the sublayer output gets 1/sqrt(k); the embedding is step 1; "after all 104
additions, every sublayer output and the input embedding carry the same weight")."""
import math

import numpy as np
import torch

import beam_synth as bs
import oracle


def test_rmsnorm_matches_torch_float64():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(7, 320)) * 3
    g = rng.normal(size=320)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (320,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-13)


def test_rmsnorm_closed_forms():
    H = 64
    c = 3.0
    out = oracle.rmsnorm(np.full((1, H), c), np.full(H, 2.0), 0.25)
    np.testing.assert_allclose(out, 2.0 * c / math.sqrt(c * c + 0.25), rtol=1e-15)
    x = np.random.default_rng(2).normal(size=(3, H))
    np.testing.assert_allclose(oracle.rmsnorm(x * 1e3, np.ones(H), 0.0), oracle.rmsnorm(x, np.ones(H), 0.0),
                               rtol=1e-13)
    r = oracle.rmsnorm(x, np.ones(H), 0.0)
    np.testing.assert_allclose(np.sqrt((r ** 2).mean(1)), 1.0, rtol=1e-14)


def test_residual_weights_are_unit_norm():
    for k in (2, 3, 7, 105):
        keep = oracle.scaled_residual(np.ones((1, 1)), np.zeros((1, 1)), k)[0, 0]
        add = oracle.scaled_residual(np.zeros((1, 1)), np.ones((1, 1)), k)[0, 0]
        assert math.isclose(keep * keep + add * add, 1.0, rel_tol=1e-15)
        assert math.isclose(add, 1 / math.sqrt(k), rel_tol=1e-15)


def test_every_addition_carries_equal_weight_after_104_steps():
    """Embedding (step 1) then sublayers k = 2..105: the final stream is (e + sum z_k) / sqrt(105)."""
    rng = np.random.default_rng(3)
    e = rng.normal(size=(4, 16))
    zs = rng.normal(size=(104, 4, 16))
    s = e.copy()
    for k in range(2, 106):
        s = oracle.scaled_residual(s, zs[k - 2], k)
    np.testing.assert_allclose(s, (e + zs.sum(0)) / math.sqrt(105), rtol=1e-12, atol=1e-12)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(4)
    v = rng.normal(size=20000) * np.exp2(rng.integers(-20, 20, size=20000))
    bits = oracle.f64_to_bf16_bits(v)
    r = oracle.bf16_bits_to_f64(bits)
    # the neighbours one bf16 ulp away are never closer
    up = oracle.bf16_bits_to_f64((bits + 1).astype(np.uint16))
    dn = oracle.bf16_bits_to_f64((bits - 1).astype(np.uint16))
    assert np.all(np.abs(r - v) <= np.abs(up - v)) and np.all(np.abs(r - v) <= np.abs(dn - v))
    # exact ties go to the even significand: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    t = oracle.f64_to_bf16_bits(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)]))
    assert t.tolist() == [0x3F80, 0x3F82, 0xBF80]


def test_block_forward_composition():
    """Pre-norm -> MoE block -> post-norm -> residual, against the pinned pieces composed in numpy."""
    wl = bs.get("mid_a").with_T(24)
    x = bs.make_x(wl)
    W = bs.make_router(wl)
    wg, wu, wd = bs.make_experts(wl, "cpu")
    fetch = lambda e: (oracle.bf16_bits(wg[e]), oracle.bf16_bits(wu[e]), oracle.bf16_bits(wd[e]))  # noqa: E731
    rng = np.random.default_rng(5)
    g_pre, g_post = 1 + 0.1 * rng.normal(size=wl.hidden), 1 + 0.1 * rng.normal(size=wl.hidden)
    sb = oracle.bf16_bits(x)
    b = oracle.block_forward(sb, g_pre, g_post, 1e-6, 7, W.numpy(), None, fetch, wl.layer)
    s64 = oracle.bf16_bits_to_f64(sb)
    u = torch.nn.functional.rms_norm(torch.from_numpy(s64), (wl.hidden,), torch.from_numpy(g_pre), eps=1e-6)
    assert np.array_equal(b["u_bits"], oracle.f64_to_bf16_bits(u.numpy()))
    y = oracle.forward(b["u_bits"], W.numpy(), None, fetch, wl.layer)["y"]
    z = torch.nn.functional.rms_norm(torch.from_numpy(y), (wl.hidden,), torch.from_numpy(g_post), eps=1e-6).numpy()
    np.testing.assert_allclose(b["out"], math.sqrt(6 / 7) * s64 + z / math.sqrt(7), rtol=1e-12, atol=1e-12)
